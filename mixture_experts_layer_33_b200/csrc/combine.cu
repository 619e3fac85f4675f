// Combine back to token order, fused with the routing-weight scale, the
// zero-computation experts, the shared expert and the residual add.
//
// DICE: Staleness-Centric Optimizations for Parallel Diffusion MoE
// Inference, "Conditional Communication": a token's output is the sum of
// its experts' outputs weighted by its routing scores.
// MMOE: Modernizing Diffusion Transformers with Efficient Expert Design,
// "MoE++ expert layer": identity experts return x, zero experts return 0,
// constant experts return a learned vector; "shared experts": one dense
// expert is always active (added with weight 1).
//
// One warp per (token, 256-feature chunk); each lane owns 8 consecutive
// features and reads them with 16-byte loads; a token's slot metadata is
// loaded once, one slot per lane, and broadcast by shuffles. Expert outputs
// arrive in the layer dtype; the sum runs in fp32 in slot order (no atomics,
// so the output is bitwise deterministic) and is rounded once. `residual`
// may alias `y` (the forward pass writes x + shared(x) into y first).
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kThreads) combine_kernel(CombineArgs a, KindTable kinds) {
  const T *__restrict__ x = static_cast<const T *>(a.x);
  const T *res = static_cast<const T *>(a.residual);  // may alias y
  const T *__restrict__ cv = static_cast<const T *>(a.const_vecs);
  const T *__restrict__ yp = static_cast<const T *>(a.y_perm);
  const T *__restrict__ ysh = static_cast<const T *>(a.y_shared);
  T *y = static_cast<T *>(a.y);
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * kThreads + threadIdx.x) >> 5;
  const int nw = (gridDim.x * kThreads) >> 5;
  const bool ec = a.routing == MOE_EXPERT_CHOICE;
  const int chunks = (a.d + 255) / 256;
  const int64_t items = (int64_t)a.T * chunks;
  // One warp per (token, 256-feature chunk); each lane owns 8 features.
  for (int64_t it = gw; it < items; it += nw) {
    const int s = (int)(it / chunks);
    const int c0 = (int)(it - (int64_t)s * chunks) * 256 + lane * 8;
    const bool live = c0 < a.d;
    int a0, a1;
    if (ec) { a0 = a.tok_ptr[s]; a1 = a.tok_ptr[s + 1]; }
    else { a0 = s * a.k; a1 = a0 + a.k; }
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    if (live && res) load8(res + (size_t)s * a.d + c0, acc);
    if (live && ysh) {
      float t[8];
      load8(ysh + (size_t)s * a.d + c0, t);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += t[i];
    }
    for (int j0 = a0; j0 < a1; j0 += 32) {
      // Lane j holds the metadata of slot j0 + j; the slot loop broadcasts it.
      int m_kind = MOE_ZERO, m_row = -1, m_ci = 0;
      float m_w = 0.f;
      if (j0 + lane < a1) {
        const int asg = ec ? a.tok_assign[j0 + lane] : j0 + lane;
        const int e = ec ? (int)((asg / a.C) % a.E) : a.sel[asg];
        if (e >= 0 && e < a.E) {  // out-of-range ids were flagged by dispatch
          m_kind = kinds.kind[e];
          m_w = a.w[asg];
          m_row = m_kind == MOE_HEAVY ? a.row_of[asg] : -1;
          m_ci = kinds.cidx[e];
        }
      }
      const int nj = min(32, a1 - j0);
#pragma unroll 2
      for (int j = 0; j < nj; ++j) {
        const int kind = __shfl_sync(0xffffffffu, m_kind, j);
        const float wgt = __shfl_sync(0xffffffffu, m_w, j);
        const int row = __shfl_sync(0xffffffffu, m_row, j);
        const int ci = __shfl_sync(0xffffffffu, m_ci, j);
        if (!live) continue;
        float t[8];
        if (kind == MOE_HEAVY) {
          if (row < 0) continue;
          load8(yp + (size_t)row * a.d + c0, t);
        } else if (kind == MOE_IDENTITY) {
          load8(x + (size_t)s * a.d + c0, t);
        } else if (kind == MOE_CONST) {
          load8(cv + (size_t)ci * a.d + c0, t);
        } else {
          continue;  // zero expert: contributes nothing
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(wgt, t[i], acc[i]);
      }
    }
    if (live) store8(y + (size_t)s * a.d + c0, acc);
  }
}

}  // namespace

int launch_combine(const CombineArgs &a, const KindTable &kinds, cudaStream_t stream) {
  if (a.T == 0) return MOE_OK;
  const int64_t items = (int64_t)a.T * ((a.d + 255) / 256);
  int64_t blocks = (items + (kThreads / 32) - 1) / (kThreads / 32);
  const int64_t cap = (int64_t)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  const int grid = (int)blocks;
  if (a.dtype == MOE_BF16) combine_kernel<__nv_bfloat16><<<grid, kThreads, 0, stream>>>(a, kinds);
  else combine_kernel<float><<<grid, kThreads, 0, stream>>>(a, kinds);
  return last_launch_status();
}

}  // namespace moe
