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
// One warp per token; each lane owns 8 consecutive features per pass and
// reads them with 16-byte loads. The sum runs in fp32 in slot order (no
// atomics, so the output is bitwise deterministic) and is rounded once.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kThreads) combine_kernel(CombineArgs a, KindTable kinds) {
  const T *x = static_cast<const T *>(a.x);
  const T *res = static_cast<const T *>(a.residual);
  const T *cv = static_cast<const T *>(a.const_vecs);
  T *y = static_cast<T *>(a.y);
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * kThreads + threadIdx.x) >> 5;
  const int nw = (gridDim.x * kThreads) >> 5;
  const bool ec = a.routing == MOE_EXPERT_CHOICE;
  for (int s = gw; s < a.T; s += nw) {
    int a0, a1;
    if (ec) { a0 = a.tok_ptr[s]; a1 = a.tok_ptr[s + 1]; }
    else { a0 = s * a.k; a1 = a0 + a.k; }
    for (int c0 = lane * 8; c0 < a.d; c0 += 256) {
      float acc[8];
      if (res) load8(res + (size_t)s * a.d + c0, acc);
      else {
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      }
      if (a.y_shared) {
        float t[8];
        load8(a.y_shared + (size_t)s * a.d + c0, t);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += t[i];
      }
      for (int j = a0; j < a1; ++j) {
        const int asg = ec ? a.tok_assign[j] : j;
        const int e = ec ? (int)((asg / a.C) % a.E) : a.sel[asg];
        if (e < 0 || e >= a.E) continue;  // flagged by dispatch
        const float wgt = a.w[asg];
        const int kind = kinds.kind[e];
        float t[8];
        if (kind == MOE_HEAVY) {
          const int row = a.row_of[asg];
          if (row < 0) continue;
          load8(a.y_perm + (size_t)row * a.d + c0, t);
        } else if (kind == MOE_IDENTITY) {
          load8(x + (size_t)s * a.d + c0, t);
        } else if (kind == MOE_CONST) {
          load8(cv + (size_t)kinds.cidx[e] * a.d + c0, t);
        } else {
          continue;  // zero expert: contributes nothing
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(wgt, t[i], acc[i]);
      }
      store8(y + (size_t)s * a.d + c0, acc);
    }
  }
}

}  // namespace

int launch_combine(const CombineArgs &a, const KindTable &kinds, cudaStream_t stream) {
  if (a.T == 0) return MOE_OK;
  int blocks = (a.T + (kThreads / 32) - 1) / (kThreads / 32);
  int cap = num_sms() * 8;
  if (blocks > cap) blocks = cap;
  if (a.dtype == MOE_BF16) combine_kernel<__nv_bfloat16><<<blocks, kThreads, 0, stream>>>(a, kinds);
  else combine_kernel<float><<<blocks, kThreads, 0, stream>>>(a, kinds);
  return last_launch_status();
}

}  // namespace moe
