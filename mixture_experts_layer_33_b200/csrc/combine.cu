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
// loaded once, one slot per lane, turned into a source row per slot and
// broadcast by shuffles; the rows of four slots are loaded before any is
// summed, so a token's loads overlap instead of queueing one behind the
// other. Expert outputs arrive in the layer dtype; the sum runs in fp32 in
// slot order (no atomics, so the output is bitwise deterministic) and is
// rounded once. `residual` may alias `y` (the forward pass writes
// x + shared(x) into y first).
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kBatch = 4;  // slots whose rows are in flight together

// 8 consecutive elements held raw until they are summed.
template <typename T> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
  uint4 u;
  __device__ __forceinline__ void load(const __nv_bfloat16 *p) { u = *reinterpret_cast<const uint4 *>(p); }
  __device__ __forceinline__ void fma_into(float wgt, float (&acc)[8]) const {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      acc[2 * i] = fmaf(wgt, f.x, acc[2 * i]);
      acc[2 * i + 1] = fmaf(wgt, f.y, acc[2 * i + 1]);
    }
  }
};
template <> struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float *p) {
    a = *reinterpret_cast<const float4 *>(p);
    b = *reinterpret_cast<const float4 *>(p + 4);
  }
  __device__ __forceinline__ void fma_into(float wgt, float (&acc)[8]) const {
    acc[0] = fmaf(wgt, a.x, acc[0]); acc[1] = fmaf(wgt, a.y, acc[1]);
    acc[2] = fmaf(wgt, a.z, acc[2]); acc[3] = fmaf(wgt, a.w, acc[3]);
    acc[4] = fmaf(wgt, b.x, acc[4]); acc[5] = fmaf(wgt, b.y, acc[5]);
    acc[6] = fmaf(wgt, b.z, acc[6]); acc[7] = fmaf(wgt, b.w, acc[7]);
  }
};

// (a0, a1) = softmax(Wc . x) of a mixed constant expert, Wc = rows 1..2 of
// its [3, d] block `vrow`; fp32 dot products by the whole warp. Out of
// line: the rare path keeps its registers to itself.
template <typename T>
__device__ __noinline__ float2 const_mix_weights(const T *xr, const T *vrow, int d) {
  const int lane = threadIdx.x & 31;
  float z0 = 0.f, z1 = 0.f;
  for (int c = lane * 8; c < d; c += 256) {
    float xv[8], w0[8], w1[8];
    load8(xr + c, xv);
    load8(vrow + d + c, w0);
    load8(vrow + 2 * d + c, w1);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      z0 = fmaf(xv[i], w0[i], z0);
      z1 = fmaf(xv[i], w1[i], z1);
    }
  }
  z0 = warp_sum(z0);
  z1 = warp_sum(z1);
  const float mz = fmaxf(z0, z1);
  const float e0 = expf(z0 - mz), e1 = expf(z1 - mz);
  return make_float2(e0 / (e0 + e1), e1 / (e0 + e1));
}

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
    float x_coef = 0.f;  // weight of x_s from mixed constant experts
    for (int j0 = a0; j0 < a1; j0 += 32) {
      // Lane j holds slot j0 + j: its weight and the first element of its
      // source row (the expert's output row, x for an identity expert, the
      // learned vector for a constant expert), or none (zero expert, a row
      // the dispatch dropped, or an id it flagged).
      const T *m_src = nullptr;
      float m_w = 0.f;
      bool m_mix = false;
      if (j0 + lane < a1) {
        const int asg = ec ? a.tok_assign[j0 + lane] : j0 + lane;
        const int e = ec ? (int)((asg / a.C) % a.E) : a.sel[asg];
        const int row = a.row_of[asg];
        const float wv = a.w[asg];
        if (e >= 0 && e < a.E) {
          const int kind = kinds.kind[e];
          if (kind == MOE_HEAVY) {
            if (row >= 0) m_src = yp + (size_t)row * a.d;
          } else if (kind == MOE_IDENTITY) {
            m_src = x + (size_t)s * a.d;
          } else if (kind == MOE_CONST) {
            m_src = cv + (size_t)kinds.cidx[e] * (a.const_mix ? 3 : 1) * a.d;
            m_mix = a.const_mix != 0;
          }
          m_w = wv;
        }
      }
      // Mixed constant experts: the warp forms (a0, a1) = softmax(Wc x_s)
      // for each such slot; the slot keeps w * a1 on v, and w * a0 joins
      // the coefficient of x_s, added after the slots.
      for (unsigned mm = __ballot_sync(0xffffffffu, m_mix); mm; mm &= mm - 1u) {
        const int j = __ffs(mm) - 1;
        const T *vrow = reinterpret_cast<const T *>(
            __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(m_src), j));
        const float2 mix = const_mix_weights(x + (size_t)s * a.d, vrow, a.d);
        const float a0 = mix.x, a1 = mix.y;
        const float wj = __shfl_sync(0xffffffffu, m_w, j);
        x_coef = fmaf(wj, a0, x_coef);
        if (lane == j) m_w = wj * a1;
      }
      const int nj = min(32, a1 - j0);
      for (int jb = 0; jb < nj; jb += kBatch) {
        Raw8<T> raw[kBatch];
        const T *src[kBatch];
        float wgt[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int j = (jb + u) & 31;
          src[u] = reinterpret_cast<const T *>(
              __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(m_src), j));
          wgt[u] = __shfl_sync(0xffffffffu, m_w, j);
          if (jb + u >= nj || !live) src[u] = nullptr;
          if (src[u]) raw[u].load(src[u] + c0);
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u)
          if (src[u]) raw[u].fma_into(wgt[u], acc);
      }
    }
    if (live && x_coef != 0.f) {
      Raw8<T> xs;
      xs.load(x + (size_t)s * a.d + c0);
      xs.fma_into(x_coef, acc);
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
