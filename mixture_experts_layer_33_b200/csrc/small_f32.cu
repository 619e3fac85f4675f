// The whole MoE layer for a small fp32 token-choice layer in one launch:
// one CTA per token runs its router row, softmax and top-k, then each of
// its experts' MLP with the weights read from L2, and the weighted combine
// with the residual.
//
// EC-DiT: Scaling Diffusion Transformers with Adaptive Expert-Choice
// Routing, section 3 (Token-Choice routing): affinities are the softmax of
// the router logits and each token keeps its top-k experts.
// MMOE: Modernizing Diffusion Transformers with Efficient Expert Design,
// "MoE++ expert layer": heavy experts are MLPs (GELU, or SwiGLU here),
// identity experts return x, zero experts return 0, constant experts return
// a learned vector; "gating residuals": the previous layer's logits, scaled,
// join the router logits.
// DICE: Staleness-Centric Optimizations for Parallel Diffusion MoE
// Inference, "Conditional Communication": the output is the routing-score-
// weighted sum of the token's experts' outputs.
//
// A small fp32 layer (the tiny workload: 256 tokens, d = 64, 8 experts of
// 64 -> 256 -> 64) is a few tens of MFLOP: as a chain of router, dispatch,
// gather, two grouped GEMMs and combine it is bound by launch latency.
// Here every token is independent, so there is no dispatch: a token's CTA
// reads its experts' weights (L2-resident after the first CTAs) and keeps
// the hidden activations in shared memory. The per-expert row counts that
// the dispatch would report are counted with atomics, and the last CTA to
// finish turns them into the dispatch offsets.
// fp32 throughout on CUDA cores (tensor cores would take fp32 inputs as
// tf32); every sum runs in a fixed order, so the output is deterministic.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxK = 32;

// Dot products of R weight rows with the token's shared-memory vector, a
// float4 at a time (n a multiple of 4, rows and vector 16-byte aligned):
// the loads of all R rows over 8 elements are issued before their sums.
template <int R>
__device__ __forceinline__ void dot_rows(const float *const (&w)[R], const float *v, int n,
                                         float (&s)[R]) {
#pragma unroll
  for (int r = 0; r < R; ++r) s[r] = 0.f;
  int i = 0;
#pragma unroll 2
  for (; i + 8 <= n; i += 8) {
    float4 wv[R][2];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      wv[r][0] = __ldg(reinterpret_cast<const float4 *>(w[r] + i));
      wv[r][1] = __ldg(reinterpret_cast<const float4 *>(w[r] + i + 4));
    }
    const float4 a0 = *reinterpret_cast<const float4 *>(v + i);
    const float4 a1 = *reinterpret_cast<const float4 *>(v + i + 4);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      s[r] = fmaf(wv[r][0].x, a0.x, s[r]); s[r] = fmaf(wv[r][0].y, a0.y, s[r]);
      s[r] = fmaf(wv[r][0].z, a0.z, s[r]); s[r] = fmaf(wv[r][0].w, a0.w, s[r]);
      s[r] = fmaf(wv[r][1].x, a1.x, s[r]); s[r] = fmaf(wv[r][1].y, a1.y, s[r]);
      s[r] = fmaf(wv[r][1].z, a1.z, s[r]); s[r] = fmaf(wv[r][1].w, a1.w, s[r]);
    }
  }
  for (; i < n; i += 4) {
    const float4 a0 = *reinterpret_cast<const float4 *>(v + i);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float4 w0 = __ldg(reinterpret_cast<const float4 *>(w[r] + i));
      s[r] = fmaf(w0.x, a0.x, s[r]); s[r] = fmaf(w0.y, a0.y, s[r]);
      s[r] = fmaf(w0.z, a0.z, s[r]); s[r] = fmaf(w0.w, a0.w, s[r]);
    }
  }
}

// Hidden activations of up to two experts (NE) for this thread's hidden
// units, all their weight rows in flight together.
template <int NE>
__device__ __forceinline__ void hidden_units(const SmallF32Args &a, const int (&e)[2],
                                             const float *xs, float *hid) {
  const int d = a.d, h = a.h;
  const int w1_rows = a.gated ? 2 * h : h;
  for (int i = threadIdx.x; i < h; i += kThreads) {
    if (a.gated) {
      const float *w[2 * NE];
      float g[2 * NE];
#pragma unroll
      for (int q = 0; q < NE; ++q) {
        const float *W1e = a.W1 + (size_t)e[q] * w1_rows * d;
        w[2 * q] = W1e + (size_t)i * d;
        w[2 * q + 1] = W1e + (size_t)(h + i) * d;
      }
      dot_rows<2 * NE>(w, xs, d, g);
#pragma unroll
      for (int q = 0; q < NE; ++q) hid[q * h + i] = silu(g[2 * q]) * g[2 * q + 1];
    } else {
      const float *w[NE];
      float g[NE];
#pragma unroll
      for (int q = 0; q < NE; ++q) w[q] = a.W1 + ((size_t)e[q] * w1_rows + i) * d;
      dot_rows<NE>(w, xs, d, g);
#pragma unroll
      for (int q = 0; q < NE; ++q) hid[q * h + i] = gelu_erf(g[q]);
    }
  }
}

// Down projections of up to two experts, added to acc in slot order:
// G adjacent lanes per output feature.
template <int NE>
__device__ __forceinline__ void down_proj(const SmallF32Args &a, const int (&e)[2],
                                          const float (&wt)[2], const float *hid, float *acc) {
  const int d = a.d, h = a.h, tid = threadIdx.x;
  int G = kThreads / d;
  G = G >= 32 ? 32 : G >= 16 ? 16 : G >= 8 ? 8 : G >= 4 ? 4 : G >= 2 ? 2 : 1;
  const int per_pass = kThreads / G;
  const int passes = (d + per_pass - 1) / per_pass;
  const int sub = tid % G;
  for (int ps = 0; ps < passes; ++ps) {
    const int o = ps * per_pass + tid / G;
    float s[NE];
#pragma unroll
    for (int q = 0; q < NE; ++q) s[q] = 0.f;
    if (o < d) {
      const float *wrow[NE];
#pragma unroll
      for (int q = 0; q < NE; ++q) wrow[q] = a.W2 + ((size_t)e[q] * d + o) * h;
#pragma unroll 4
      for (int i = 4 * sub; i < h; i += 4 * G) {
        float4 wv[NE];
#pragma unroll
        for (int q = 0; q < NE; ++q) wv[q] = __ldg(reinterpret_cast<const float4 *>(wrow[q] + i));
#pragma unroll
        for (int q = 0; q < NE; ++q) {
          const float4 hv = *reinterpret_cast<const float4 *>(hid + q * h + i);
          s[q] = fmaf(wv[q].x, hv.x, s[q]); s[q] = fmaf(wv[q].y, hv.y, s[q]);
          s[q] = fmaf(wv[q].z, hv.z, s[q]); s[q] = fmaf(wv[q].w, hv.w, s[q]);
        }
      }
    }
#pragma unroll
    for (int q = 0; q < NE; ++q)
      for (int off = G >> 1; off > 0; off >>= 1) s[q] += __shfl_xor_sync(0xffffffffu, s[q], off);
    if (o < d && sub == 0) {
      float v = acc[o];
#pragma unroll
      for (int q = 0; q < NE; ++q) v = fmaf(wt[q], s[q], v);
      acc[o] = v;
    }
  }
}

__global__ void __launch_bounds__(kThreads) small_f32_kernel(SmallF32Args a, KindTable kinds) {
  extern __shared__ __align__(16) float sm[];
  const int d = a.d, h = a.h, E = a.E, k = a.k;
  float *xs = sm;          // [d]  the token's x row
  float *acc = xs + d;     // [d]  its output, accumulated
  float *hid = acc + d;    // [2][h]  hidden activations of the current experts
  float *zs = hid + 2 * h; // [E]  logits
  float *As = zs + E;      // [E]  affinities
  __shared__ int slot_e[kMaxK];
  __shared__ float slot_w[kMaxK];
  __shared__ int last_cta;

  const int t = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float *xrow = a.x + (size_t)t * d;
  for (int i = tid; i < d; i += kThreads) {
    xs[i] = xrow[i];
    acc[i] = a.residual ? a.residual[(size_t)t * d + i] : 0.f;
  }
  if (tid < kMaxK) { slot_e[tid] = -1; slot_w[tid] = 0.f; }
  __syncthreads();

  // Router logits z = (x W_r + bias) + scale * z_prev: a warp per expert.
  for (int e = warp; e < E; e += kWarps) {
    const float *wr = a.W_r + (size_t)e * d;
    float s = 0.f;
    for (int i = lane; i < d; i += 32) s = fmaf(xs[i], __ldg(wr + i), s);
    s = warp_sum(s);
    if (lane == 0) {
      if (a.bias) s += a.bias[e];
      if (a.zprev) s += a.zscale * a.zprev[(size_t)t * E + e];
      zs[e] = s;
    }
  }
  __syncthreads();
  // Softmax over all E experts (max-subtracted).
  if (warp == 0) {
    float m = -INFINITY;
    for (int e = lane; e < E; e += 32) m = fmaxf(m, zs[e]);
    m = warp_max(m);
    float s = 0.f;
    for (int e = lane; e < E; e += 32) {
      const float ex = expf(zs[e] - m);
      As[e] = ex;
      s += ex;
    }
    s = warp_sum(s);
    for (int e = lane; e < E; e += 32) {
      const float A = As[e] / s;
      As[e] = A;
      a.logits[(size_t)t * E + e] = zs[e];
      a.probs[(size_t)t * E + e] = A;
    }
  }
  __syncthreads();
  // Top-k on the logits by rank: expert e takes slot #{f : z_f > z_e, or
  // z_f == z_e and f < e} if that is below k (ties to the lower id).
  for (int e = tid; e < E; e += kThreads) {
    const float ze = zs[e];
    int rank = 0;
    for (int f = 0; f < E; ++f) {
      const float zf = zs[f];
      rank += (zf > ze) || (zf == ze && f < e);
    }
    if (rank < k) { slot_e[rank] = e; slot_w[rank] = As[e]; }
  }
  __syncthreads();
  if (a.renorm && tid == 0) {
    float ws = 0.f;
    for (int j = 0; j < k; ++j) ws += slot_w[j];
    for (int j = 0; j < k; ++j) slot_w[j] = slot_w[j] / ws;
  }
  __syncthreads();
  if (tid < k) {
    const int e = slot_e[tid];
    a.sel[(size_t)t * k + tid] = e;
    a.w[(size_t)t * k + tid] = slot_w[tid];
    if (e >= 0 && e < a.n_heavy) atomicAdd(a.counts + e, 1u);
  }

  // The experts, in slot order: acc = residual + sum_j w_j * E_j(x); two
  // consecutive heavy slots at a time, so both experts' weights are in
  // flight together.
  for (int j = 0; j < k;) {
    const int e0 = slot_e[j];
    const float w0 = slot_w[j];
    const int kind0 = (e0 >= 0 && e0 < E) ? kinds.kind[e0] : MOE_ZERO;
    if (kind0 == MOE_HEAVY && e0 < a.n_heavy) {
      const int e1 = j + 1 < k ? slot_e[j + 1] : -1;
      const bool two = e1 >= 0 && e1 < a.n_heavy && kinds.kind[e1] == MOE_HEAVY;
      const int ee[2] = {e0, two ? e1 : e0};
      const float ww[2] = {w0, two ? slot_w[j + 1] : 0.f};
      if (two) hidden_units<2>(a, ee, xs, hid);
      else hidden_units<1>(a, ee, xs, hid);
      __syncthreads();
      if (two) down_proj<2>(a, ee, ww, hid, acc);
      else down_proj<1>(a, ee, ww, hid, acc);
      __syncthreads();  // hid is rewritten by the next slots
      j += two ? 2 : 1;
      continue;
    }
    if (kind0 == MOE_IDENTITY) {
      for (int i = tid; i < d; i += kThreads) acc[i] = fmaf(w0, xs[i], acc[i]);
      __syncthreads();
    } else if (kind0 == MOE_CONST) {
      const float *v = a.const_vecs + (size_t)kinds.cidx[e0] * d;
      for (int i = tid; i < d; i += kThreads) acc[i] = fmaf(w0, v[i], acc[i]);
      __syncthreads();
    }
    ++j;
  }
  for (int i = tid; i < d; i += kThreads) a.y[(size_t)t * d + i] = acc[i];

  // Dispatch offsets: the last CTA to finish scans the heavy-expert counts.
  __threadfence();
  __syncthreads();
  if (tid == 0) last_cta = atomicAdd(a.counts + a.n_heavy, 1u) == gridDim.x - 1;
  __syncthreads();
  if (last_cta && tid == 0) {
    __threadfence();
    int run = 0;
    for (int e = 0; e < a.n_heavy; ++e) {
      a.offsets[e] = run;
      run += (int)__ldcg(a.counts + e);
    }
    a.offsets[a.n_heavy] = run;
  }
}

}  // namespace

bool small_f32_supported(const moe_config &c) {
  return c.dtype == MOE_F32 && c.routing == MOE_TOKEN_TOPK && c.n_shared == 0 &&
         c.const_mix == 0 && c.T >= 1 && c.T <= 1024 && c.E >= 1 && c.E <= MOE_MAX_EXPERTS &&
         c.k >= 1 && c.k <= kMaxK && c.k <= c.E && c.d >= 4 && c.d <= 1024 && c.d % 4 == 0 &&
         c.h >= 4 && c.h <= 2048 && c.h % 4 == 0;
}

size_t small_f32_zero_bytes(int n_heavy) { return (size_t)(n_heavy + 1) * 4; }

int launch_small_f32(const SmallF32Args &a, const KindTable &kinds, cudaStream_t stream) {
  if (a.T == 0) return MOE_OK;
  const size_t smem = (size_t)(2 * a.d + 2 * a.h + 2 * a.E) * sizeof(float);
  small_f32_kernel<<<a.T, kThreads, smem, stream>>>(a, kinds);
  return last_launch_status();
}

}  // namespace moe
