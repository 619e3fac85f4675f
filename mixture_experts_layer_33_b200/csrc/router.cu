// Router GEMM + softmax + token-choice top-k, fused (one kernel).
//
// EC-DiT: Scaling Diffusion Transformers with Adaptive Expert-Choice
// Routing, section 3 "Expert-Choice routing formula": the affinity of token
// s to expert i is the softmax over the E experts of (x' W_r)_{s,i}.
// MMOE: Modernizing Diffusion Transformers with Efficient Expert Design,
// "gate-residual routing": the previous expert layer's gate logits are
// added to the router logits (z = x W_r + b + scale * z_prev).
// EC-DiT section 3 "Token-Choice routing": each token keeps its top-k
// experts.
//
// bf16 path: a CTA owns 32 tokens; its 2 warps each run m16n8k16 bf16
// tensor-core MMAs (fp32 accumulate) over a 6-deep cp.async ring of x and
// W_r tiles, so x is read from HBM exactly once with many tiles in flight.
// The N dimension of this GEMM is E <= 128, far too narrow for a 128-wide
// tcgen05 tile; the kernel is bound by reading x. The logits tile is then
// parked in shared memory; for E <= 32 each thread finishes one token's
// softmax and top-k serially, for wider E each warp finishes its tokens
// with warp-shuffle softmax and warp-shuffle argmax rounds (ties to the
// lower expert id either way). Small blocks (T <= 512) use one CTA per
// token instead, with 8 warps sharing the E dot products.
// fp32 path: plain FMA dot products, one warp per token (fp32 layers are
// small and must stay exact to fp32 rounding).
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "mma_sync.cuh"

namespace moe {
namespace {

constexpr int kBK = 64;        // model-width slice per pipeline stage
constexpr int kLDS = kBK + 8;  // padded smem row (bf16): conflict-free ldmatrix
constexpr int kThreads = 128;
constexpr int kRowwiseMaxTokens = 512;  // bf16 layers this small use one CTA per token
constexpr int kMmaBM = 32;               // tokens per CTA of the MMA router (two halves of 16)
constexpr int kMmaWarps = 4;             // two 16-token halves x two K parities
constexpr int kMmaThreads = 32 * kMmaWarps;
// cp.async ring depth: up to 16 experts, twelve 64-wide slices of the
// token tile in flight per CTA (a 1152-wide tile in 1.5 round trips);
// 17-32 experts, eleven, so that two CTAs still fit on an SM; wider expert
// tiles keep six to stay within shared memory.
template <int NT>
constexpr int mma_stages() { return NT <= 2 ? 12 : NT <= 4 ? 11 : 6; }

// Softmax of one token row held by a warp: expert e = lane + 32*v.
template <int VPL>
__device__ __forceinline__ void row_softmax(const float (&z)[VPL], int E, float (&A)[VPL]) {
  const int lane = threadIdx.x & 31;
  float m = -INFINITY;
#pragma unroll
  for (int v = 0; v < VPL; ++v)
    if (lane + 32 * v < E) m = fmaxf(m, z[v]);
  m = warp_max(m);
  float s = 0.f;
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    A[v] = (lane + 32 * v < E) ? expf(z[v] - m) : 0.f;
    s += A[v];
  }
  s = warp_sum(s);
#pragma unroll
  for (int v = 0; v < VPL; ++v) A[v] = A[v] / s;
}

// Top-k of one token row held by a warp, ranked by z, ties to the lower id.
// Lane 0 writes idx_row[0..k) in rank order and w_row = A (or A / sum).
template <int VPL>
__device__ __forceinline__ void row_topk(const float (&z)[VPL], const float (&A)[VPL], int E,
                                         int k, int renorm, int32_t *idx_row, float *w_row) {
  const int lane = threadIdx.x & 31;
  bool taken[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) taken[v] = false;
  float wsum = 0.f;
  for (int r = 0; r < k; ++r) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      int e = lane + 32 * v;
      if (e < E && !taken[v] && better(z[v], e, bv, bi)) { bv = z[v]; bi = e; }
    }
    warp_argmax(bv, bi);
    float a_own = 0.f;
#pragma unroll
    for (int v = 0; v < VPL; ++v)
      if (lane + 32 * v == bi) { taken[v] = true; a_own = A[v]; }
    float a = __shfl_sync(0xffffffffu, a_own, bi & 31);
    wsum += a;
    if (lane == 0) {
      idx_row[r] = bi;
      w_row[r] = a;
    }
  }
  if (renorm && lane == 0)
    for (int r = 0; r < k; ++r) w_row[r] = w_row[r] / wsum;
}

// PARTIAL: blockIdx.y selects a slice of the model width; the CTA writes
// its partial logits to `logits` laid out [gridDim.y][T][E] and stops.
template <int NT, bool PARTIAL = false>
__global__ void __launch_bounds__(kMmaThreads)
router_bf16_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ Wr,
                   const float *__restrict__ bias, const float *__restrict__ zprev, float zscale,
                   int T, int d, int E, float *__restrict__ logits, float *__restrict__ probs,
                   int k, int renorm, int32_t *__restrict__ idx, float *__restrict__ w,
                   ZeroList zero) {
  constexpr int EP = NT * 8;
  constexpr int VPL = (EP + 31) / 32;
  constexpr int kMmaStages = mma_stages<NT>();
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __nv_bfloat16 *sX = reinterpret_cast<__nv_bfloat16 *>(smem_raw);   // [stages][kMmaBM][kLDS]
  __nv_bfloat16 *sW = sX + kMmaStages * kMmaBM * kLDS;                      // [stages][EP][kLDS]
  float *sZ = reinterpret_cast<float *>(sW + kMmaStages * EP * kLDS);    // [2][kMmaBM][EP + 1]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (PARTIAL && blockIdx.x == 0 && blockIdx.y == 0) {
#pragma unroll
    for (int l = 0; l < 3; ++l)
      for (int i = tid; i < zero.n[l]; i += kMmaThreads) zero.p[l][i] = 0;
  }
  const int t0 = blockIdx.x * kMmaBM;
  const int nk_all = (d + kBK - 1) / kBK;
  const int kb_per = PARTIAL ? (nk_all + gridDim.y - 1) / gridDim.y : nk_all;
  const int kb0 = PARTIAL ? blockIdx.y * kb_per : 0;
  const int nk = PARTIAL ? max(0, min(nk_all, kb0 + kb_per) - kb0) : nk_all;

  auto load_stage = [&](int stage, int kb) {
    const int k0 = (kb0 + kb) * kBK;
    for (int c = tid; c < kMmaBM * (kBK / 8); c += kMmaThreads) {
      int r = c >> 3, cc = c & 7, gr = t0 + r, gk = k0 + cc * 8;
      bool ok = gr < T && gk < d;
      const __nv_bfloat16 *src = x + (size_t)(ok ? gr : 0) * d + (ok ? gk : 0);
      cp_async16(sX + (stage * kMmaBM + r) * kLDS + cc * 8, src, ok);
    }
    for (int c = tid; c < EP * (kBK / 8); c += kMmaThreads) {
      int r = c >> 3, cc = c & 7, gk = k0 + cc * 8;
      bool ok = r < E && gk < d;
      const __nv_bfloat16 *src = Wr + (size_t)(ok ? r : 0) * d + (ok ? gk : 0);
      cp_async16(sW + (stage * EP + r) * kLDS + cc * 8, src, ok);
    }
  };

#pragma unroll
  for (int s = 0; s < kMmaStages - 1; ++s) {
    if (s < nk) load_stage(s, s);
    cp_async_commit();
  }

  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[n][i] = 0.f;

  for (int kb = 0; kb < nk; ++kb) {
    cp_async_wait<kMmaStages - 2>();
    __syncthreads();
    {
      int nkb = kb + kMmaStages - 1;
      if (nkb < nk) load_stage(nkb % kMmaStages, nkb);
      cp_async_commit();
    }
    const int st = kb % kMmaStages;
    // Warp w takes tokens (w & 1) * 16 .. +15 and the k16 steps of parity
    // w >> 1; the two parities' sums are added once at the end.
    const __nv_bfloat16 *tX = sX + (st * kMmaBM + (warp & 1) * 16) * kLDS;
    const __nv_bfloat16 *tW = sW + st * EP * kLDS;
#pragma unroll
    for (int kk = warp >> 1; kk < kBK / 16; kk += 2) {
      uint32_t a[4];
      ldmatrix_x4(a, tX + (lane & 15) * kLDS + kk * 16 + (lane >> 4) * 8);
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        uint32_t b[2];
        ldmatrix_x2(b, tW + (n * 8 + (lane & 7)) * kLDS + kk * 16 + ((lane >> 3) & 1) * 8);
        mma_bf16_16816(acc[n], a, b);
      }
    }
  }
  cp_async_wait<0>();

  // Park the two K parities' kMmaBM x EP sums in shared memory, then add
  // them (even + odd, the same order for every element).
  {
    const int r0 = (warp & 1) * 16 + (lane >> 2);
    float *z = sZ + (warp >> 1) * kMmaBM * (EP + 1);
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int c0 = n * 8 + (lane & 3) * 2;
      z[r0 * (EP + 1) + c0] = acc[n][0];
      z[r0 * (EP + 1) + c0 + 1] = acc[n][1];
      z[(r0 + 8) * (EP + 1) + c0] = acc[n][2];
      z[(r0 + 8) * (EP + 1) + c0 + 1] = acc[n][3];
    }
  }
  __syncthreads();
  for (int i = tid; i < kMmaBM * (EP + 1); i += kMmaThreads) sZ[i] += sZ[kMmaBM * (EP + 1) + i];
  __syncthreads();
  if (PARTIAL) {
    float *part = logits + (size_t)blockIdx.y * T * E;
    for (int i = tid; i < kMmaBM * E; i += kMmaThreads) {
      const int r = i / E, e = i - r * E;
      if (t0 + r < T) part[(size_t)(t0 + r) * E + e] = sZ[r * (EP + 1) + e];
    }
    return;
  }

  if constexpr (EP <= 32) {
    // E <= 32: four lanes per token (tid / 4 is the token, tid % 4 the
    // lane in its quad), each holding experts q, q + 4, ...; the max, the
    // sum and each top-k round reduce over the quad with two shuffles.
    // Ties go to the lower expert id.
    constexpr int PER = EP / 4;
    static_assert(EP % 4 == 0 && kMmaThreads == 4 * kMmaBM, "a quad of lanes per token");
    const int r = tid >> 2, q = tid & 3, s = t0 + r;
    const bool live = s < T;
    float z[PER], A[PER];
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int e = q + 4 * j;
      float zz = -INFINITY;
      if (e < E) {
        zz = sZ[r * (EP + 1) + e];
        if (live) {
          if (bias) zz += bias[e];
          if (zprev) zz += zscale * zprev[(size_t)s * E + e];
          logits[(size_t)s * E + e] = zz;
        }
        m = fmaxf(m, zz);
      }
      z[j] = zz;
    }
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      A[j] = q + 4 * j < E ? expf(z[j] - m) : 0.f;
      sum += A[j];
    }
    sum += __shfl_xor_sync(0xffffffffu, sum, 1);
    sum += __shfl_xor_sync(0xffffffffu, sum, 2);
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      A[j] = A[j] / sum;
      if (live && q + 4 * j < E) probs[(size_t)s * E + q + 4 * j] = A[j];
    }
    if (k > 0) {
      uint32_t taken = 0;  // bit j: this lane's expert q + 4j is picked
      float wsum = 0.f;
      for (int jj = 0; jj < k; ++jj) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        float ba = 0.f;
#pragma unroll
        for (int j = 0; j < PER; ++j) {
          const int e = q + 4 * j;
          if (e < E && !((taken >> j) & 1u) && better(z[j], e, bv, bi)) { bv = z[j]; bi = e; ba = A[j]; }
        }
#pragma unroll
        for (int off = 1; off <= 2; off <<= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
          const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
          const float oa = __shfl_xor_sync(0xffffffffu, ba, off);
          if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; ba = oa; }
        }
        if ((bi & 3) == q) taken |= 1u << (bi >> 2);
        if (live && q == 0) {
          idx[(size_t)s * k + jj] = bi;
          w[(size_t)s * k + jj] = ba;
        }
        wsum += ba;
      }
      if (renorm && live && q == 0)
        for (int jj = 0; jj < k; ++jj) w[(size_t)s * k + jj] = w[(size_t)s * k + jj] / wsum;
    }
  } else {
    for (int i = 0; i < kMmaBM / kMmaWarps; ++i) {
      const int r = warp * (kMmaBM / kMmaWarps) + i, s = t0 + r;
      if (s >= T) break;
      float z[VPL], A[VPL];
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        int e = lane + 32 * v;
        float zz = -INFINITY;
        if (e < E) {
          zz = sZ[r * (EP + 1) + e];
          if (bias) zz += bias[e];
          if (zprev) zz += zscale * zprev[(size_t)s * E + e];
          logits[(size_t)s * E + e] = zz;
        }
        z[v] = zz;
      }
      row_softmax<VPL>(z, E, A);
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        int e = lane + 32 * v;
        if (e < E) probs[(size_t)s * E + e] = A[v];
      }
      if (k > 0) row_topk<VPL>(z, A, E, k, renorm, idx + (size_t)s * k, w + (size_t)s * k);
    }
  }
}

template <int VPL>
__global__ void __launch_bounds__(kThreads)
router_f32_kernel(const float *__restrict__ x, const float *__restrict__ Wr,
                  const float *__restrict__ bias, const float *__restrict__ zprev, float zscale,
                  int T, int d, int E, float *__restrict__ logits, float *__restrict__ probs,
                  int k, int renorm, int32_t *__restrict__ idx, float *__restrict__ w) {
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  for (int s = gw; s < T; s += nw) {
    const float *xr = x + (size_t)s * d;
    float z[VPL], A[VPL];
#pragma unroll
    for (int v = 0; v < VPL; ++v) z[v] = -INFINITY;
    for (int e = 0; e < E; ++e) {
      const float *wr = Wr + (size_t)e * d;
      float p = 0.f;
      for (int j = lane; j < d; j += 32) p = fmaf(xr[j], wr[j], p);
      p = warp_sum(p);
      if (bias) p += bias[e];
      if (zprev) p += zscale * zprev[(size_t)s * E + e];
#pragma unroll
      for (int v = 0; v < VPL; ++v)
        if (lane + 32 * v == e) z[v] = p;
    }
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      int e = lane + 32 * v;
      if (e < E) logits[(size_t)s * E + e] = z[v];
    }
    row_softmax<VPL>(z, E, A);
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      int e = lane + 32 * v;
      if (e < E) probs[(size_t)s * E + e] = A[v];
    }
    if (k > 0) row_topk<VPL>(z, A, E, k, renorm, idx + (size_t)s * k, w + (size_t)s * k);
  }
}

// Small blocks: one CTA per token, 8 warps sharing the E dot products of
// length d (16-byte loads of the x row and of W_r rows), then warp 0
// finishes softmax and top-k. Latency-bound; used when T is small enough
// that a 64-token MMA tile would leave most of the GPU idle.
constexpr int kRowThreads = 256;
template <int VPL>
__global__ void __launch_bounds__(kRowThreads)
router_rowwise_bf16_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ Wr,
                           const float *__restrict__ bias, const float *__restrict__ zprev,
                           float zscale, int T, int d, int E, float *__restrict__ logits,
                           float *__restrict__ probs, int k, int renorm,
                           int32_t *__restrict__ idx, float *__restrict__ w,
                           unsigned long long *__restrict__ votes, int k_vote) {
  __shared__ float zs[32 * VPL];
  const int s = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int kWarps = kRowThreads / 32;
  constexpr int kEB = 8;  // experts per register block: their loads are issued together
  const __nv_bfloat16 *xr = x + (size_t)s * d;
  for (int e0 = warp * kEB; e0 < E; e0 += kWarps * kEB) {
    float p[kEB];
#pragma unroll
    for (int j = 0; j < kEB; ++j) p[j] = 0.f;
    const __nv_bfloat16 *w0 = Wr + (size_t)e0 * d;
#pragma unroll 2
    for (int c = lane * 8; c < d; c += 256) {
      uint4 xa = *reinterpret_cast<const uint4 *>(xr + c);
      uint4 wb[kEB];
#pragma unroll
      for (int j = 0; j < kEB; ++j)
        wb[j] = (e0 + j < E) ? *reinterpret_cast<const uint4 *>(w0 + (size_t)j * d + c)
                             : make_uint4(0, 0, 0, 0);
      const __nv_bfloat162 *xh = reinterpret_cast<const __nv_bfloat162 *>(&xa);
#pragma unroll
      for (int j = 0; j < kEB; ++j) {
        const __nv_bfloat162 *wh = reinterpret_cast<const __nv_bfloat162 *>(&wb[j]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 a = __bfloat1622float2(xh[i]), b = __bfloat1622float2(wh[i]);
          p[j] = fmaf(a.x, b.x, p[j]);
          p[j] = fmaf(a.y, b.y, p[j]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kEB; ++j) {
      const float t = warp_sum(p[j]);
      if (lane == 0 && e0 + j < E) zs[e0 + j] = t;
    }
  }
  __syncthreads();
  if (warp != 0) return;
  float z[VPL], A[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int e = lane + 32 * v;
    float zz = -INFINITY;
    if (e < E) {
      zz = zs[e];
      if (bias) zz += bias[e];
      if (zprev) zz += zscale * zprev[(size_t)s * E + e];
      logits[(size_t)s * E + e] = zz;
    }
    z[v] = zz;
  }
  row_softmax<VPL>(z, E, A);
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int e = lane + 32 * v;
    if (e < E) probs[(size_t)s * E + e] = A[v];
  }
  if (k > 0) row_topk<VPL>(z, A, E, k, renorm, idx + (size_t)s * k, w + (size_t)s * k);
  if (votes) {
    // DES-Vote (i)+(ii) for this token: its top-K by P, ties to the lower
    // id; each kept expert's vote q(P) is added to the block's total.
    bool taken[VPL];
#pragma unroll
    for (int v = 0; v < VPL; ++v) taken[v] = false;
    for (int r = 0; r < k_vote; ++r) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        const int e = lane + 32 * v;
        if (e < E && !taken[v] && better(A[v], e, bv, bi)) { bv = A[v]; bi = e; }
      }
      warp_argmax(bv, bi);
#pragma unroll
      for (int v = 0; v < VPL; ++v)
        if (lane + 32 * v == bi) {
          taken[v] = true;
          atomicAdd(votes + bi, (unsigned long long)vote_quantum(A[v]));
        }
    }
  }
}

// Finish of the split router: warp per token sums the width slices' partial
// logits in slice order (deterministic), adds bias and gate residual, then
// softmax, token-choice top-k and/or the DES vote (as in the rowwise kernel).
template <int VPL>
__global__ void __launch_bounds__(kThreads)
router_finish_kernel(const float *__restrict__ part, int n_part, const float *__restrict__ bias,
                     const float *__restrict__ zprev, float zscale, int T, int E,
                     float *__restrict__ logits, float *__restrict__ probs, int k, int renorm,
                     int32_t *__restrict__ idx, float *__restrict__ w,
                     unsigned long long *__restrict__ votes, int k_vote) {
  const int lane = threadIdx.x & 31;
  const int s = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (s >= T) return;
  float z[VPL], A[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int e = lane + 32 * v;
    float zz = -INFINITY;
    if (e < E) {
      zz = 0.f;
#pragma unroll 8
      for (int j = 0; j < n_part; ++j) zz += part[((size_t)j * T + s) * E + e];
      if (bias) zz += bias[e];
      if (zprev) zz += zscale * zprev[(size_t)s * E + e];
      logits[(size_t)s * E + e] = zz;
    }
    z[v] = zz;
  }
  row_softmax<VPL>(z, E, A);
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int e = lane + 32 * v;
    if (e < E) probs[(size_t)s * E + e] = A[v];
  }
  if (k > 0) row_topk<VPL>(z, A, E, k, renorm, idx + (size_t)s * k, w + (size_t)s * k);
  if (votes) {
    bool taken[VPL];
#pragma unroll
    for (int v = 0; v < VPL; ++v) taken[v] = false;
    for (int r = 0; r < k_vote; ++r) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        const int e = lane + 32 * v;
        if (e < E && !taken[v] && better(A[v], e, bv, bi)) { bv = A[v]; bi = e; }
      }
      warp_argmax(bv, bi);
#pragma unroll
      for (int v = 0; v < VPL; ++v)
        if (lane + 32 * v == bi) {
          taken[v] = true;
          atomicAdd(votes + bi, (unsigned long long)vote_quantum(A[v]));
        }
    }
  }
}

template <int VPL>
__global__ void __launch_bounds__(kThreads)
select_topk_kernel(const float *__restrict__ logits, const float *__restrict__ probs, int T,
                   int E, int k, int renorm, int32_t *__restrict__ idx, float *__restrict__ w) {
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  for (int s = gw; s < T; s += nw) {
    float z[VPL], A[VPL];
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      int e = lane + 32 * v;
      z[v] = e < E ? logits[(size_t)s * E + e] : -INFINITY;
      A[v] = e < E ? probs[(size_t)s * E + e] : 0.f;
    }
    row_topk<VPL>(z, A, E, k, renorm, idx + (size_t)s * k, w + (size_t)s * k);
  }
}

template <int NT>
int run_router_bf16(const void *x, const void *Wr, const float *bias, const float *zprev,
                    float zscale, int T, int d, int E, float *logits, float *probs, int k,
                    int renorm, int32_t *idx, float *w, cudaStream_t stream) {
  constexpr int EP = NT * 8;
  constexpr int kMmaStages = mma_stages<NT>();
  const size_t smem = (size_t)kMmaStages * (kMmaBM + EP) * kLDS * sizeof(__nv_bfloat16) +
                      2 * (size_t)kMmaBM * (EP + 1) * sizeof(float);
  auto kern = router_bf16_kernel<NT>;
  MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  dim3 grid((T + kMmaBM - 1) / kMmaBM);
  kern<<<grid, kMmaThreads, smem, stream>>>(static_cast<const __nv_bfloat16 *>(x),
                                         static_cast<const __nv_bfloat16 *>(Wr), bias, zprev,
                                         zscale, T, d, E, logits, probs, k, renorm, idx, w, ZeroList{});
  return last_launch_status();
}

template <int NT>
int run_router_partial(const void *x, const void *Wr, int T, int d, int E, float *part,
                       int n_part, const ZeroList &zero, cudaStream_t stream) {
  constexpr int EP = NT * 8;
  constexpr int kMmaStages = mma_stages<NT>();
  const size_t smem = (size_t)kMmaStages * (kMmaBM + EP) * kLDS * sizeof(__nv_bfloat16) +
                      2 * (size_t)kMmaBM * (EP + 1) * sizeof(float);
  auto kern = router_bf16_kernel<NT, true>;
  MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  dim3 grid((T + kMmaBM - 1) / kMmaBM, n_part);
  kern<<<grid, kMmaThreads, smem, stream>>>(static_cast<const __nv_bfloat16 *>(x),
                                            static_cast<const __nv_bfloat16 *>(Wr), nullptr, nullptr,
                                            0.f, T, d, E, part, nullptr, 0, 0, nullptr, nullptr,
                                            zero);
  return last_launch_status();
}

template <int NT>
int run_router_split(const void *x, const void *Wr, const float *bias, const float *zprev,
                     float zscale, int T, int d, int E, float *part, int n_part, float *logits,
                     float *probs, int k, int renorm, int32_t *idx, float *w,
                     unsigned long long *votes, int k_vote, cudaStream_t stream) {
  ZeroList zero{};
  if (votes) {  // the partial kernel clears the vote totals the finish adds into
    zero.p[0] = reinterpret_cast<int32_t *>(votes);
    zero.n[0] = 2 * E;
  }
  const int st = run_router_partial<NT>(x, Wr, T, d, E, part, n_part, zero, stream);
  if (st != MOE_OK) return st;
  const int wpb = kThreads / 32;
  const int blocks = (T + wpb - 1) / wpb;
  const int vpl = (E + 31) / 32;
  if (vpl == 1) router_finish_kernel<1><<<blocks, kThreads, 0, stream>>>(part, n_part, bias, zprev, zscale, T, E, logits, probs, k, renorm, idx, w, votes, k_vote);
  else if (vpl == 2) router_finish_kernel<2><<<blocks, kThreads, 0, stream>>>(part, n_part, bias, zprev, zscale, T, E, logits, probs, k, renorm, idx, w, votes, k_vote);
  else router_finish_kernel<4><<<blocks, kThreads, 0, stream>>>(part, n_part, bias, zprev, zscale, T, E, logits, probs, k, renorm, idx, w, votes, k_vote);
  return last_launch_status();
}

int warp_grid(int rows) {
  int warps_per_block = kThreads / 32;
  int blocks = (rows + warps_per_block - 1) / warps_per_block;
  int cap = num_sms() * 16;
  return blocks < cap ? blocks : cap;
}

}  // namespace

int router_split_parts(int T, int d, int dtype) {
  if (dtype != MOE_BF16 || T <= 0 || T > kRowwiseMaxTokens) return 0;
  const int tiles = (T + kMmaBM - 1) / kMmaBM;
  const int nk = (d + kBK - 1) / kBK;
  int parts = (2 * num_sms() + tiles - 1) / tiles;
  if (parts > nk) parts = nk;
  if (parts > 64) parts = 64;
  return parts < 1 ? 1 : parts;
}

int launch_router_split(const void *x, const void *W_r, const float *bias, const float *z_prev,
                        float z_prev_scale, int T, int d, int E, float *part, int n_part,
                        float *logits, float *probs, int k, int renorm, int32_t *idx, float *w,
                        int64_t *votes, int k_vote, cudaStream_t stream) {
  if (T == 0) return MOE_OK;
  unsigned long long *vacc = reinterpret_cast<unsigned long long *>(votes);
  const int nt = (E + 7) / 8;
  if (nt <= 1) return run_router_split<1>(x, W_r, bias, z_prev, z_prev_scale, T, d, E, part, n_part, logits, probs, k, renorm, idx, w, vacc, k_vote, stream);
  if (nt <= 2) return run_router_split<2>(x, W_r, bias, z_prev, z_prev_scale, T, d, E, part, n_part, logits, probs, k, renorm, idx, w, vacc, k_vote, stream);
  if (nt <= 3) return run_router_split<3>(x, W_r, bias, z_prev, z_prev_scale, T, d, E, part, n_part, logits, probs, k, renorm, idx, w, vacc, k_vote, stream);
  if (nt <= 4) return run_router_split<4>(x, W_r, bias, z_prev, z_prev_scale, T, d, E, part, n_part, logits, probs, k, renorm, idx, w, vacc, k_vote, stream);
  if (nt <= 8) return run_router_split<8>(x, W_r, bias, z_prev, z_prev_scale, T, d, E, part, n_part, logits, probs, k, renorm, idx, w, vacc, k_vote, stream);
  return run_router_split<16>(x, W_r, bias, z_prev, z_prev_scale, T, d, E, part, n_part, logits, probs, k, renorm, idx, w, vacc, k_vote, stream);
}

int launch_router_partial(const void *x, const void *W_r, int T, int d, int E, float *part,
                          int n_part, const ZeroList &zero, cudaStream_t stream) {
  if (T == 0) return MOE_OK;
  const int nt = (E + 7) / 8;
  if (nt <= 1) return run_router_partial<1>(x, W_r, T, d, E, part, n_part, zero, stream);
  if (nt <= 2) return run_router_partial<2>(x, W_r, T, d, E, part, n_part, zero, stream);
  if (nt <= 3) return run_router_partial<3>(x, W_r, T, d, E, part, n_part, zero, stream);
  if (nt <= 4) return run_router_partial<4>(x, W_r, T, d, E, part, n_part, zero, stream);
  if (nt <= 8) return run_router_partial<8>(x, W_r, T, d, E, part, n_part, zero, stream);
  return run_router_partial<16>(x, W_r, T, d, E, part, n_part, zero, stream);
}

bool router_can_vote(int T, int dtype) { return dtype == MOE_BF16 && T > 0 && T <= kRowwiseMaxTokens; }

int launch_router(const void *x, const void *W_r, const float *bias, const float *z_prev,
                  float z_prev_scale, int T, int d, int E, int dtype, float *logits,
                  float *probs, int k, int renorm, int32_t *idx, float *w,
                  cudaStream_t stream, int64_t *votes, int k_vote) {
  if (votes && !router_can_vote(T, dtype)) return MOE_ERR_UNSUPPORTED;
  unsigned long long *vacc = reinterpret_cast<unsigned long long *>(votes);
  if (T == 0) return MOE_OK;
  if (dtype == MOE_BF16 && T <= kRowwiseMaxTokens) {
    const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(x);
    const __nv_bfloat16 *wb = static_cast<const __nv_bfloat16 *>(W_r);
    const int vpl = (E + 31) / 32;
    if (vpl == 1) router_rowwise_bf16_kernel<1><<<T, kRowThreads, 0, stream>>>(xb, wb, bias, z_prev, z_prev_scale, T, d, E, logits, probs, k, renorm, idx, w, vacc, k_vote);
    else if (vpl == 2) router_rowwise_bf16_kernel<2><<<T, kRowThreads, 0, stream>>>(xb, wb, bias, z_prev, z_prev_scale, T, d, E, logits, probs, k, renorm, idx, w, vacc, k_vote);
    else router_rowwise_bf16_kernel<4><<<T, kRowThreads, 0, stream>>>(xb, wb, bias, z_prev, z_prev_scale, T, d, E, logits, probs, k, renorm, idx, w, vacc, k_vote);
    return last_launch_status();
  }
  if (dtype == MOE_BF16) {
    const int nt = (E + 7) / 8;
    if (nt <= 1) return run_router_bf16<1>(x, W_r, bias, z_prev, z_prev_scale, T, d, E, logits, probs, k, renorm, idx, w, stream);
    if (nt <= 2) return run_router_bf16<2>(x, W_r, bias, z_prev, z_prev_scale, T, d, E, logits, probs, k, renorm, idx, w, stream);
    if (nt <= 3) return run_router_bf16<3>(x, W_r, bias, z_prev, z_prev_scale, T, d, E, logits, probs, k, renorm, idx, w, stream);
    if (nt <= 4) return run_router_bf16<4>(x, W_r, bias, z_prev, z_prev_scale, T, d, E, logits, probs, k, renorm, idx, w, stream);
    if (nt <= 8) return run_router_bf16<8>(x, W_r, bias, z_prev, z_prev_scale, T, d, E, logits, probs, k, renorm, idx, w, stream);
    return run_router_bf16<16>(x, W_r, bias, z_prev, z_prev_scale, T, d, E, logits, probs, k, renorm, idx, w, stream);
  }
  const float *xf = static_cast<const float *>(x);
  const float *wf = static_cast<const float *>(W_r);
  const int grid = warp_grid(T);
  const int vpl = (E + 31) / 32;
  if (vpl == 1) router_f32_kernel<1><<<grid, kThreads, 0, stream>>>(xf, wf, bias, z_prev, z_prev_scale, T, d, E, logits, probs, k, renorm, idx, w);
  else if (vpl == 2) router_f32_kernel<2><<<grid, kThreads, 0, stream>>>(xf, wf, bias, z_prev, z_prev_scale, T, d, E, logits, probs, k, renorm, idx, w);
  else router_f32_kernel<4><<<grid, kThreads, 0, stream>>>(xf, wf, bias, z_prev, z_prev_scale, T, d, E, logits, probs, k, renorm, idx, w);
  return last_launch_status();
}

int launch_select_topk(const float *logits, const float *probs, int T, int E, int k,
                       int renorm, int32_t *idx, float *w, cudaStream_t stream) {
  if (T == 0) return MOE_OK;
  const int grid = warp_grid(T);
  const int vpl = (E + 31) / 32;
  if (vpl == 1) select_topk_kernel<1><<<grid, kThreads, 0, stream>>>(logits, probs, T, E, k, renorm, idx, w);
  else if (vpl == 2) select_topk_kernel<2><<<grid, kThreads, 0, stream>>>(logits, probs, T, E, k, renorm, idx, w);
  else select_topk_kernel<4><<<grid, kThreads, 0, stream>>>(logits, probs, T, E, k, renorm, idx, w);
  return last_launch_status();
}

}  // namespace moe
