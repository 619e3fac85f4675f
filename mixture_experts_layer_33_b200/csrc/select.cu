// Expert-choice top-C (block radix select) and the DES-Vote core set.
//
// EC-DiT: Scaling Diffusion Transformers with Adaptive Expert-Choice
// Routing, section 3 "Expert-Choice routing": each expert chooses its
// top tokens; "capacity factor": every expert takes C = f_c * S / E tokens
// of its routing group of S tokens.
//
// Dynamic Expert Sharing: Decoupling Memory from Parallelism in
// Mixture-of-Experts Diffusion LLMs, section 2.4 "DES-Vote": each token
// filters to its own top-K experts, votes their routing weights, and the
// M_core experts with the most votes form the core set that serves the
// whole block; section 4.3: tokens then re-activate experts from the core
// set at their original per-token count.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

// Monotone map of fp32 to uint32 (larger float -> larger key); -0 is
// folded onto +0 first so the IEEE tie between them survives.
__device__ __forceinline__ uint32_t orderable(float f) {
  if (f == 0.f) f = 0.f;
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kEcThreads = 256;

// One CTA per (group g, expert e). The column A[g*S : (g+1)*S, e] is
// staged in shared memory as orderable keys; four 8-bit radix passes find
// the C-th largest key `thr` and how many keys equal to it are still
// needed; two block scans then emit the chosen tokens in ascending order
// (keys > thr, plus the lowest-id keys == thr).
__global__ void __launch_bounds__(kEcThreads)
expert_choice_kernel(const float *__restrict__ probs, int E, int S, int C,
                     int32_t *__restrict__ tok, float *__restrict__ w) {
  extern __shared__ uint32_t keys[];  // [S]
  __shared__ int hist[256];
  __shared__ int scan_scratch[33];
  __shared__ int sel_digit, sel_above;

  const int g = blockIdx.x / E, e = blockIdx.x % E;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float *col = probs + (size_t)g * S * E + e;

  for (int s = tid; s < S; s += blockDim.x) keys[s] = orderable(col[(size_t)s * E]);

  uint32_t prefix = 0, mask = 0;
  int want = C;  // rank (1-based) of the wanted key among the candidates
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int s = tid; s < S; s += blockDim.x) {
      uint32_t kk = keys[s];
      if ((kk & mask) == prefix) atomicAdd(&hist[(kk >> shift) & 255u], 1);
    }
    __syncthreads();
    if (warp == 0) {
      // Lane l owns digits 255-8l .. 248-8l (descending).
      int local = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) local += hist[255 - 8 * lane - j];
      int inc = warp_inclusive_scan(local);
      int excl = inc - local;
      bool here = excl < want && inc >= want;
      if (here) {
        int run = excl;
        for (int j = 0; j < 8; ++j) {
          int dgt = 255 - 8 * lane - j;
          int c = hist[dgt];
          if (run + c >= want) {
            sel_digit = dgt;
            sel_above = run;
            break;
          }
          run += c;
        }
      }
    }
    __syncthreads();
    want -= sel_above;
    prefix |= (uint32_t)sel_digit << shift;
    mask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t thr = prefix;  // the C-th largest key; `want` equal keys are taken

  // Thread t owns the contiguous tokens [t*per, (t+1)*per).
  const int per = (S + blockDim.x - 1) / blockDim.x;
  const int lo = tid * per, hi = min(S, lo + per);
  int n_eq = 0;
  for (int s = lo; s < hi; ++s) n_eq += keys[s] == thr;
  int total;
  int eq_before = block_exclusive_scan(n_eq, scan_scratch, &total);
  int n_take = 0;
  {
    int eq = eq_before;
    for (int s = lo; s < hi; ++s) {
      uint32_t kk = keys[s];
      if (kk > thr) ++n_take;
      else if (kk == thr) { n_take += eq < want; ++eq; }
    }
  }
  int pos = block_exclusive_scan(n_take, scan_scratch, &total);
  {
    int eq = eq_before;
    int32_t *tout = tok + ((size_t)g * E + e) * C;
    float *wout = w + ((size_t)g * E + e) * C;
    for (int s = lo; s < hi; ++s) {
      uint32_t kk = keys[s];
      bool take = kk > thr;
      if (kk == thr) { take = eq < want; ++eq; }
      if (take && pos < C) {
        tout[pos] = g * S + s;
        wout[pos] = col[(size_t)s * E];
        ++pos;
      }
    }
  }
  (void)lane;
}

constexpr int kDesThreads = 1024;  // one warp per token of a 32-token block

// One CTA for the whole block of N tokens; each lane holds kDesVpl of a
// token's M <= 32*kDesVpl probabilities.
template <int kDesVpl>
__global__ void __launch_bounds__(kDesThreads)
des_vote_kernel(const float *__restrict__ P, int N, int M, int K, int Mc,
                int64_t *__restrict__ votes, int32_t *__restrict__ core,
                int32_t *__restrict__ idx, float *__restrict__ w) {
  __shared__ unsigned long long V[MOE_MAX_EXPERTS];
  __shared__ int in_core[MOE_MAX_EXPERTS];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  for (int e = tid; e < M; e += blockDim.x) V[e] = 0ull;
  __syncthreads();

  // (i) filter to the own top-K, (ii) vote with the routing weights.
  for (int n = warp; n < N; n += nwarps) {
    float p[kDesVpl];
    bool taken[kDesVpl];
#pragma unroll
    for (int v = 0; v < kDesVpl; ++v) {
      int e = lane + 32 * v;
      p[v] = e < M ? P[(size_t)n * M + e] : -INFINITY;
      taken[v] = false;
    }
    for (int r = 0; r < K; ++r) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int v = 0; v < kDesVpl; ++v) {
        int e = lane + 32 * v;
        if (e < M && !taken[v] && better(p[v], e, bv, bi)) { bv = p[v]; bi = e; }
      }
      warp_argmax(bv, bi);
#pragma unroll
      for (int v = 0; v < kDesVpl; ++v)
        if (lane + 32 * v == bi) {
          taken[v] = true;
          atomicAdd(&V[bi], (unsigned long long)vote_quantum(p[v]));
        }
    }
  }
  __syncthreads();

  // (iii) elect the M_core most voted, ties to the lower id.
  for (int e = tid; e < M; e += blockDim.x) {
    long long ve = (long long)V[e];
    int rank = 0;
    for (int f = 0; f < M; ++f) {
      long long vf = (long long)V[f];
      rank += (vf > ve) || (vf == ve && f < e);
    }
    in_core[e] = rank < Mc;
    votes[e] = ve;
  }
  __syncthreads();
  for (int e = tid; e < M; e += blockDim.x) {
    if (in_core[e]) {
      int pos = 0;
      for (int f = 0; f < e; ++f) pos += in_core[f];
      core[pos] = e;
    }
  }

  // Re-route: each token's K largest P over the core set.
  for (int n = warp; n < N; n += nwarps) {
    float p[kDesVpl];
    bool taken[kDesVpl];
#pragma unroll
    for (int v = 0; v < kDesVpl; ++v) {
      int e = lane + 32 * v;
      bool ok = e < M && in_core[e];
      p[v] = ok ? P[(size_t)n * M + e] : -INFINITY;
      taken[v] = !ok;
    }
    for (int r = 0; r < K; ++r) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int v = 0; v < kDesVpl; ++v) {
        int e = lane + 32 * v;
        if (!taken[v] && better(p[v], e, bv, bi)) { bv = p[v]; bi = e; }
      }
      warp_argmax(bv, bi);
      float own = 0.f;
#pragma unroll
      for (int v = 0; v < kDesVpl; ++v)
        if (lane + 32 * v == bi) { taken[v] = true; own = p[v]; }
      float pw = __shfl_sync(0xffffffffu, own, bi & 31);
      if (lane == 0) {
        idx[(size_t)n * K + r] = bi;
        w[(size_t)n * K + r] = pw;
      }
    }
  }
}

// Small-block DES tail, parallel over tokens: the votes were summed into
// `votes` (exact int64, order-free) by the router's per-token CTAs; every
// CTA here re-derives the same election from them (M <= 256 values) and
// re-routes its own token over the core set. CTA 0 also writes the core set.
template <int VPL>
__global__ void __launch_bounds__(256)
des_reroute_kernel(const float *__restrict__ P, const int64_t *__restrict__ votes, int N, int M,
                   int K, int Mc, int32_t *__restrict__ core, int32_t *__restrict__ idx,
                   float *__restrict__ w) {
  __shared__ int in_core[MOE_MAX_EXPERTS];
  const int n = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int e = tid; e < M; e += blockDim.x) {
    const long long ve = votes[e];
    int rank = 0;
    for (int f = 0; f < M; ++f) {
      const long long vf = votes[f];
      rank += (vf > ve) || (vf == ve && f < e);
    }
    in_core[e] = rank < Mc;
  }
  __syncthreads();
  if (n == 0)
    for (int e = tid; e < M; e += blockDim.x)
      if (in_core[e]) {
        int pos = 0;
        for (int f = 0; f < e; ++f) pos += in_core[f];
        core[pos] = e;
      }
  if (warp != 0) return;
  float p[VPL];
  bool taken[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int e = lane + 32 * v;
    const bool ok = e < M && in_core[e];
    p[v] = ok ? P[(size_t)n * M + e] : -INFINITY;
    taken[v] = !ok;
  }
  for (int r = 0; r < K; ++r) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      const int e = lane + 32 * v;
      if (!taken[v] && better(p[v], e, bv, bi)) { bv = p[v]; bi = e; }
    }
    warp_argmax(bv, bi);
    float own = 0.f;
#pragma unroll
    for (int v = 0; v < VPL; ++v)
      if (lane + 32 * v == bi) { taken[v] = true; own = p[v]; }
    const float pw = __shfl_sync(0xffffffffu, own, bi & 31);
    if (lane == 0) {
      idx[(size_t)n * K + r] = bi;
      w[(size_t)n * K + r] = pw;
    }
  }
}

// DES-Seq for one block of N tokens, one CTA: every token's top-k_local by
// P marks the core set (a bitmask); the core list ascends; each token then
// takes its min(K, |core|) largest P over the core, the rest empty (-1).
template <int kDesVpl>
__global__ void __launch_bounds__(kDesThreads)
des_seq_kernel(const float *__restrict__ P, int N, int M, int K, int kl,
               int32_t *__restrict__ core, int32_t *__restrict__ n_core,
               int32_t *__restrict__ idx, float *__restrict__ w) {
  __shared__ unsigned bits[MOE_MAX_EXPERTS / 32];
  __shared__ int in_core[MOE_MAX_EXPERTS];
  __shared__ int ncore_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  if (tid < MOE_MAX_EXPERTS / 32) bits[tid] = 0u;
  __syncthreads();
  for (int n = warp; n < N; n += nwarps) {
    float p[kDesVpl];
    bool taken[kDesVpl];
#pragma unroll
    for (int v = 0; v < kDesVpl; ++v) {
      const int e = lane + 32 * v;
      p[v] = e < M ? P[(size_t)n * M + e] : -INFINITY;
      taken[v] = false;
    }
    for (int r = 0; r < kl; ++r) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int v = 0; v < kDesVpl; ++v) {
        const int e = lane + 32 * v;
        if (e < M && !taken[v] && better(p[v], e, bv, bi)) { bv = p[v]; bi = e; }
      }
      warp_argmax(bv, bi);
#pragma unroll
      for (int v = 0; v < kDesVpl; ++v)
        if (lane + 32 * v == bi) {
          taken[v] = true;
          atomicOr(&bits[bi >> 5], 1u << (bi & 31));
        }
    }
  }
  __syncthreads();
  for (int e = tid; e < M; e += blockDim.x) {
    const bool in = (bits[e >> 5] >> (e & 31)) & 1u;
    in_core[e] = in;
    if (in) {
      int pos = __popc(bits[e >> 5] & ((1u << (e & 31)) - 1u));
      for (int q = 0; q < (e >> 5); ++q) pos += __popc(bits[q]);
      core[pos] = e;
    }
  }
  if (tid == 0) {
    int c = 0;
    for (int q = 0; q < (M + 31) / 32; ++q) c += __popc(bits[q]);
    ncore_s = c;
    *n_core = c;
  }
  __syncthreads();
  const int nc = ncore_s;
  for (int e = nc + tid; e < M; e += blockDim.x) core[e] = -1;
  const int take = nc < K ? nc : K;
  for (int n = warp; n < N; n += nwarps) {
    float p[kDesVpl];
    bool taken[kDesVpl];
#pragma unroll
    for (int v = 0; v < kDesVpl; ++v) {
      const int e = lane + 32 * v;
      const bool ok = e < M && in_core[e];
      p[v] = ok ? P[(size_t)n * M + e] : -INFINITY;
      taken[v] = !ok;
    }
    for (int r = 0; r < K; ++r) {
      int bi = -1;
      float pw = 0.f;
      if (r < take) {
        float bv = -INFINITY;
        bi = 0x7fffffff;
#pragma unroll
        for (int v = 0; v < kDesVpl; ++v) {
          const int e = lane + 32 * v;
          if (!taken[v] && better(p[v], e, bv, bi)) { bv = p[v]; bi = e; }
        }
        warp_argmax(bv, bi);
        float own = 0.f;
#pragma unroll
        for (int v = 0; v < kDesVpl; ++v)
          if (lane + 32 * v == bi) { taken[v] = true; own = p[v]; }
        pw = __shfl_sync(0xffffffffu, own, bi & 31);
      }
      if (lane == 0) {
        idx[(size_t)n * K + r] = bi;
        w[(size_t)n * K + r] = pw;
      }
    }
  }
}

}  // namespace

int launch_des_seq(const float *probs, int N, int M, int K, int k_local, int32_t *core,
                   int32_t *n_core, int32_t *idx, float *w, cudaStream_t stream) {
  if (M <= 32) des_seq_kernel<1><<<1, kDesThreads, 0, stream>>>(probs, N, M, K, k_local, core, n_core, idx, w);
  else if (M <= 64) des_seq_kernel<2><<<1, kDesThreads, 0, stream>>>(probs, N, M, K, k_local, core, n_core, idx, w);
  else if (M <= 128) des_seq_kernel<4><<<1, kDesThreads, 0, stream>>>(probs, N, M, K, k_local, core, n_core, idx, w);
  else des_seq_kernel<8><<<1, kDesThreads, 0, stream>>>(probs, N, M, K, k_local, core, n_core, idx, w);
  return last_launch_status();
}

int launch_expert_choice(const float *probs, int T, int E, int S, int C, int32_t *tok,
                         float *w, cudaStream_t stream) {
  const int G = T / S;
  if (G == 0) return MOE_OK;
  const size_t smem = (size_t)S * sizeof(uint32_t);
  MOE_CUDA_TRY(cudaFuncSetAttribute(expert_choice_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  int threads = S < kEcThreads ? ((S + 31) / 32) * 32 : kEcThreads;
  expert_choice_kernel<<<G * E, threads, smem, stream>>>(probs, E, S, C, tok, w);
  return last_launch_status();
}

int launch_des_reroute(const float *probs, const int64_t *votes, int N, int M, int K, int M_core,
                       int32_t *core, int32_t *idx, float *w, cudaStream_t stream) {
  if (N == 0) return MOE_OK;
  if (M <= 32) des_reroute_kernel<1><<<N, 256, 0, stream>>>(probs, votes, N, M, K, M_core, core, idx, w);
  else if (M <= 64) des_reroute_kernel<2><<<N, 256, 0, stream>>>(probs, votes, N, M, K, M_core, core, idx, w);
  else if (M <= 128) des_reroute_kernel<4><<<N, 256, 0, stream>>>(probs, votes, N, M, K, M_core, core, idx, w);
  else des_reroute_kernel<8><<<N, 256, 0, stream>>>(probs, votes, N, M, K, M_core, core, idx, w);
  return last_launch_status();
}

int launch_des_vote(const float *probs, int N, int M, int K, int M_core, int64_t *votes,
                    int32_t *core, int32_t *idx, float *w, cudaStream_t stream) {
  if (M <= 32) des_vote_kernel<1><<<1, kDesThreads, 0, stream>>>(probs, N, M, K, M_core, votes, core, idx, w);
  else if (M <= 64) des_vote_kernel<2><<<1, kDesThreads, 0, stream>>>(probs, N, M, K, M_core, votes, core, idx, w);
  else if (M <= 128) des_vote_kernel<4><<<1, kDesThreads, 0, stream>>>(probs, N, M, K, M_core, votes, core, idx, w);
  else des_vote_kernel<8><<<1, kDesThreads, 0, stream>>>(probs, N, M, K, M_core, votes, core, idx, w);
  return last_launch_status();
}

}  // namespace moe
