// The whole MoE layer for a small block of tokens (<= 128) in one
// persistent cooperative kernel: router finish -> token-choice top-k or
// DES-Vote election and re-route -> weight-streaming expert MLP -> weighted
// combine with the residual.
//
// Dynamic Expert Sharing: Decoupling Memory from Parallelism in MoE
// Diffusion LLMs, section 2.1: a small block's MoE latency is set by the
// fetch of each distinct expert's weights (the b term of f(c) = a*c + b),
// so the kernel's job is to start streaming the used experts' weights from
// HBM as early as possible and never let the stream pause. Section 2.4
// (DES-Vote): each token keeps its top-K experts and votes for them with
// its routing weights; the M_core most voted experts form the core set and
// every token re-routes to its top-K experts within it.
// EC-DiT: Scaling Diffusion Transformers with Adaptive Expert-Choice
// Routing, section 3 (Token-Choice routing): each token keeps its top-k.
// DICE: Staleness-Centric Optimizations for Parallel Diffusion MoE
// Inference, Conditional Communication: a token's output is the sum of its
// experts' outputs weighted by the routing scores (plus the residual).
//
// One CTA per SM (cooperative launch, so bounded spin-waits between CTAs
// always end). CTA t < T owns token t for the routing steps.
//   1. token CTAs finish the router (sum the split-K partial logits in a
//      fixed order, bias, gate residual, softmax) and take the top-k by
//      rank: DES adds exact int64 votes, token choice marks its picks in
//      per-expert token bitmasks. Grid barrier.
//   2. every CTA derives the list of experts to stream: the elected core
//      set (DES) or the experts some token picked (token choice). From here
//      the weight stream runs: the up projection's B operand is all T tokens
//      (x as is, zero rows past T), so it needs no dispatch at all, and the
//      epilogue keeps only the columns of tokens that picked the expert.
//   3. meanwhile the epilogue warps finish the routing: DES tokens re-route
//      over the core set and mark the bitmasks (second grid barrier); every
//      CTA turns the bitmasks into row offsets (expert-major, tokens
//      ascending), token CTAs write their slots.
//   4. expert units, one list for the whole grid: first every (expert,
//      128 hidden units) block of the up projection, then every (expert,
//      128 output features) block of the down projection; a down unit of an
//      expert waits (bounded) until all of that expert's hidden rows are
//      stored. Warp roles as in the weight-streaming MLP: warp 0 TMA
//      producer, warp 1 tcgen05.mma issuer, warps 2..5 TMEM epilogue.
//   5. after the last unit everywhere (completion counter), the epilogue
//      warps of all CTAs combine: y = residual + sum_j w_j * expert_j(x)
//      (zero-computation experts resolved here), fp32 sum in slot order.
// Every wait is bounded (2 s) and reports MOE_DEV_TIMEOUT.
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "mma_sync.cuh"
#include "tc_ptx.cuh"

namespace moe {
namespace {

using namespace tc;

constexpr int kThreads = 192;  // 6 warps
constexpr int kWarps = kThreads / 32;
constexpr int kEpiThreads = 128;  // warps 2..5
constexpr int kMaxE = 128;
constexpr int kMaxK = 32;
constexpr int BMW = 128;  // weight rows per unit (MMA M)
constexpr int BK = 64;
constexpr int kUQ = 8;  // unit-id ring between the producer and the other roles
// Bytes of leading weight boxes warmed into L2 while the routing runs.
constexpr int64_t kWarmBytes = 32ll << 20;

__device__ __forceinline__ void epi_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ int ld_acquire_s32(const int32_t *p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bounded wait until *p >= target; on expiry raise the abort flag and the
// timeout status. Returns false on expiry or abort.
__device__ __noinline__ bool wait_u32(const unsigned *p, unsigned target, volatile int *abort_flag,
                                      int32_t *status) {
  if (ld_acquire_u32(p) >= target) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t spin = 1;; ++spin) {
    __nanosleep(32);  // many CTAs poll one word: keep the line free for the arrivals
    if (ld_acquire_u32(p) >= target) return true;
    if ((spin & 15u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > kTimeoutNs) {
        *abort_flag = 1;
        set_status(status, MOE_DEV_TIMEOUT);
        return false;
      }
    }
  }
}
__device__ __noinline__ bool wait_s32(const int32_t *p, int target, volatile int *abort_flag,
                                      int32_t *status) {
  if (ld_acquire_s32(p) >= target) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t spin = 1;; ++spin) {
    if (ld_acquire_s32(p) >= target) return true;
    if ((spin & 63u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > kTimeoutNs) {
        *abort_flag = 1;
        set_status(status, MOE_DEV_TIMEOUT);
        return false;
      }
    }
  }
}
// Bounded wait on a flag set by other warps of this CTA.
__device__ __noinline__ bool wait_local(volatile int *flag, volatile int *abort_flag,
                                        int32_t *status) {
  if (*flag) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t spin = 1;; ++spin) {
    if (*flag) return true;
    if ((spin & 63u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > kTimeoutNs) {
        *abort_flag = 1;
        set_status(status, MOE_DEV_TIMEOUT);
        return false;
      }
    }
  }
}

// 8 consecutive bf16 of a row written by another CTA of this grid (L2).
__device__ __forceinline__ uint4 ld_cg_v4(const void *p) {
  return __ldcg(reinterpret_cast<const uint4 *>(p));
}
__device__ __forceinline__ void fma8(float wgt, const uint4 &u, float (&acc)[8]) {
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    acc[2 * i] = fmaf(wgt, f.x, acc[2 * i]);
    acc[2 * i + 1] = fmaf(wgt, f.y, acc[2 * i + 1]);
  }
}

// Unit u of the grid-wide list. Up units come first: block 0 of every
// streamed expert (the blocks whose leading weight boxes were warmed into
// L2 during the routing), then the other blocks expert by expert; then the
// down units expert by expert. gi indexes the streamed-expert list.
struct BlockUnit {
  bool up;
  int gi, blk;
};
__device__ __forceinline__ BlockUnit unit_of(int u, int n_groups, int up_blocks, int down_blocks) {
  BlockUnit r;
  const int n_up = n_groups * up_blocks;
  r.up = u < n_up;
  if (!r.up) {
    r.gi = (u - n_up) / down_blocks;
    r.blk = (u - n_up) % down_blocks;
  } else if (u < n_groups) {
    r.gi = u;
    r.blk = 0;
  } else {  // up_blocks >= 2 here
    r.gi = (u - n_groups) / (up_blocks - 1);
    r.blk = 1 + (u - n_groups) % (up_blocks - 1);
  }
  return r;
}

__device__ __forceinline__ void prefetch_box_l2(const CUtensorMap *map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y)
               : "memory");
}

template <int NB, int ACT>
__global__ void __launch_bounds__(kThreads, 1)
moe_block_kernel(const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmX,
                 const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ CUtensorMap tmH,
                 const BlockArgs a, const KindTable kinds) {
  constexpr bool GATED = ACT == kActSwiglu;
  constexpr uint32_t A_BYTES = BMW * BK * 2;  // 16 KB
  constexpr uint32_t B_BYTES = NB * BK * 2;
  constexpr uint32_t STAGE_BYTES = 2 * A_BYTES + 2 * B_BYTES;
  constexpr int STAGES0 = (200 * 1024) / STAGE_BYTES;
  constexpr int STAGES = STAGES0 > 8 ? 8 : STAGES0;
  constexpr int ACC_COLS = 2 * NB;  // D0 and (gated up) D1
  constexpr uint32_t TMEM_COLS = 2 * ACC_COLS <= 32 ? 32 : 2 * ACC_COLS <= 64 ? 64
                                 : 2 * ACC_COLS <= 128 ? 128 : 2 * ACC_COLS <= 256 ? 256 : 512;
  constexpr uint32_t IDESC = idesc_bf16_f32(BMW, NB);

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[2 * STAGES + 5 + 2 * kUQ];
  __shared__ int uq[kUQ];
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ volatile int route_ready;
  __shared__ int ok_slot;
  __shared__ float red[kWarps][kMaxE];
  __shared__ float zs[kMaxE], As[kMaxE];
  __shared__ long long V[kMaxE];
  __shared__ int core_list[kMaxE];
  __shared__ int glist[kMaxE];  // experts streamed, ascending id
  __shared__ unsigned wbits[kMaxE / 32], sbits[kMaxE / 32], lbits[kMaxE / 32];
  __shared__ int n_groups_s, n_core_s;
  __shared__ int offs[kMaxE + 1];
  __shared__ unsigned mask[kMaxE][4];  // tokens (<= 128) that picked expert e
  __shared__ int own_ids[kMaxK];
  __shared__ float own_w[kMaxK];
  __shared__ int wsum_s[4];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int t = blockIdx.x, G = gridDim.x;
  const int T = a.T, E = a.E, k = a.k, nh = a.n_heavy;
  const bool des = a.routing == MOE_DES_VOTE;
  const bool seq = a.routing == MOE_DES_SEQ;  // DES-Seq: core = union of local top-k_local
  const bool core_routed = des || seq;         // tokens re-route over a core set

  uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~(uintptr_t)1023);
  const uint32_t s0 = smem_u32(ring);
  const uint32_t full0 = smem_u32(&bars[0]);
  const uint32_t empty0 = smem_u32(&bars[STAGES]);
  const uint32_t tfull0 = smem_u32(&bars[2 * STAGES]);
  const uint32_t tempty0 = smem_u32(&bars[2 * STAGES + 2]);
  const uint32_t drain = smem_u32(&bars[2 * STAGES + 4]);
  const uint32_t uqf0 = smem_u32(&bars[2 * STAGES + 5]);        // unit id written
  const uint32_t uqe0 = smem_u32(&bars[2 * STAGES + 5 + kUQ]);  // unit done by the epilogue

  // ---- setup (overlaps the routing below)
  if (tid == 0) {
    abort_flag = 0;
    route_ready = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, 4);
    }
    mbar_init(drain, 1);
    for (int q = 0; q < kUQ; ++q) {
      mbar_init(uqf0 + 8 * q, 1);
      mbar_init(uqe0 + 8 * q, 4);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid < kMaxK) { own_ids[tid] = -1; own_w[tid] = 0.f; }

  // The router's per-expert terms of token t, read now (off the critical path).
  float zb[kMaxE / 32], zq[kMaxE / 32];
  if (warp == 0 && t < T) {
#pragma unroll
    for (int v = 0; v < kMaxE / 32; ++v) {
      const int e = lane + 32 * v;
      zb[v] = (e < E && a.bias) ? __ldg(a.bias + e) : 0.f;
      zq[v] = (e < E && a.zprev) ? a.zscale * __ldg(a.zprev + (size_t)t * E + e) : 0.f;
    }
  }

  // ---- 0. router GEMM, K-sliced over the CTAs: CTA s < n_slices computes
  // every token's partial logits over columns [s*kslice, (s+1)*kslice) on
  // the tensor cores (mma.sync m16n8k16, fp32 accumulate), operands staged
  // in the (not yet used) operand ring with padded rows, zero past T, E and
  // the end of the row.
  if (t < a.n_slices) {
    const int ks = a.kslice;  // a multiple of 16
    const int ld = ks + 8;    // padded row: conflict-free ldmatrix
    const int k0 = t * ks;
    const int kw = min(ks, a.d - k0);
    const int T16 = (T + 15) & ~15, E8 = (E + 7) & ~7;
    __nv_bfloat16 *sx = reinterpret_cast<__nv_bfloat16 *>(smem_raw);  // [T16][ld]
    __nv_bfloat16 *sw = sx + T16 * ld;                                 // [E8][ld]
    const __nv_bfloat16 *xg = static_cast<const __nv_bfloat16 *>(a.x);
    const __nv_bfloat16 *wg = static_cast<const __nv_bfloat16 *>(a.W_r);
    const int vpr = ks >> 3;
    const int nvec = (T16 + E8) * vpr;
    for (int base = tid; base < nvec; base += 8 * kThreads) {
      uint4 r[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {  // all loads first, then the stores
        const int i = base + u * kThreads;
        r[u] = make_uint4(0u, 0u, 0u, 0u);
        if (i < nvec) {
          const int row = i / vpr, v = i - row * vpr;
          const bool isx = row < T16;
          const int rr = isx ? row : row - T16;
          if ((isx ? rr < T : rr < E) && v * 8 < kw)
            r[u] = __ldg(reinterpret_cast<const uint4 *>((isx ? xg : wg) + (size_t)rr * a.d + k0 + v * 8));
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = base + u * kThreads;
        if (i < nvec) {
          const int row = i / vpr, v = i - row * vpr;
          *reinterpret_cast<uint4 *>((row < T16 ? sx + row * ld : sw + (row - T16) * ld) + v * 8) = r[u];
        }
      }
    }
    __syncthreads();
    const int mt = T16 >> 4, nt = E8 >> 3;
    for (int tile = warp; tile < mt * nt; tile += kWarps) {
      const int mi = tile / nt, ni = tile - mi * nt;
      float c[4] = {0.f, 0.f, 0.f, 0.f};
      const __nv_bfloat16 *tX = sx + (mi * 16) * ld;
      const __nv_bfloat16 *tW = sw + (ni * 8) * ld;
      for (int kk = 0; kk < (ks >> 4); ++kk) {
        uint32_t af[4], bf[2];
        ldmatrix_x4(af, tX + (lane & 15) * ld + kk * 16 + (lane >> 4) * 8);
        ldmatrix_x2(bf, tW + (lane & 7) * ld + kk * 16 + ((lane >> 3) & 1) * 8);
        mma_bf16_16816(c, af, bf);
      }
      const int r0 = mi * 16 + (lane >> 2), c0 = ni * 8 + (lane & 3) * 2;
      float *pp = a.part + (size_t)t * T * E;
      if (r0 < T) {
        if (c0 < E) pp[(size_t)r0 * E + c0] = c[0];
        if (c0 + 1 < E) pp[(size_t)r0 * E + c0 + 1] = c[1];
      }
      if (r0 + 8 < T) {
        if (c0 < E) pp[(size_t)(r0 + 8) * E + c0] = c[2];
        if (c0 + 1 < E) pp[(size_t)(r0 + 8) * E + c0 + 1] = c[3];
      }
    }
    // The ring is written by TMA (async proxy) later on.
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  // Grid barrier 0: every slice's partial logits are out.
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    atomicAdd(a.sync + 0, 1u);
    ok_slot = wait_u32(a.sync + 0, (unsigned)G, &abort_flag, a.dev_status) ? 1 : 0;
  }
  __syncthreads();

  // CTAs without a token warm L2 with the leading k-blocks of block 0 of
  // every heavy expert's up projection (up to kWarmBytes): which experts
  // will stream is not known until the votes are in, HBM is idle until
  // then, and block 0 of each streamed expert is the first unit claimed.
  if (t >= T && ok_slot && tid == 0 && nh > 0) {
    const int per = GATED ? 2 : 1;  // gate and up rows
    const int nkb = (a.d + BK - 1) / BK;
    const int64_t fit = kWarmBytes / ((int64_t)nh * per * BMW * BK * 2);
    const int pk = (int)(fit < nkb ? fit : nkb);
    const int n_box = nh * per * pk;
    for (int i = t - T; i < n_box; i += G - T) {
      const int e = i / (per * pk), r = i - e * (per * pk);
      const int half = r / pk, kb = r - half * pk;
      prefetch_box_l2(&tmW1, kb * BK, e * a.w1_rows_per_group + half * a.h);
    }
  }

  // ---- 1. token CTAs finish the router and pick.
  if (t < T && ok_slot) {
    {
      float acc[kMaxE / 32];
#pragma unroll
      for (int v = 0; v < kMaxE / 32; ++v) acc[v] = 0.f;
      const float *pt = a.part + (size_t)t * E;
      const size_t slice = (size_t)T * E;
#pragma unroll 8
      for (int j = warp; j < a.n_slices; j += kWarps) {
#pragma unroll
        for (int v = 0; v < kMaxE / 32; ++v) {
          const int e = lane + 32 * v;
          if (e < E) acc[v] += __ldcg(pt + j * slice + e);
        }
      }
#pragma unroll
      for (int v = 0; v < kMaxE / 32; ++v) red[warp][lane + 32 * v] = acc[v];
    }
    __syncthreads();
    if (warp == 0) {
      float z[kMaxE / 32];
      float m = -INFINITY;
#pragma unroll
      for (int v = 0; v < kMaxE / 32; ++v) {
        const int e = lane + 32 * v;
        float zz = -INFINITY;
        if (e < E) {
          zz = 0.f;
#pragma unroll
          for (int w = 0; w < kWarps; ++w) zz += red[w][e];
          // The association of z = (x W_r + bias) + scale * z_prev.
          if (a.bias) zz += zb[v];
          if (a.zprev) zz += zq[v];
          a.logits[(size_t)t * E + e] = zz;
          zs[e] = zz;
        }
        z[v] = zz;
        m = fmaxf(m, zz);
      }
      m = warp_max(m);
      float ex[kMaxE / 32];
      float s = 0.f;
#pragma unroll
      for (int v = 0; v < kMaxE / 32; ++v) {
        ex[v] = (lane + 32 * v < E) ? expf(z[v] - m) : 0.f;
        s += ex[v];
      }
      s = warp_sum(s);
#pragma unroll
      for (int v = 0; v < kMaxE / 32; ++v) {
        const int e = lane + 32 * v;
        if (e < E) {
          const float A = ex[v] / s;
          a.probs[(size_t)t * E + e] = A;
          As[e] = A;
        }
      }
    }
    __syncthreads();
    // Top-k by rank: the candidate (v, e) takes slot #{f : v_f > v or
    // (v_f == v and f < e)} if below k (the picks and order of repeated
    // argmax with ties to the lower id). DES-Vote ranks P and votes with
    // its top-K; DES-Seq ranks P and marks its top-k_local in the union;
    // token choice ranks the logits, weight P.
    if (tid < E) {
      const int e = tid;
      const float *key = core_routed ? As : zs;
      const float ke = key[e];
      int rank = 0;
      for (int f = 0; f < E; ++f) {
        const float kf = key[f];
        rank += (kf > ke) || (kf == ke && f < e);
      }
      if (seq) {
        if (rank < a.k_local)
          atomicOr(reinterpret_cast<unsigned *>(a.votes) + (e >> 5), 1u << (e & 31));
      } else if (rank < k) {
        if (des) {
          atomicAdd(a.votes + e, (unsigned long long)vote_quantum(As[e]));
        } else {
          own_ids[rank] = e;
          own_w[rank] = As[e];
          if (e < nh) atomicOr(a.gmask + 4 * e + (t >> 5), 1u << (t & 31));
        }
      }
    }
    if (!core_routed && a.renorm) {
      __syncthreads();
      if (tid == 0) {
        float ws = 0.f;
        for (int r = 0; r < k; ++r) ws += own_w[r];
        for (int r = 0; r < k; ++r) own_w[r] = own_w[r] / ws;
      }
    }
  }

  // Grid barrier 1: every token's probabilities, votes and picks are out.
  __syncthreads();
  if (tid == 0 && ok_slot) {
    __threadfence();
    atomicAdd(a.sync + 0, 1u);
    ok_slot = wait_u32(a.sync + 0, 2u * (unsigned)G, &abort_flag, a.dev_status) ? 1 : 0;
  }
  __syncthreads();
  bool alive = ok_slot != 0;

  // ---- 2. the experts to stream, identical in every CTA.
  if (alive) {
    bool in = false;
    if (des) {
      if (tid < E) V[tid] = (long long)__ldcg(a.votes + tid);
      __syncthreads();
      if (tid < E) {
        const long long ve = V[tid];
        int rank = 0;
        for (int f = 0; f < E; ++f) {
          const long long vf = V[f];
          rank += (vf > ve) || (vf == ve && f < tid);
        }
        in = rank < a.M_core;
      }
    } else if (seq) {
      if (tid < E) in = (__ldcg(reinterpret_cast<const unsigned *>(a.votes) + (tid >> 5)) >> (tid & 31)) & 1u;
    } else {
      for (int i = tid; i < 4 * nh; i += kThreads) (&mask[0][0])[i] = __ldcg(a.gmask + i);
      __syncthreads();
      if (tid < nh) in = (mask[tid][0] | mask[tid][1] | mask[tid][2] | mask[tid][3]) != 0u;
    }
    // The core set (DES) and the experts to stream (its heavy members; for
    // token choice the heavy experts some token picked), ascending id.
    // Streamed first: experts certain to get rows; last: DES-Vote core
    // members without votes, which get rows only in corner cases (their
    // units are skipped if the routing shows no rows by the time they are
    // claimed).
    const bool streamed = in && tid < nh;
    const bool late = streamed && des && V[tid] == 0;
    if (tid < kMaxE) {
      const unsigned b = __ballot_sync(0xffffffffu, in);
      const unsigned bs = __ballot_sync(0xffffffffu, streamed && !late);
      const unsigned bl = __ballot_sync(0xffffffffu, late);
      if (lane == 0) { wbits[warp] = b; sbits[warp] = bs; lbits[warp] = bl; }
    }
    __syncthreads();
    if (in && core_routed) {
      int pos = __popc(wbits[warp] & ((1u << lane) - 1u));
      for (int w = 0; w < warp; ++w) pos += __popc(wbits[w]);
      core_list[pos] = tid;
      if (t == 0) a.core[pos] = tid;
    }
    if (tid == 0) {
      int n = 0;
#pragma unroll
      for (int w = 0; w < kMaxE / 32; ++w) n += __popc(wbits[w]);
      n_core_s = n;
    }
    __syncthreads();
    // DES-Seq's core list is as long as the union: the rest of the caller's
    // core array reads -1.
    if (seq && t == 0 && tid >= n_core_s && tid < E) a.core[tid] = -1;
    if (streamed) {
      const unsigned *bits = late ? lbits : sbits;
      int pos = __popc(bits[warp] & ((1u << lane) - 1u));
      for (int w = 0; w < warp; ++w) pos += __popc(bits[w]);
      if (late)
        for (int w = 0; w < kMaxE / 32; ++w) pos += __popc(sbits[w]);
      glist[pos] = tid;
    }
    if (des && t == 0 && tid < E && a.votes_out) a.votes_out[tid] = V[tid];
    if (tid == 0) {
      int n = 0;
#pragma unroll
      for (int w = 0; w < kMaxE / 32; ++w) n += __popc(sbits[w]) + __popc(lbits[w]);
      n_groups_s = n;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = tmem_slot;
  const int n_groups = alive ? n_groups_s : 0;
  const int up_N = a.h, up_blocks = (up_N + BMW - 1) / BMW;
  const int down_N = a.d, down_blocks = (down_N + BMW - 1) / BMW;
  const int n_up = n_groups * up_blocks;
  const int total = n_groups * (up_blocks + down_blocks);
  const int w1_rows = a.w1_rows_per_group;

  if (warp == 0) {
    if (lane == 0 && alive) {
      // ---------------- TMA producer
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmW1)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmX)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmW2)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmH)) : "memory");
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_parity = 0;
      bool ok = true, routed = false;
      int qs = 0;
      uint32_t qph = 0;
      while (ok) {
        // Claim the next unit of the grid-wide list (up units first, so an
        // up unit is always claimed before any down unit that waits on it);
        // hand its id to the MMA and epilogue warps; -1 ends the list.
        int u = (int)atomicAdd(a.sync + 2, 1u);
        if (u >= total) u = -1;
        int code = u;
        if (u >= 0 && route_ready) {
          __threadfence_block();  // the offsets written before the flag
          // The routing is known: an expert that got no rows needs no
          // weights (the unit is passed on as skipped: -2 - u).
          const int g0 = glist[unit_of(u, n_groups, up_blocks, down_blocks).gi];
          if (offs[g0 + 1] == offs[g0]) code = -2 - u;
        }
        if (!mbar_wait(uqe0 + 8 * qs, qph ^ 1u, &abort_flag, a.dev_status)) { ok = false; break; }
        uq[qs] = code;
        mbar_arrive(uqf0 + 8 * qs);
        if (++qs == kUQ) { qs = 0; qph ^= 1u; }
        if (u < 0) break;
        if (code < -1) continue;
        const BlockUnit un = unit_of(u, n_groups, up_blocks, down_blocks);
        const bool up = un.up;
        const int g = glist[un.gi];
        const int blk = un.blk;
        const CUtensorMap *mW = up ? &tmW1 : &tmW2;
        const CUtensorMap *mB = up ? &tmX : &tmH;
        const int w_row = up ? g * w1_rows + blk * BMW : g * down_N + blk * BMW;
        int b_row = 0;  // up: all tokens, x rows 0..NB-1 (zero past T)
        if (!up) {
          // The expert's hidden rows: known once this CTA's routing is done,
          // complete once all of the expert's up units are stored.
          if (!routed) {
            if (!wait_local(&route_ready, &abort_flag, a.dev_status)) { ok = false; break; }
            __threadfence_block();  // the offsets written before the flag
            routed = true;
          }
          if (!wait_s32(a.done + g, 4 * up_blocks, &abort_flag, a.dev_status)) { ok = false; break; }
          asm volatile("fence.proxy.async.global;" ::: "memory");
          b_row = offs[g];
        }
        const int K = up ? a.d : a.h;
        const int nkb = (K + BK - 1) / BK;
        const bool paired = up && GATED;
        const int nst = paired ? nkb : (nkb + 1) / 2;
        for (int st = 0; st < nst; ++st) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, &abort_flag, a.dev_status)) { ok = false; break; }
          const uint32_t fb = full0 + 8 * stage;
          const uint32_t a0 = s0 + stage * STAGE_BYTES;
          const uint32_t a1 = a0 + A_BYTES, b0 = a0 + 2 * A_BYTES, b1 = b0 + B_BYTES;
          if (paired) {
            mbar_arrive_expect_tx(fb, 2 * A_BYTES + B_BYTES);
            tma_load_2d(a0, mW, st * BK, w_row, fb);
            tma_load_2d(a1, mW, st * BK, w_row + up_N, fb);
            tma_load_2d(b0, mB, st * BK, b_row, fb);
          } else {
            const bool two = 2 * st + 1 < nkb;
            mbar_arrive_expect_tx(fb, (two ? 2u : 1u) * (A_BYTES + B_BYTES));
            tma_load_2d(a0, mW, 2 * st * BK, w_row, fb);
            tma_load_2d(b0, mB, 2 * st * BK, b_row, fb);
            if (two) {
              tma_load_2d(a1, mW, (2 * st + 1) * BK, w_row, fb);
              tma_load_2d(b1, mB, (2 * st + 1) * BK, b_row, fb);
            }
          }
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // Let every copy this thread started land before the CTA can exit.
      for (int s = 0; s < STAGES; ++s)
        if (armed & (1u << s))
          mbar_wait(full0 + 8 * s, (armed_parity >> s) & 1u, &abort_flag, a.dev_status, false);
    }
  } else if (warp == 1) {
    if (lane == 0 && alive) {
      // ---------------- MMA issuer
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      int qs = 0;
      uint32_t qph = 0;
      while (ok) {
        if (!mbar_wait(uqf0 + 8 * qs, qph, &abort_flag, a.dev_status)) break;
        const int u = uq[qs];
        if (++qs == kUQ) { qs = 0; qph ^= 1u; }
        if (u == -1) break;
        if (u < -1) continue;  // skipped unit: no MMA
        const bool up = u < n_up;
        const int K = up ? a.d : a.h;
        const int nkb = (K + BK - 1) / BK;
        const bool paired = up && GATED;
        const int nst = paired ? nkb : (nkb + 1) / 2;
        if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1u, &abort_flag, a.dev_status)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + (uint32_t)(acc * ACC_COLS);
        for (int st = 0; st < nst; ++st) {
          if (!mbar_wait(full0 + 8 * stage, phase, &abort_flag, a.dev_status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = s0 + stage * STAGE_BYTES;
          const uint32_t a1 = a0 + A_BYTES, b0 = a0 + 2 * A_BYTES, b1 = b0 + B_BYTES;
          const uint64_t da0 = smem_desc_sw128(a0), da1 = smem_desc_sw128(a1);
          const uint64_t db0 = smem_desc_sw128(b0), db1 = smem_desc_sw128(b1);
          if (paired) {
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint32_t accum = (st | kk) != 0 ? 1u : 0u;
              tc_mma(d0, da0 + (uint64_t)(2 * kk), db0 + (uint64_t)(2 * kk), IDESC, accum);
              tc_mma(d0 + NB, da1 + (uint64_t)(2 * kk), db0 + (uint64_t)(2 * kk), IDESC, accum);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              tc_mma(d0, da0 + (uint64_t)(2 * kk), db0 + (uint64_t)(2 * kk), IDESC,
                     (st | kk) != 0 ? 1u : 0u);
            if (2 * st + 1 < nkb) {
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk)
                tc_mma(d0, da1 + (uint64_t)(2 * kk), db1 + (uint64_t)(2 * kk), IDESC, 1u);
            }
          }
          tc_commit(empty0 + 8 * stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(tfull0 + 8 * acc);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      tc_commit(drain);
      mbar_wait(drain, 0, &abort_flag, a.dev_status, false);
    }
  } else if (alive) {
    // ---------------- warps 2..5: routing tail, epilogue, combine
    const int et = tid - 64;  // 0..127
    const int ew = et >> 5;   // 0..3
    bool ok = true;
    if (core_routed) {
      // Re-route the own token over the core set, by rank (the core list
      // ascends, so a lower position is a lower id), and mark the picks:
      // min(K, |core|) of them (DES-Seq's core can be smaller than K; the
      // other slots stay empty).
      const int Mc = des ? a.M_core : n_core_s;
      if (t < T && et < Mc) {
        const int e = core_list[et];
        const float p = As[e];
        int rank = 0;
        for (int c2 = 0; c2 < Mc; ++c2) {
          const float q = As[core_list[c2]];
          rank += (q > p) || (q == p && c2 < et);
        }
        if (rank < k) {
          own_ids[rank] = e;
          own_w[rank] = p;
          if (e < nh) atomicOr(a.gmask + 4 * e + (t >> 5), 1u << (t & 31));
        }
      }
      // Grid barrier 2 among the epilogue warps of all CTAs.
      epi_sync();
      if (et == 0) {
        __threadfence();
        atomicAdd(a.sync + 0, 1u);
        ok_slot = wait_u32(a.sync + 0, 3u * (unsigned)G, &abort_flag, a.dev_status) ? 1 : 0;
      }
      epi_sync();
      ok = ok_slot != 0;
      if (ok)
        for (int i = et; i < 4 * nh; i += kEpiThreads) (&mask[0][0])[i] = __ldcg(a.gmask + i);
    }
    // Row offsets: experts in id order, tokens ascending within an expert.
    epi_sync();
    if (ok) {
      const int cnt = et < nh ? __popc(mask[et][0]) + __popc(mask[et][1]) + __popc(mask[et][2]) +
                                    __popc(mask[et][3])
                              : 0;
      const int inc = warp_inclusive_scan(cnt);
      if (lane == 31) wsum_s[ew] = inc;
      epi_sync();
      int base = 0;
      for (int w = 0; w < ew; ++w) base += wsum_s[w];
      if (et < nh) offs[et] = base + inc - cnt;
      if (et == kEpiThreads - 1) offs[nh] = base + inc;
      epi_sync();
      if (t == 0)
        for (int e = et; e <= nh; e += kEpiThreads) a.offsets[e] = offs[e];
      // The token's slots, for the combine and the caller.
      if (t < T && et < k) {
        const int j = et, i = t * k + j;
        const int e = own_ids[j];
        int row = -1;
        if (e == -1) {
          // an empty slot (DES-Seq with a core smaller than K)
        } else if (e < 0 || e >= E) {
          set_status(a.dev_status, MOE_DEV_BAD_EXPERT);
        } else if (e < nh) {
          const int q = t >> 5;
          int before = __popc(mask[e][q] & ((1u << (t & 31)) - 1u));
          for (int qq = 0; qq < q; ++qq) before += __popc(mask[e][qq]);
          row = offs[e] + before;
          a.perm[row] = t;
        }
        a.sel[i] = e;
        a.w[i] = own_w[j];
        a.row_of[i] = row;
      }
      __threadfence_block();
      epi_sync();
      if (et == 0) {
        route_ready = 1;
        if (t < T) {  // this token's slots are out (for the combine)
          __threadfence();
          atomicAdd(a.sync + 3, 1u);
        }
      }
    }

    // Epilogue: lane j of quadrant q holds feature blk*128 + 32q + j.
    const int quad = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    int qs = 0;
    uint32_t qph = 0;
    while (ok) {
      const bool got = mbar_wait(uqf0 + 8 * qs, qph, &abort_flag, a.dev_status);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      const int code = uq[qs];
      const uint32_t uq_done = uqe0 + 8 * qs;
      if (++qs == kUQ) { qs = 0; qph ^= 1u; }
      if (code == -1) break;
      if (code < -1) {
        // Skipped unit (its expert got no rows): nothing to store, but an
        // up unit still counts toward its expert's arrivals.
        const int su = -2 - code;
        __syncwarp();
        if (lane == 0) {
          if (su < n_up) atomicAdd(a.done + glist[unit_of(su, n_groups, up_blocks, down_blocks).gi], 1);
          mbar_arrive(uq_done);
        }
        continue;
      }
      const int u = code;
      const BlockUnit un = unit_of(u, n_groups, up_blocks, down_blocks);
      const bool up = un.up;
      const int g = glist[un.gi];
      const int blk = un.blk;
      const int N = up ? up_N : down_N;
      const int feat = blk * BMW + quad * 32 + lane;
      const bool valid = feat < N;
      const bool ready = mbar_wait(tfull0 + 8 * acc, acc_phase, &abort_flag, a.dev_status);
      if (!__all_sync(0xffffffffu, ready)) { ok = false; break; }
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * ACC_COLS);
      const int row0 = offs[g];
      if (up) {
        // Column c is token c; keep the tokens that picked expert g.
        __nv_bfloat16 *H = static_cast<__nv_bfloat16 *>(a.H);
        int before = 0;
#pragma unroll 1
        for (int c0 = 0; c0 < NB && c0 < T; c0 += 32) {
          const unsigned mw = mask[g][c0 >> 5];
          if (mw != 0u) {
            float v[32];
            tmem_ld32(taddr + c0, v);
            if (GATED) {
              float uu[32];
              tmem_ld32(taddr + NB + c0, uu);
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = silu(v[i]) * uu[i];
            } else {
#pragma unroll
              for (int i = 0; i < 32; i += 2) gelu_erf_x2(v[i], v[i + 1]);
            }
            if (valid) {
              int r = row0 + before;
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if ((mw >> i) & 1u) H[(int64_t)(r++) * up_N + feat] = __float2bfloat16_rn(v[i]);
            }
          }
          before += __popc(mw);
        }
      } else {
        // Column c is the expert's c-th row.
        __nv_bfloat16 *Y = static_cast<__nv_bfloat16 *>(a.Y);
        const int cnt = offs[g + 1] - row0;
#pragma unroll 1
        for (int c0 = 0; c0 < NB && c0 < cnt; c0 += 32) {
          float v[32];
          tmem_ld32(taddr + c0, v);
          if (valid) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c0 + i < cnt) Y[(int64_t)(row0 + c0 + i) * down_N + feat] = __float2bfloat16_rn(v[i]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(tempty0 + 8 * acc);
        mbar_arrive(uq_done);
      }
      if (up) {
        // Publish this warp's quarter of the hidden rows; a down unit of g
        // waits for 4 arrivals per up unit of g.
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(a.done + g, 1);
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }

    // Combine: y = residual + sum_j w_j * expert_j(x), one warp per (token,
    // 256 features), fp32 in slot order. The warp's first item (its
    // residual and the token's slots, final once every token CTA has
    // signalled) is read before the wait for the last unit of the grid, so
    // only the expert rows are left to read after it.
    const __nv_bfloat16 *x = static_cast<const __nv_bfloat16 *>(a.x);
    const __nv_bfloat16 *res = static_cast<const __nv_bfloat16 *>(a.residual);  // may alias y
    const __nv_bfloat16 *cv = static_cast<const __nv_bfloat16 *>(a.const_vecs);
    const __nv_bfloat16 *Yp = static_cast<const __nv_bfloat16 *>(a.Y);
    __nv_bfloat16 *y = static_cast<__nv_bfloat16 *>(a.y);
    const int d = a.d;
    const int chunks = (d + 255) / 256;
    const int items = T * chunks;
    struct Item {
      float acc8[8];
      const __nv_bfloat16 *m_src;
      bool m_l2;  // an expert row written by this grid (read via L2)
      float m_w;
    };
    // Lane j holds slot j of the token: weight and source row.
    auto prepare = [&](int it, Item &p) {
      const int s = it / chunks;
      const int c0 = (it - s * chunks) * 256 + lane * 8;
#pragma unroll
      for (int i = 0; i < 8; ++i) p.acc8[i] = 0.f;
      if (c0 < d && res) load8(res + (size_t)s * d + c0, p.acc8);
      p.m_src = nullptr;
      p.m_l2 = false;
      p.m_w = 0.f;
      if (lane < k) {
        const int i = s * k + lane;
        const int e = __ldcg(a.sel + i);
        const int row = __ldcg(a.row_of + i);
        const float wv = __ldcg(a.w + i);
        if (e >= 0 && e < E) {
          const int kind = kinds.kind[e];
          if (kind == MOE_HEAVY) {
            if (row >= 0) { p.m_src = Yp + (size_t)row * d; p.m_l2 = true; }
          } else if (kind == MOE_IDENTITY) {
            p.m_src = x + (size_t)s * d;
          } else if (kind == MOE_CONST) {
            p.m_src = cv + (size_t)kinds.cidx[e] * d;
          }
          p.m_w = wv;
        }
      }
    };
    auto finish = [&](int it, Item &p) {
      const int s = it / chunks;
      const int c0 = (it - s * chunks) * 256 + lane * 8;
      const bool live = c0 < d;
      for (int jb = 0; jb < k; jb += 8) {  // 8 slots' rows in flight together
        uint4 raw[8];
        const __nv_bfloat16 *src[8];
        float wgt[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int j = (jb + q) & 31;
          src[q] = reinterpret_cast<const __nv_bfloat16 *>(
              __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(p.m_src), j));
          const bool l2 = __shfl_sync(0xffffffffu, p.m_l2, j);
          wgt[q] = __shfl_sync(0xffffffffu, p.m_w, j);
          if (jb + q >= k || !live) src[q] = nullptr;
          if (src[q])
            raw[q] = l2 ? ld_cg_v4(src[q] + c0) : *reinterpret_cast<const uint4 *>(src[q] + c0);
        }
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (src[q]) fma8(wgt[q], raw[q], p.acc8);
      }
      if (live) store8(y + (size_t)s * d + c0, p.acc8);
    };

    epi_sync();
    if (et == 0) {
      int sok = 0;
      if (ok && !abort_flag) {
        __threadfence();
        atomicAdd(a.sync + 1, 1u);  // this CTA's units are stored
        sok = wait_u32(a.sync + 3, (unsigned)T, &abort_flag, a.dev_status) ? 1 : 0;
      }
      ok_slot = sok;
    }
    epi_sync();
    const bool slots_ok = ok_slot != 0;
    // Items go to warps in the order their CTAs finish their units (a
    // ticket per warp), so the CTAs that finish first take them.
    auto claim = [&]() {
      int it = 0;
      if (lane == 0) it = (int)atomicAdd(a.sync + 4, 1u);
      return __shfl_sync(0xffffffffu, it, 0);
    };
    const int it0 = slots_ok ? claim() : items;
    Item first;
    if (it0 < items) prepare(it0, first);
    epi_sync();
    if (et == 0)
      ok_slot = (slots_ok && wait_u32(a.sync + 1, (unsigned)G, &abort_flag, a.dev_status)) ? 1 : 0;
    epi_sync();
    if (ok_slot) {
      // With no more items than warps every item went out in the first
      // round of claims; only claim again when there are more.
      for (int it = it0; it < items; it = items > 4 * G ? claim() : items) {
        if (it == it0) {
          finish(it, first);
        } else {
          Item p;
          prepare(it, p);
          finish(it, p);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TMEM_COLS)
                 : "memory");
  }
}

template <int NB, int ACT>
int run_block(const BlockArgs &a, const KindTable &kinds, const void *W1, const void *W2,
              cudaStream_t stream) {
  constexpr uint32_t STAGE_BYTES = 2 * BMW * BK * 2 + 2 * NB * BK * 2;
  constexpr int S0 = (200 * 1024) / STAGE_BYTES;
  constexpr int STAGES = S0 > 8 ? 8 : S0;
  const size_t smem = 1024 + (size_t)STAGES * STAGE_BYTES;
  const int64_t na = (int64_t)a.T * a.k;
  CUtensorMap mW1, mX, mW2, mH;
  if (!make_tma_2d_bf16(&mW1, W1, (int64_t)a.n_heavy * a.w1_rows_per_group, a.d, BMW) ||
      !make_tma_2d_bf16(&mX, a.x, a.T, a.d, NB) ||
      !make_tma_2d_bf16(&mW2, W2, (int64_t)a.n_heavy * a.d, a.h, BMW) ||
      !make_tma_2d_bf16(&mH, a.H, na > 0 ? na : 1, a.h, NB))
    return MOE_ERR_CUDA;
  auto kern = moe_block_kernel<NB, ACT>;
  MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(num_sms());  // one CTA per SM; CTAs t < T own token t
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // the grid-wide waits need every CTA resident
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  MOE_CUDA_TRY(cudaLaunchKernelEx(&cfg, kern, mW1, mX, mW2, mH, a, kinds));
  return last_launch_status();
}

}  // namespace

bool moe_block_supported(const moe_config &c) {
  return c.dtype == MOE_BF16 &&
         (c.routing == MOE_TOKEN_TOPK || c.routing == MOE_DES_VOTE || c.routing == MOE_DES_SEQ) &&
         c.T >= 1 && c.T <= 128 && c.T < num_sms() && c.E >= 1 && c.E <= kMaxE && c.k >= 1 &&
         c.k <= kMaxK && c.n_shared == 0 && c.n_heavy >= 0 && c.h >= 8 && c.d >= 8 &&
         c.const_mix == 0 &&
         c.d <= 32768;
}

// About 32 slices: a token's partial sums stay one round of loads, and
// each slice's operands (T + E rows of the slice) are a few KB; a slice is
// a multiple of 16 columns (the MMA's K) and at most 256 so that its
// staging fits the operand ring.
int block_router_slices(int d, int *kslice) {
  int ks = (d + 31) / 32;
  ks = (ks + 15) & ~15;
  if (ks < 32) ks = 32;
  if (ks > 256) ks = 256;
  *kslice = ks;
  return (d + ks - 1) / ks;
}

// Zeroed region: 8 sync words, 4 mask words per expert, the int64 vote
// totals, one arrival counter per heavy expert.
size_t block_zero_bytes(int E, int n_heavy) {
  return (size_t)(8 + 4 * E) * 4 + (size_t)E * 8 + (size_t)(n_heavy + 1) * 4;
}

void block_zero_layout(BlockArgs &a, void *z, int E) {
  uint8_t *p = static_cast<uint8_t *>(z);
  a.sync = reinterpret_cast<unsigned *>(p);
  a.gmask = reinterpret_cast<unsigned *>(p) + 8;
  a.votes = reinterpret_cast<unsigned long long *>(p + (size_t)(8 + 4 * E) * 4);
  a.done = reinterpret_cast<int32_t *>(p + (size_t)(8 + 4 * E) * 4 + (size_t)E * 8);
}

int launch_moe_block(const BlockArgs &a, const KindTable &kinds, const void *W1, const void *W2,
                     int act, cudaStream_t stream) {
  const bool gated = act == MOE_SWIGLU;
  if (a.T <= 32)
    return gated ? run_block<32, kActSwiglu>(a, kinds, W1, W2, stream)
                 : run_block<32, kActGelu>(a, kinds, W1, W2, stream);
  if (a.T <= 64)
    return gated ? run_block<64, kActSwiglu>(a, kinds, W1, W2, stream)
                 : run_block<64, kActGelu>(a, kinds, W1, W2, stream);
  if (a.T <= 128)
    return gated ? run_block<128, kActSwiglu>(a, kinds, W1, W2, stream)
                 : run_block<128, kActGelu>(a, kinds, W1, W2, stream);
  return MOE_ERR_UNSUPPORTED;
}

}  // namespace moe
