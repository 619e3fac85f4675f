// Small-block routing tail, one cooperative kernel: router finish ->
// (DES-Vote election and re-route) -> dispatch -> row gather.
//
// For a block of T <= 128 tokens every one of these steps is a few
// microseconds of latency and almost no work, so separate launches cost
// more than the work. One CTA per token:
//   phase 1: sum the router's split-K partial logits for the token (warps
//     over slices, lanes over experts, a fixed order: deterministic), add
//     bias and gate residual, softmax, then either the token-choice top-k
//     or the DES-Vote top-K votes (exact int64 fixed point, atomics).
//     Token choice also marks its picks in per-expert token bitmasks.
//   grid barrier (bounded wait; on expiry the CTA flags MOE_DEV_TIMEOUT,
//     leaves its token's slots empty -- expert -1, weight 0, no row -- and,
//     in CTA 0, zero row offsets, so the later stages of the layer see an
//     empty, in-bounds routing for what did not finish).
//   DES only: every CTA re-runs the same election from the summed votes,
//     re-routes its own token over the core set, marks its picks in the
//     bitmasks; second grid barrier.
//   phase 2: every CTA reads the bitmasks, derives the per-expert row
//     offsets and its own token's rows (tokens ascending within an
//     expert), writes its slots and copies its x row (loaded at kernel
//     start) to each of its expert rows; CTA 0 writes the offsets and the
//     core set.
// Every top-k here is computed by ranks, not by k rounds of argmax: the
// candidate (v, e) takes slot #{f : v_f > v or (v_f == v and f < e)} if
// that is below k, so all candidates are placed at once with no serial
// chain (the same picks and order as repeated argmax with ties to the
// lower id).
//
// Dynamic Expert Sharing: Decoupling Memory from Parallelism in MoE
// Diffusion LLMs, section 2.4 (DES-Vote): each token keeps its top-K
// experts and votes for them with its routing weights; the M_core most
// voted experts form the core set and every token re-routes to its top-K
// experts within the core set.
// EC-DiT: Scaling Diffusion Transformers with Adaptive Expert-Choice
// Routing, section 3 (Token-Choice routing): each token keeps its top-k.
// DICE: Staleness-Centric Optimizations for Parallel Diffusion MoE
// Inference, Conditional Communication: tokens are dispatched to their
// experts (here: rows grouped by expert, ascending by token, in HBM).
#include <math.h>
#include <string.h>

#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxE = 128;
constexpr int kXVecs = 4;  // x-row vectors held per thread from the start (rows <= 8192 bf16)
constexpr uint64_t kBarrierTimeoutNs = 2000000000ull;

// Test hook (moe_test_set_barrier_wait): a shorter wait limit and extra
// arrivals the grid barriers wait for, read at each launch.
std::atomic<unsigned long long> g_test_wait_ns{0};
std::atomic<int> g_test_extra_arrivals{0};

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// 16-byte read-only load issued where it stands (not sunk to its use).
__device__ __forceinline__ uint4 ld_nc_v4(const uint4 *p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// Grid barrier among the co-resident CTAs: arrive, then wait (at most
// `limit_ns`) until `target` arrivals. Returns false if the wait expired.
__device__ __forceinline__ bool grid_barrier(unsigned *ctr, unsigned target, uint64_t limit_ns,
                                             int *ok_slot) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(ctr, 1u);
    int ok = 1;
    if (ld_acquire_u32(ctr) < target) {
      const uint64_t t0 = global_timer_ns();
      while (ld_acquire_u32(ctr) < target) {
        if (global_timer_ns() - t0 > limit_ns) { ok = 0; break; }
        __nanosleep(32);
      }
    }
    *ok_slot = ok;
  }
  __syncthreads();
  return *ok_slot != 0;
}

// After an expired barrier: flag the timeout and leave this CTA's token
// with empty slots (and, in CTA 0, zero row offsets) so that the dispatch
// outputs the later stages read stay in bounds. CTA-wide.
__device__ __forceinline__ void abandon_token(const SmallRouteArgs &a, int t) {
  const int tid = threadIdx.x;
  if (tid == 0) set_status(a.dev_status, MOE_DEV_TIMEOUT);
  if (tid < a.k) {
    const int i = t * a.k + tid;
    a.sel[i] = -1;
    a.w[i] = 0.f;
    a.row_of[i] = -1;
  }
  if (t == 0)
    for (int e = tid; e <= a.n_heavy; e += kThreads) a.offsets[e] = 0;
}

// DES election, identical in every CTA: the M_core largest vote totals
// (ties to the lower id); the core set in ascending id order. CTA-wide
// (all threads call it).
__device__ __forceinline__ void elect(const SmallRouteArgs &a, long long *V, unsigned *core_wmask,
                                      int *core_list, bool write_core) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = a.E, Mc = a.M_core;
  if (tid < E) V[tid] = (long long)__ldcg(a.votes + tid);
  __syncthreads();
  bool in = false;
  if (tid < E) {
    const long long ve = V[tid];
    int rank = 0;
    for (int f = 0; f < E; ++f) {
      const long long vf = V[f];
      rank += (vf > ve) || (vf == ve && f < tid);
    }
    in = rank < Mc;
  }
  if (tid < kMaxE) {
    const unsigned b = __ballot_sync(0xffffffffu, in);
    if (lane == 0) core_wmask[warp] = b;
  }
  __syncthreads();
  if (in) {
    int pos = __popc(core_wmask[warp] & ((1u << lane) - 1u));
    for (int w = 0; w < warp; ++w) pos += __popc(core_wmask[w]);
    core_list[pos] = tid;
    if (write_core) a.core[pos] = tid;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kThreads)
small_route_kernel(SmallRouteArgs a) {
  __shared__ float red[kWarps][kMaxE];
  __shared__ float zs[kMaxE], As[kMaxE];
  __shared__ long long V[kMaxE];
  __shared__ int core_list[kMaxE];
  __shared__ unsigned core_wmask[kMaxE / 32];
  __shared__ int offs[kMaxE + 1];
  __shared__ unsigned mask[kMaxE][4];  // tokens (<= 128) that chose expert e
  __shared__ int own_ids[kSmallRouteMaxK];
  __shared__ float own_w[kSmallRouteMaxK];
  __shared__ int own_row[kSmallRouteMaxK];
  __shared__ int scratch[33];
  __shared__ int barrier_ok;

  const int t = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int T = a.T, E = a.E, k = a.k;
  const bool des = a.routing == MOE_DES_VOTE;

  if (tid < kSmallRouteMaxK) { own_ids[tid] = -1; own_w[tid] = 0.f; }  // a pick not made stays -1

  // x row t and the router's per-expert terms, read now so that nothing
  // later waits on them.
  const uint4 *src = a.x + (size_t)t * a.row_vecs;
  uint4 xv[kXVecs];
#pragma unroll
  for (int i = 0; i < kXVecs; ++i) {
    const int v = tid + i * kThreads;
    if (v < a.row_vecs) xv[i] = ld_nc_v4(src + v);
  }
  float zb[kMaxE / 32], zq[kMaxE / 32];
  if (warp == 0) {
#pragma unroll
    for (int v = 0; v < kMaxE / 32; ++v) {
      const int e = lane + 32 * v;
      zb[v] = (e < E && a.bias) ? __ldg(a.bias + e) : 0.f;
      zq[v] = (e < E && a.zprev) ? a.zscale * __ldg(a.zprev + (size_t)t * E + e) : 0.f;
    }
  }

  // ---- phase 1: finish token t.
  {
    float acc[kMaxE / 32];
#pragma unroll
    for (int v = 0; v < kMaxE / 32; ++v) acc[v] = 0.f;
    const float *pt = a.part + (size_t)t * E;
    const size_t slice = (size_t)T * E;
#pragma unroll 4
    for (int j = warp; j < a.n_part; j += kWarps) {
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
        // The same association as z = (x W_r + bias) + scale * z_prev.
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
  // Top-k of the token by rank: DES ranks P (and votes with it), token
  // choice ranks the logits (weight P) and marks its picks.
  if (tid < E) {
    const int e = tid;
    const float *key = des ? As : zs;
    const float ke = key[e];
    int rank = 0;
    for (int f = 0; f < E; ++f) {
      const float kf = key[f];
      rank += (kf > ke) || (kf == ke && f < e);
    }
    if (rank < k) {
      if (des) {
        atomicAdd(a.votes + e, (unsigned long long)vote_quantum(As[e]));
      } else {
        own_ids[rank] = e;
        own_w[rank] = As[e];
        if (e < a.n_heavy) atomicOr(a.gmask + 4 * e + (t >> 5), 1u << (t & 31));
      }
    }
  }
  if (!des && a.renorm) {
    __syncthreads();
    if (tid == 0) {
      float ws = 0.f;
      for (int r = 0; r < k; ++r) ws += own_w[r];
      for (int r = 0; r < k; ++r) own_w[r] = own_w[r] / ws;
    }
  }

  if (!grid_barrier(a.barrier, T + a.extra_arrivals, a.wait_ns, &barrier_ok)) {
    abandon_token(a, t);
    return;
  }

  if (des) {
    const int Mc = a.M_core;
    elect(a, V, core_wmask, core_list, t == 0);
    // Re-route the own token: its K largest P over the core set, by rank.
    if (tid < Mc) {
      const int e = core_list[tid];
      const float p = As[e];
      int rank = 0;
      for (int c2 = 0; c2 < Mc; ++c2) {
        const float q = As[core_list[c2]];
        rank += (q > p) || (q == p && c2 < tid);
      }
      if (rank < k) {
        own_ids[rank] = e;
        own_w[rank] = p;
        if (e < a.n_heavy) atomicOr(a.gmask + 4 * e + (t >> 5), 1u << (t & 31));
      }
    }
    if (!grid_barrier(a.barrier, 2 * T + 2 * a.extra_arrivals, a.wait_ns, &barrier_ok)) {
      abandon_token(a, t);
      return;
    }
  } else {
    __syncthreads();
  }

  // ---- phase 2: per-expert token masks -> row offsets and own rows.
  const int nh = a.n_heavy;
  for (int i = tid; i < 4 * nh; i += kThreads) (&mask[0][0])[i] = __ldcg(a.gmask + i);
  __syncthreads();
  {
    int cnt = 0;
    if (tid < nh) cnt = __popc(mask[tid][0]) + __popc(mask[tid][1]) + __popc(mask[tid][2]) +
                        __popc(mask[tid][3]);
    int total;
    const int off = block_exclusive_scan(cnt, scratch, &total);
    if (tid < nh) offs[tid] = off;
    if (tid == 0) offs[nh] = total;
  }
  __syncthreads();
  if (t == 0)
    for (int e = tid; e <= nh; e += kThreads) a.offsets[e] = offs[e];

  // Own token's slots: row = first row of the expert + tokens before t.
  if (tid < k) {
    const int j = tid, i = t * k + j;
    const int e = own_ids[j];
    int row = -1;
    if (e < 0 || e >= E) {
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
    own_row[j] = row;
  }
  __syncthreads();

  // Copy x row t to each of its expert rows (16-byte vectors).
#pragma unroll
  for (int i = 0; i < kXVecs; ++i) {
    const int v = tid + i * kThreads;
    if (v < a.row_vecs)
      for (int j = 0; j < k; ++j) {
        const int row = own_row[j];
        if (row >= 0) a.x_perm[(size_t)row * a.row_vecs + v] = xv[i];
      }
  }
  for (int v = tid + kXVecs * kThreads; v < a.row_vecs; v += kThreads) {
    const uint4 val = __ldg(src + v);
    for (int j = 0; j < k; ++j) {
      const int row = own_row[j];
      if (row >= 0) a.x_perm[(size_t)row * a.row_vecs + v] = val;
    }
  }
}

}  // namespace

bool small_route_supported(int T, int E, int k, int routing, int dtype) {
  return dtype == MOE_BF16 && (routing == MOE_TOKEN_TOPK || routing == MOE_DES_VOTE) &&
         T >= 1 && T <= kSmallRouteMaxTokens && E >= 1 && E <= kMaxE && k >= 1 &&
         k <= kSmallRouteMaxK && (int64_t)T * k <= kSmallRouteMaxAssign;
}

void set_small_route_test_wait(unsigned long long limit_ns, int extra_arrivals) {
  g_test_wait_ns.store(limit_ns);
  g_test_extra_arrivals.store(extra_arrivals);
}

int launch_small_route(const SmallRouteArgs &args, cudaStream_t stream) {
  if (args.T == 0) return MOE_OK;
  if (!small_route_supported(args.T, args.E, args.k, args.routing, MOE_BF16)) return MOE_ERR_UNSUPPORTED;
  SmallRouteArgs a = args;
  const unsigned long long test_ns = g_test_wait_ns.load();
  a.wait_ns = test_ns ? test_ns : kBarrierTimeoutNs;
  a.extra_arrivals = g_test_extra_arrivals.load();
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(a.T);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // the grid barriers need every CTA resident
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  MOE_CUDA_TRY(cudaLaunchKernelEx(&cfg, small_route_kernel, a));
  return MOE_OK;
}

}  // namespace moe
