// Grouped expert GEMM on Blackwell tensor cores: D = act(A . B_g^T),
// bf16 operands, fp32 accumulation in tensor memory.
//
// MMOE: Modernizing Diffusion Transformers with Efficient Expert Design,
// "MoE++ expert layer": heavy experts are standard MLPs (GELU here, SwiGLU
// for the dLLM experts); "shared experts": an always-active dense expert.
// Each launch runs up to two problems (the routed experts, whose row groups
// are read from device offsets, and the shared expert over all tokens) as
// one persistent tile stream, so no host synchronisation is needed and
// experts without tokens (and the zero-computation experts, which never get
// rows) issue no MMA at all.
//
// Per CTA (one per SM, persistent over tiles):
//   warp 0       TMA producer: 128x64 A tile + BNx64 B tile per stage,
//                128-byte swizzle, into a STAGES-deep shared-memory ring
//   warp 1       MMA issuer: one thread issues tcgen05.mma (M=128, N=BN,
//                K=16) into a double-buffered TMEM accumulator and frees
//                ring slots / publishes accumulators with tcgen05.commit
//   warps 2..9   epilogue: tcgen05.ld of the accumulator (two warps per
//                TMEM lane quadrant, each taking half the columns),
//                activation, rounding; bf16 tiles go out as TMA stores
//                from a 32 x 32 staging tile per warp (per-lane stores
//                for rows past a group's end and for fp32); overlaps the
//                next tile's MMAs
// SwiGLU: the B tile holds BN/2 gate rows and the matching BN/2 up rows, so
// one accumulator carries both halves and the epilogue forms
// silu(gate) * up without another pass.
// Every mbarrier wait is bounded: on expiry the kernel flags
// MOE_DEV_TIMEOUT, lets its in-flight copies and MMAs finish (again with a
// bound), frees its tensor memory and returns.
#include <string.h>

#include <algorithm>
#include <functional>
#include <queue>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace moe {
namespace {

using namespace tc;

constexpr int BM = 128;
constexpr int BK = 64;  // 64 bf16 = 128 bytes = one swizzle atom row
constexpr int kEpiWarps = 8;                    // two per TMEM lane quadrant
constexpr int kThreads = 64 + 32 * kEpiWarps;   // producer warp, MMA warp, epilogue warps
constexpr int kMaxEntries = 2 * kMaxLayerExperts + 2;  // (problem, group) entries of a launch
constexpr uint32_t kStageOutBytes = 32 * 32 * 2;           // an epilogue warp's 32 x 32 bf16 staging tile

struct ProbDev {
  const int32_t *offsets;
  int n_groups;
  int64_t a_rows;
  int b_rows_per_group;
  int N, K;
  void *out;
  int64_t ld_out;
  int vec32;  // rows of `out` start on 32-byte boundaries: 256-bit stores
  const __nv_bfloat16 *residual;  // optional, added before rounding (bf16 outputs)
  int64_t ld_res;
  int tma_out;  // bf16 output stored by TMA from shared-memory staging tiles (one-SM kernel)
};
struct ParamsDev {
  int n_probs;
  ProbDev pr[2];
  int32_t *status;
};

struct Sched {
  int n_entries;
  int total_tiles;
  int prob_end[2];  // tiles of problem 0 are [0, prob_end[0]), problem 1 [prob_end[0], prob_end[1])
  int tile_start[kMaxEntries + 1];
  int prob[kMaxEntries];
  int group[kMaxEntries];
  int row0[kMaxEntries];
  int row_end[kMaxEntries];
};

// The tiles one CTA pair runs, in order. Every tile of a problem costs the
// same (its K blocks), so with two problems of different K a round-robin
// deal can leave some pairs a whole long tile behind the others, which
// matters when there are few tiles per pair. Instead the longer problem's
// tiles are dealt round-robin first, and then each tile of the shorter
// problem, in order, goes to the pair that becomes free first (list
// scheduling with known durations, equal free times to the lower id). After
// the long deal the pairs below r hold one long tile more than the rest, so
// pair c's m-th short slot starts at a known time and its rank in the
// merged (start time, pair id) order, which is the short tile it gets, has a
// closed form. Tiles close in the order still run at about the same time,
// as with round-robin. Equal K (or one problem) is round-robin over the
// whole table.
struct TileSeq {
  int c, P;
  int startA, nA, startB, nB;
  int a, b, r, plo;
  int j, m;

  __device__ void init(const Sched &s, int kb0, int kb1, int n_probs, int id, int n) {
    c = id; P = n; j = id; m = 0;
    const int n0 = s.prob_end[0], n1 = n_probs > 1 ? s.prob_end[1] - s.prob_end[0] : 0;
    if (n1 == 0 || n0 == 0 || kb0 == kb1) {
      startA = 0; nA = s.total_tiles; startB = 0; nB = 0; a = b = 1;
    } else if (kb0 > kb1) {
      startA = 0; nA = n0; a = kb0; startB = n0; nB = n1; b = kb1;
    } else {
      startA = n0; nA = n1; a = kb1; startB = 0; nB = n0; b = kb0;
    }
    r = nA % P;
    plo = P - r;
  }
  // Next tile of this pair, or -1.
  __device__ int next() {
    if (j < nA) { const int t = startA + j; j += P; return t; }
    if (nB == 0) return -1;
    int pos;
    if (c >= r) {  // free at m*b (relative to the lower load after the long deal)
      const int t = m * b;
      const int hi_before = t >= a ? (t - a) / b + 1 : 0;  // slots of the r loaded pairs at times <= t
      pos = m * plo + (c - r) + r * hi_before;
    } else {       // free at a + m*b
      const int t = a + m * b;
      const int lo_before = (t + b - 1) / b;               // slots of the others at times < t
      pos = m * r + c + plo * lo_before;
    }
    ++m;
    return pos < nB ? startB + pos : -1;
  }
};

__device__ __forceinline__ int find_entry(const Sched &s, int t) {
  int lo = 0, hi = s.n_entries - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (s.tile_start[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ void st_global_v8(void *p, const uint32_t (&w)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(w[0]), "r"(w[1]),
               "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

// 32 consecutive output columns of one row: whole 32-byte sectors per
// store when rows are 32-byte aligned, 16-byte stores otherwise, scalar
// stores at a ragged right edge.
template <bool OUT_F32>
__device__ __forceinline__ void store_row32(const ProbDev &pr, int row, int col, const float (&v)[32]) {
  if (OUT_F32) {
    float *o = static_cast<float *>(pr.out) + (int64_t)row * pr.ld_out + col;
    if (col + 32 <= pr.N) {
      if (pr.vec32) {
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          uint32_t w[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) w[j] = __float_as_uint(v[i + j]);
          st_global_v8(o + i, w);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4 *>(o + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
      }
    } else {
      for (int i = 0; i < 32 && col + i < pr.N; ++i) o[i] = v[i];
    }
  } else {
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(pr.out) + (int64_t)row * pr.ld_out + col;
    float r[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = 0.f;
    if (pr.residual) {
      const __nv_bfloat16 *rp = pr.residual + (int64_t)row * pr.ld_res + col;
      if (col + 32 <= pr.N) {
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          float t[8];
          load8(rp + i, t);
#pragma unroll
          for (int j = 0; j < 8; ++j) r[i + j] = t[j];
        }
      } else {
        for (int i = 0; i < 32 && col + i < pr.N; ++i) r[i] = __bfloat162float(rp[i]);
      }
    }
    if (col + 32 <= pr.N) {
      uint32_t w[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * j] + r[2 * j], v[2 * j + 1] + r[2 * j + 1]);
        w[j] = *reinterpret_cast<uint32_t *>(&h2);
      }
      if (pr.vec32) {
        st_global_v8(o, *reinterpret_cast<const uint32_t(*)[8]>(&w[0]));
        st_global_v8(o + 16, *reinterpret_cast<const uint32_t(*)[8]>(&w[8]));
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          *reinterpret_cast<uint4 *>(o + 8 * i) = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
      }
    } else {
      for (int i = 0; i < 32 && col + i < pr.N; ++i) o[i] = __float2bfloat16_rn(v[i] + r[i]);
    }
  }
}

// 32 consecutive output columns of this lane's row as bf16 (residual added
// before rounding), written as row `lane` of the warp's 32 x 32 staging tile
// in the TMA 64-byte swizzle: 16-byte chunk q of row r lands at chunk
// q ^ ((r >> 1) & 3), so the 32 lanes' 16-byte writes spread over all banks.
// Columns past N are staged as zero and clipped by the TMA store.
__device__ __forceinline__ void stage_row32_bf16(const ProbDev &pr, int row, int col, const float (&v)[32],
                                                 uint32_t stg, int lane) {
  float r[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) r[i] = 0.f;
  const bool full = col + 32 <= pr.N;
  if (pr.residual) {
    const __nv_bfloat16 *rp = pr.residual + (int64_t)row * pr.ld_res + col;
    if (full) {
#pragma unroll
      for (int i = 0; i < 32; i += 8) {
        float t[8];
        load8(rp + i, t);
#pragma unroll
        for (int j = 0; j < 8; ++j) r[i + j] = t[j];
      }
    } else {
      for (int i = 0; i < 32 && col + i < pr.N; ++i) r[i] = __bfloat162float(rp[i]);
    }
  }
  uint32_t w[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const bool in = full || col + 2 * j < pr.N;
    __nv_bfloat162 h2 = __floats2bfloat162_rn(in ? v[2 * j] + r[2 * j] : 0.f,
                                              in ? v[2 * j + 1] + r[2 * j + 1] : 0.f);
    w[j] = *reinterpret_cast<uint32_t *>(&h2);
  }
  const uint32_t rowaddr = stg + (uint32_t)lane * 64u;
  const uint32_t sw = (uint32_t)((lane >> 1) & 3);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(rowaddr + (((uint32_t)q ^ sw) << 4)),
                 "r"(w[4 * q]), "r"(w[4 * q + 1]), "r"(w[4 * q + 2]), "r"(w[4 * q + 3])
                 : "memory");
}

template <int BN, int ACT, bool OUT_F32, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                       const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                       const __grid_constant__ CUtensorMap tmO0, const __grid_constant__ CUtensorMap tmO1,
                       const ParamsDev p) {
  constexpr int BNO = (ACT == kActSwiglu) ? BN / 2 : BN;  // output columns per tile
  constexpr uint32_t A_BYTES = BM * BK * 2;
  constexpr uint32_t B_BYTES = BN * BK * 2;
  constexpr uint32_t STAGE_TX = A_BYTES + B_BYTES;
  constexpr uint32_t TMEM_COLS = (2 * BN <= 256) ? 256 : 512;
  constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN);

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[2 * STAGES + 5];
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ Sched sched;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~(uintptr_t)1023);
  const uint32_t sA = smem_u32(base);
  const uint32_t sB = sA + STAGES * A_BYTES;
  const uint32_t sO = sB + STAGES * B_BYTES;  // the epilogue warps' staging tiles
  const uint32_t full0 = smem_u32(&bars[0]);
  const uint32_t empty0 = smem_u32(&bars[STAGES]);
  const uint32_t tfull0 = smem_u32(&bars[2 * STAGES]);
  const uint32_t tempty0 = smem_u32(&bars[2 * STAGES + 2]);
  const uint32_t drain = smem_u32(&bars[2 * STAGES + 4]);

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull0 + 8 * a, 1);
      mbar_init(tempty0 + 8 * a, kEpiWarps);
    }
    mbar_init(drain, 1);
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
  if (warp == 2) {
    // Tile table: one entry per (problem, group); tiles are (entry, m, n), n fastest.
    int run = 0, ne = 0;
    for (int pi = 0; pi < p.n_probs; ++pi) {
      const ProbDev &pr = p.pr[pi];
      const int ntn = (pr.N + BNO - 1) / BNO;
      for (int g0 = 0; g0 < pr.n_groups; g0 += 32) {
        int g = g0 + lane;
        int lo = 0, hi = 0;
        if (g < pr.n_groups) {
          lo = pr.offsets ? pr.offsets[g] : 0;
          hi = pr.offsets ? pr.offsets[g + 1] : (int)pr.a_rows;
          check_group_rows(lo, hi, pr.a_rows, p.status);
        }
        int tiles = (g < pr.n_groups && hi > lo) ? ((hi - lo + BM - 1) / BM) * ntn : 0;
        int inc = warp_inclusive_scan(tiles);
        if (g < pr.n_groups) {
          const int e = ne + lane;
          sched.tile_start[e] = run + inc - tiles;
          sched.prob[e] = pi;
          sched.group[e] = g;
          sched.row0[e] = lo;
          sched.row_end[e] = hi;
        }
        run += __shfl_sync(0xffffffffu, inc, 31);
        ne += min(32, pr.n_groups - g0);
      }
      if (lane == 0) sched.prob_end[pi] = run;
    }
    if (lane == 0) {
      if (p.n_probs < 2) sched.prob_end[1] = run;
      sched.n_entries = ne;
      sched.total_tiles = run;
      sched.tile_start[ne] = run;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  const int total_tiles = sched.total_tiles;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA0)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB0)) : "memory");
    int stage = 0;
    uint32_t phase = 0;
    uint32_t armed = 0, armed_parity = 0;  // per-stage bits: ever armed / parity of last arming
    bool ok = true;
    for (int t = blockIdx.x; ok && t < total_tiles; t += gridDim.x) {
      const int e = find_entry(sched, t);
      const int pi = sched.prob[e];
      const ProbDev &pr = p.pr[pi];
      const int ntn = (pr.N + BNO - 1) / BNO;
      const int local = t - sched.tile_start[e];
      const int mt = local / ntn, nt = local - mt * ntn;
      const int a_row = sched.row0[e] + mt * BM;
      const int b_row = sched.group[e] * pr.b_rows_per_group + nt * BNO;
      const int b_row2 = (ACT == kActSwiglu) ? b_row + pr.N : b_row + BN / 2;
      const CUtensorMap *mA = pi ? &tmA1 : &tmA0;
      const CUtensorMap *mB = pi ? &tmB1 : &tmB0;
      const int nkb = (pr.K + BK - 1) / BK;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, &abort_flag, p.status)) { ok = false; break; }
        const uint32_t fb = full0 + 8 * stage;
        mbar_arrive_expect_tx(fb, STAGE_TX);
        const uint32_t dA = sA + stage * A_BYTES, dB = sB + stage * B_BYTES;
        tma_load_2d(dA, mA, kb * BK, a_row, fb);
        tma_load_2d(dB, mB, kb * BK, b_row, fb);
        tma_load_2d(dB + B_BYTES / 2, mB, kb * BK, b_row2, fb);
        armed |= 1u << stage;
        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    // Let every copy this thread started land before the CTA can exit.
    for (int s = 0; s < STAGES; ++s)
      if (armed & (1u << s))
        mbar_wait(full0 + 8 * s, (armed_parity >> s) & 1u, &abort_flag, p.status, false);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    int stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < total_tiles; t += gridDim.x) {
      const int e = find_entry(sched, t);
      const int nkb = (p.pr[sched.prob[e]].K + BK - 1) / BK;
      if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1u, &abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait(full0 + 8 * stage, phase, &abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint64_t adesc = smem_desc_sw128(sA + stage * A_BYTES);
        const uint64_t bdesc = smem_desc_sw128(sB + stage * B_BYTES);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          tc_mma(d_tmem, adesc + (uint64_t)(2 * kk), bdesc + (uint64_t)(2 * kk), IDESC,
                 (kb | kk) != 0 ? 1u : 0u);
        tc_commit(empty0 + 8 * stage);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      tc_commit(tfull0 + 8 * acc);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    // All MMAs this thread issued are complete once `drain` fires.
    tc_commit(drain);
    mbar_wait(drain, 0, &abort_flag, p.status, false);
  } else if (warp >= 2) {
    // ---------------- epilogue
    const int quad = warp & 3;                  // TMEM lanes this warp may read
    const int lrow = quad * 32 + lane;
    const int c_lo = ((warp - 2) / 4) * (BNO / 2);  // this warp's half of the columns
    const uint32_t stg = sO + (uint32_t)(warp - 2) * kStageOutBytes;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
      const int e = find_entry(sched, t);
      const ProbDev &pr = p.pr[sched.prob[e]];
      const int ntn = (pr.N + BNO - 1) / BNO;
      const int local = t - sched.tile_start[e];
      const int mt = local / ntn, nt = local - mt * ntn;
      const int row = sched.row0[e] + mt * BM + lrow;
      const bool valid = row < sched.row_end[e];
      const int col0 = nt * BNO;
      // Whole 32-row blocks of the group go out as TMA tile stores; a block
      // reaching past the group's last row (whose next rows belong to the
      // next group) keeps per-lane stores of its valid rows.
      const int wrow0 = sched.row0[e] + mt * BM + quad * 32;
      const bool tma_rows = !OUT_F32 && pr.tma_out && wrow0 + 32 <= sched.row_end[e];
      const CUtensorMap *mO = sched.prob[e] ? &tmO1 : &tmO0;
      // Warp-uniform: tcgen05.ld below is .sync.aligned, so either every
      // lane proceeds or every lane leaves.
      const bool ready = mbar_wait(tfull0 + 8 * acc, acc_phase, &abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ready)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * BN);
#pragma unroll 1
      for (int c = c_lo; c < c_lo + BNO / 2; c += 32) {
        float v[32];
        tmem_ld32(taddr + c, v);
        if (ACT == kActSwiglu) {
          float u[32];
          tmem_ld32(taddr + BN / 2 + c, u);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = silu(v[i]) * u[i];
        } else if (ACT == kActGelu) {
#pragma unroll
          for (int i = 0; i < 32; i += 2) gelu_erf_x2(v[i], v[i + 1]);
        }
        if (tma_rows) {
          if (lane == 0) bulk_wait_read_all();  // the tile's previous store has read it
          __syncwarp();
          stage_row32_bf16(pr, row, col0 + c, v, stg, lane);
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(mO, col0 + c, wrow0, stg);
            bulk_commit();
          }
        } else if (valid) {
          store_row32<OUT_F32>(pr, row, col0 + c, v);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (lane == 0) bulk_wait_all();  // every tile store has landed before the CTA exits
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


// Two-SM variant: a cluster of 2 CTAs computes one 256 x (NH*BN) tile with
// tcgen05.mma.cta_group::2. Each CTA loads its own 128 rows of A and its
// own half of the BN rows of B of each of the NH MMAs (for SwiGLU: gate rows
// in rank 0, up rows in rank 1), so each SM moves 2/3 (NH = 1) or 1/2
// (NH = 2) of the operand bytes the 1-SM kernel does per unit of MMA work.
// With NH = 2 the two MMAs of a k-step share the A tile and fill tensor
// memory (one accumulator, so the epilogue does not overlap the next tile's
// MMAs): meant for long K, where a tile's MMAs outlast its epilogue many
// times over. Both CTAs' loads complete on the leader's (rank 0) full
// barrier; the leader's single MMA thread issues the M=256 MMAs and
// releases ring slots and accumulators in both CTAs with one multicast
// commit; both CTAs' epilogue warps read their own TMEM rows and arrive on
// the leader's accumulator-empty barrier.
template <int BN, int ACT, bool OUT_F32, int STAGES, int NH>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                         const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                         const __grid_constant__ CUtensorMap tmO0, const __grid_constant__ CUtensorMap tmO1,
                         const ParamsDev p) {
  static_assert(NH == 1 || (NH == 2 && ACT != kActSwiglu), "two MMAs per k-step only without gating");
  constexpr int BMP = 2 * BM;                              // rows per pair tile
  constexpr int BNO = (ACT == kActSwiglu) ? BN / 2 : BN;   // output columns per MMA
  constexpr int TNO = NH * BNO;                            // output columns per tile
  constexpr uint32_t A_BYTES = BM * BK * 2;                // this CTA's rows of A
  constexpr uint32_t B_BYTES = (BN / 2) * BK * 2;          // this CTA's half of one MMA's B
  constexpr uint32_t STAGE_TX = 2 * (A_BYTES + NH * B_BYTES);  // both CTAs, counted by the leader
  constexpr int NACC = NH == 1 ? 2 : 1;                    // accumulator buffers
  constexpr uint32_t ACC_COLS = NH * BN;
  static_assert(NACC * ACC_COLS <= 512, "accumulators exceed tensor memory");
  constexpr uint32_t TMEM_COLS = (NACC * ACC_COLS <= 256) ? 256 : 512;
  constexpr uint32_t IDESC = idesc_bf16_f32(BMP, BN);

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[2 * STAGES + 5];
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ Sched sched;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = (int)cluster_id_x(), npairs = (int)nclusters_x();
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~(uintptr_t)1023);
  const uint32_t sA = smem_u32(base);
  const uint32_t sB = sA + STAGES * A_BYTES;
  const uint32_t sO = sB + STAGES * NH * B_BYTES;  // the epilogue warps' staging tiles
  const uint32_t full0 = smem_u32(&bars[0]);
  const uint32_t empty0 = smem_u32(&bars[STAGES]);
  const uint32_t tfull0 = smem_u32(&bars[2 * STAGES]);
  const uint32_t tempty0 = smem_u32(&bars[2 * STAGES + 2]);
  const uint32_t drain = smem_u32(&bars[2 * STAGES + 4]);

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull0 + 8 * a, 1);
      mbar_init(tempty0 + 8 * a, 2 * kEpiWarps);  // epilogue warps of both CTAs
    }
    mbar_init(drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  if (warp == 2) {
    int run = 0, ne = 0;
    for (int pi = 0; pi < p.n_probs; ++pi) {
      const ProbDev &pr = p.pr[pi];
      const int ntn = (pr.N + TNO - 1) / TNO;
      for (int g0 = 0; g0 < pr.n_groups; g0 += 32) {
        int g = g0 + lane;
        int lo = 0, hi = 0;
        if (g < pr.n_groups) {
          lo = pr.offsets ? pr.offsets[g] : 0;
          hi = pr.offsets ? pr.offsets[g + 1] : (int)pr.a_rows;
          check_group_rows(lo, hi, pr.a_rows, p.status);
        }
        int tiles = (g < pr.n_groups && hi > lo) ? ((hi - lo + BMP - 1) / BMP) * ntn : 0;
        int inc = warp_inclusive_scan(tiles);
        if (g < pr.n_groups) {
          const int e = ne + lane;
          sched.tile_start[e] = run + inc - tiles;
          sched.prob[e] = pi;
          sched.group[e] = g;
          sched.row0[e] = lo;
          sched.row_end[e] = hi;
        }
        run += __shfl_sync(0xffffffffu, inc, 31);
        ne += min(32, pr.n_groups - g0);
      }
      if (lane == 0) sched.prob_end[pi] = run;
    }
    if (lane == 0) {
      if (p.n_probs < 2) sched.prob_end[1] = run;
      sched.n_entries = ne;
      sched.total_tiles = run;
      sched.tile_start[ne] = run;
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's barriers exist before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  TileSeq seq;  // identical in both CTAs of the pair
  seq.init(sched, (p.pr[0].K + BK - 1) / BK, (p.pr[1].K + BK - 1) / BK, p.n_probs, pair, npairs);
  const uint32_t leader_full0 = mapa_shared(full0, 0);
  const uint32_t leader_tempty0 = mapa_shared(tempty0, 0);

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer (both CTAs)
    int stage = 0;
    uint32_t phase = 0, armed = 0, armed_parity = 0;
    bool ok = true;
    for (int t = seq.next(); ok && t >= 0; t = seq.next()) {
      const int e = find_entry(sched, t);
      const int pi = sched.prob[e];
      const ProbDev &pr = p.pr[pi];
      const int ntn = (pr.N + TNO - 1) / TNO;
      const int local = t - sched.tile_start[e];
      const int mt = local / ntn, nt = local - mt * ntn;
      const int a_row = sched.row0[e] + mt * BMP + (int)rank * BM;
      const int b_row = sched.group[e] * pr.b_rows_per_group + nt * TNO +
                        (int)rank * ((ACT == kActSwiglu) ? pr.N : BN / 2);
      const CUtensorMap *mA = pi ? &tmA1 : &tmA0;
      const CUtensorMap *mB = pi ? &tmB1 : &tmB0;
      const int nkb = (pr.K + BK - 1) / BK;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait_cluster(empty0 + 8 * stage, phase ^ 1u, &abort_flag, p.status)) { ok = false; break; }
        if (leader) mbar_arrive_expect_tx(full0 + 8 * stage, STAGE_TX);
        const uint32_t fb = leader_full0 + 8 * stage;
        tma_load_2d_pair(sA + stage * A_BYTES, mA, kb * BK, a_row, fb);
#pragma unroll
        for (int h = 0; h < NH; ++h)
          tma_load_2d_pair(sB + (stage * NH + h) * B_BYTES, mB, kb * BK, b_row + h * BN, fb);
        armed |= 1u << stage;
        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    if (leader)  // the leader's full barriers count both CTAs' copies
      for (int s = 0; s < STAGES; ++s)
        if (armed & (1u << s))
          mbar_wait_cluster(full0 + 8 * s, (armed_parity >> s) & 1u, &abort_flag, p.status, false);
  } else if (warp == 1 && lane == 0) {
    if (leader) {
      // ---------------- MMA issuer (leader only)
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int t = seq.next(); ok && t >= 0; t = seq.next()) {
        const int e = find_entry(sched, t);
        const int nkb = (p.pr[sched.prob[e]].K + BK - 1) / BK;
        if (!mbar_wait_cluster(tempty0 + 8 * acc, acc_phase ^ 1u, &abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * ACC_COLS);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_cluster(full0 + 8 * stage, phase, &abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = smem_desc_sw128(sA + stage * A_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
#pragma unroll
            for (int h = 0; h < NH; ++h)
              tc_mma_pair(d_tmem + (uint32_t)(h * BN), adesc + (uint64_t)(2 * kk),
                          smem_desc_sw128(sB + (stage * NH + h) * B_BYTES) + (uint64_t)(2 * kk), IDESC,
                          (kb | kk) != 0 ? 1u : 0u);
          tc_commit_pair(empty0 + 8 * stage, 0x3);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair(tfull0 + 8 * acc, 0x3);
        if (++acc == NACC) { acc = 0; acc_phase ^= 1u; }
      }
      tc_commit_pair(drain, 0x3);
    }
    // Both CTAs: every MMA that reads this CTA's shared memory or writes its
    // TMEM has completed once the leader's last commit lands here.
    mbar_wait_cluster(drain, 0, &abort_flag, p.status, false);
  } else if (warp >= 2) {
    // ---------------- epilogue (both CTAs, own TMEM rows)
    const int quad = warp & 3;                  // TMEM lanes this warp may read
    const int lrow = quad * 32 + lane;
    const int c_lo = ((warp - 2) / 4) * (TNO / 2);  // this warp's half of the columns
    const uint32_t stg = sO + (uint32_t)(warp - 2) * kStageOutBytes;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = seq.next(); t >= 0; t = seq.next()) {
      const int e = find_entry(sched, t);
      const ProbDev &pr = p.pr[sched.prob[e]];
      const int ntn = (pr.N + TNO - 1) / TNO;
      const int local = t - sched.tile_start[e];
      const int mt = local / ntn, nt = local - mt * ntn;
      const int row = sched.row0[e] + mt * BMP + (int)rank * BM + lrow;
      const bool valid = row < sched.row_end[e];
      const int col0 = nt * TNO;
      // Whole 32-row blocks go out as TMA tile stores, a block reaching past
      // the group's last row as per-lane stores of its valid rows.
      const int wrow0 = sched.row0[e] + mt * BMP + (int)rank * BM + quad * 32;
      const bool tma_rows = !OUT_F32 && pr.tma_out && wrow0 + 32 <= sched.row_end[e];
      const CUtensorMap *mO = sched.prob[e] ? &tmO1 : &tmO0;
      const bool ready = mbar_wait_cluster(tfull0 + 8 * acc, acc_phase, &abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ready)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * ACC_COLS);
#pragma unroll 1
      for (int c = c_lo; c < c_lo + TNO / 2; c += 32) {
        float v[32];
        tmem_ld32(taddr + c, v);
        if (ACT == kActSwiglu) {
          float u[32];
          tmem_ld32(taddr + BN / 2 + c, u);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = silu(v[i]) * u[i];
        } else if (ACT == kActGelu) {
#pragma unroll
          for (int i = 0; i < 32; i += 2) gelu_erf_x2(v[i], v[i + 1]);
        }
        if (tma_rows) {
          if (lane == 0) bulk_wait_read_all();  // the tile's previous store has read it
          __syncwarp();
          stage_row32_bf16(pr, row, col0 + c, v, stg, lane);
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(mO, col0 + c, wrow0, stg);
            bulk_commit();
          }
        } else if (valid) {
          store_row32<OUT_F32>(pr, row, col0 + c, v);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_tempty0 + 8 * acc);
      if (++acc == NACC) { acc = 0; acc_phase ^= 1u; }
    }
    if (lane == 0) bulk_wait_all();  // every tile store has landed before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA leaves while its peer may still signal it
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TMEM_COLS)
                 : "memory");
  }
}

// ------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once (a function-local static
// is initialised once, safely under concurrent first calls); null if the
// driver does not provide it.
EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(ptr);
    return static_cast<EncodeTiledFn>(nullptr);
  }();
  return fn;
}

// 2D bf16 tensor [rows, cols] (cols contiguous), box {64, box_rows}, 128B swizzle.
bool make_map(CUtensorMap *m, const void *ptr, int64_t rows, int64_t cols, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// bf16 output [rows, N] with row stride ld_out, box of 32 x 32 staged with the
// 64-byte swizzle. False when the output cannot take TMA stores (a base off
// 16 bytes or a row stride that is not a multiple of 16 bytes).
bool make_out_map(CUtensorMap *m, const GemmProblem &q) {
  if ((reinterpret_cast<uintptr_t>(q.out) & 15u) != 0 || (q.ld_out * 2) % 16 != 0 || q.a_rows <= 0)
    return false;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)q.N, (cuuint64_t)q.a_rows};
  cuuint64_t strides[1] = {(cuuint64_t)q.ld_out * 2};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q.out, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool vec32_ok(const GemmProblem &q, int elem) {
  return (reinterpret_cast<uintptr_t>(q.out) & 31u) == 0 && (q.ld_out * elem) % 32 == 0;
}

template <int BN, int ACT, bool OUT_F32>
int run_tc(const GemmProblem *probs, int n_probs, int32_t *status, cudaStream_t stream) {
  constexpr uint32_t STAGE_BYTES = (BM + BN) * BK * 2;
  constexpr int STAGES = (200 * 1024) / STAGE_BYTES > 8 ? 8 : (200 * 1024) / STAGE_BYTES;
  constexpr int BNO = (ACT == kActSwiglu) ? BN / 2 : BN;
  const size_t smem = 1024 + (size_t)STAGES * STAGE_BYTES + (OUT_F32 ? 0 : kEpiWarps * kStageOutBytes);

  CUtensorMap maps[4], omaps[2];
  memset(maps, 0, sizeof(maps));
  memset(omaps, 0, sizeof(omaps));
  ParamsDev pd;
  memset(&pd, 0, sizeof(pd));
  pd.n_probs = n_probs;
  pd.status = status;
  int64_t max_tiles = 0;
  for (int i = 0; i < n_probs; ++i) {
    const GemmProblem &q = probs[i];
    if (!make_map(&maps[2 * i], q.A, q.a_rows, q.K, BM)) return MOE_ERR_CUDA;
    if (!make_map(&maps[2 * i + 1], q.B, (int64_t)q.n_groups * q.b_rows_per_group, q.K, BN / 2))
      return MOE_ERR_CUDA;
    pd.pr[i].offsets = q.offsets;
    pd.pr[i].n_groups = q.n_groups;
    pd.pr[i].a_rows = q.a_rows;
    pd.pr[i].b_rows_per_group = q.b_rows_per_group;
    pd.pr[i].N = q.N;
    pd.pr[i].K = q.K;
    pd.pr[i].out = q.out;
    pd.pr[i].ld_out = q.ld_out;
    pd.pr[i].vec32 = vec32_ok(q, OUT_F32 ? 4 : 2);
    pd.pr[i].residual = static_cast<const __nv_bfloat16 *>(q.residual);
    pd.pr[i].ld_res = q.ld_res;
    pd.pr[i].tma_out = !OUT_F32 && make_out_map(&omaps[i], q);
    max_tiles += max_m_tiles(q, BM) * ((q.N + BNO - 1) / BNO);
  }
  if (n_probs == 1) { maps[2] = maps[0]; maps[3] = maps[1]; omaps[1] = omaps[0]; }
  if (max_tiles == 0) return MOE_OK;
  auto kern = grouped_gemm_tc_kernel<BN, ACT, OUT_F32, STAGES>;
  MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  int grid = num_sms();
  if (max_tiles < grid) grid = (int)max_tiles;
  kern<<<grid, kThreads, smem, stream>>>(maps[0], maps[1], maps[2], maps[3], omaps[0], omaps[1], pd);
  return last_launch_status();
}

template <int BN, int ACT, bool OUT_F32, int NH = 1>
int run_tc_pair(const GemmProblem *probs, int n_probs, int32_t *status, cudaStream_t stream) {
  constexpr uint32_t STAGE_BYTES = (BM + NH * BN / 2) * BK * 2;  // per CTA
  constexpr int S0 = (200 * 1024) / STAGE_BYTES;
  constexpr int STAGES = S0 > 8 ? 8 : S0;
  constexpr int BNO = NH * ((ACT == kActSwiglu) ? BN / 2 : BN);  // output columns per tile
  // Staging tiles for the TMA-stored output: bf16, narrow form only.
  constexpr bool kTmaOut = !OUT_F32 && NH == 1;
  const size_t smem = 1024 + (size_t)STAGES * STAGE_BYTES + (kTmaOut ? kEpiWarps * kStageOutBytes : 0);

  CUtensorMap maps[4], omaps[2];
  memset(maps, 0, sizeof(maps));
  memset(omaps, 0, sizeof(omaps));
  ParamsDev pd;
  memset(&pd, 0, sizeof(pd));
  pd.n_probs = n_probs;
  pd.status = status;
  int64_t max_tiles = 0;
  for (int i = 0; i < n_probs; ++i) {
    const GemmProblem &q = probs[i];
    if (!make_map(&maps[2 * i], q.A, q.a_rows, q.K, BM)) return MOE_ERR_CUDA;
    if (!make_map(&maps[2 * i + 1], q.B, (int64_t)q.n_groups * q.b_rows_per_group, q.K, BN / 2))
      return MOE_ERR_CUDA;
    pd.pr[i].offsets = q.offsets;
    pd.pr[i].n_groups = q.n_groups;
    pd.pr[i].a_rows = q.a_rows;
    pd.pr[i].b_rows_per_group = q.b_rows_per_group;
    pd.pr[i].N = q.N;
    pd.pr[i].K = q.K;
    pd.pr[i].out = q.out;
    pd.pr[i].ld_out = q.ld_out;
    pd.pr[i].vec32 = vec32_ok(q, OUT_F32 ? 4 : 2);
    pd.pr[i].residual = static_cast<const __nv_bfloat16 *>(q.residual);
    pd.pr[i].ld_res = q.ld_res;
    // TMA-stored tiles on the narrow form only: the wide form's single
    // accumulator keeps its epilogue on the critical path, where waiting for
    // a staging tile to be read measured no better than per-lane stores.
    pd.pr[i].tma_out = kTmaOut && make_out_map(&omaps[i], q);
    max_tiles += max_m_tiles(q, 2 * BM) * ((q.N + BNO - 1) / BNO);
  }
  if (n_probs == 1) { maps[2] = maps[0]; maps[3] = maps[1]; omaps[1] = omaps[0]; }
  if (max_tiles == 0) return MOE_OK;
  auto kern = grouped_gemm_pair_kernel<BN, ACT, OUT_F32, STAGES, NH>;
  MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.gridDim = dim3(2 * (unsigned)(num_sms() / 2));
  // Co-resident CTA pairs of this kernel, asked once per instantiation (a
  // function-local static is initialised once, safely under concurrent
  // first calls).
  static const int max_clusters = [&] {
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) n = 0;
    return n;
  }();
  int clusters = max_clusters;
  if (clusters < 1) return MOE_ERR_UNSUPPORTED;
  if (max_tiles < clusters) clusters = (int)max_tiles;
  cfg.gridDim = dim3(2 * (unsigned)clusters);
  MOE_CUDA_TRY(cudaLaunchKernelEx(&cfg, kern, maps[0], maps[1], maps[2], maps[3], omaps[0], omaps[1], pd));
  return last_launch_status();
}

}  // namespace

bool make_tma_2d_bf16(CUtensorMap *map, const void *ptr, int64_t rows, int64_t cols, int box_rows) {
  return make_map(map, ptr, rows, cols, box_rows);
}

// Largest tile width whose output columns divide every problem's N.
static int pick_bn(const GemmProblem *probs, int n_probs, int act) {
  const int cands[3] = {256, 192, 128};
  for (int c : cands) {
    int bno = act == kActSwiglu ? c / 2 : c;
    if (act == kActSwiglu && c == 192) continue;
    bool ok = true;
    for (int i = 0; i < n_probs; ++i) ok = ok && probs[i].N % bno == 0;
    if (ok) return c;
  }
  return 128;
}

// The pair (2-SM) kernel pays off with full 256-wide tiles and groups large
// enough to fill 256-row tiles; measured on B200 it is slower with N=192
// tiles. With short K (~1152) it beat the single-SM kernel on DiT-MoE-XL's
// up projection (16384 assignments over 8 experts: layer 0.584 -> 0.571 ms)
// but lost on MMOE's (16384 over 16 heavy experts, ~860 rows each once the
// zero-computation experts take theirs: 0.431 -> 0.435 ms), whose 256-row
// tiles leave twice the ragged rows of 128-row ones. So short K takes the
// pair only when every problem has at least 1536 rows (assignments, an
// upper bound on the host) per group on average.
static bool use_pair(const GemmProblem *probs, int n_probs, int bn) {
  if (bn != 256) return false;
  int64_t rows = 0, groups = 0;
  for (int i = 0; i < n_probs; ++i) {
    const int64_t g = probs[i].offsets ? probs[i].n_groups : 1;
    if (probs[i].K < 2048 && probs[i].a_rows < 1536 * g) return false;
    rows += probs[i].a_rows;
    groups += g;
  }
  return groups > 0 && rows >= 256 * groups;
}

// Longest-first list-scheduling makespan, in K blocks, of the tiles of (at
// most two) problems on `workers` CTAs (or CTA pairs): the longer problem's
// tiles first, then each of the other's to the worker free first -- the
// order the kernels deal them in.
static int64_t lpt_makespan(const int64_t *tiles, const int64_t *kb, int n, int workers) {
  int64_t nA = tiles[0], a = kb[0], nB = n > 1 ? tiles[1] : 0, b = n > 1 ? kb[1] : 0;
  if (nB > 0 && b > a) { std::swap(nA, nB); std::swap(a, b); }
  // With many tiles per worker the last wave is a small part of the whole:
  // the mean load plus one long tile bounds the makespan without simulating
  // every tile (this runs on the host at every launch).
  if (nA + nB > 32 * (int64_t)workers)
    return (nA * a + nB * b + workers - 1) / workers + a;
  std::priority_queue<int64_t, std::vector<int64_t>, std::greater<int64_t>> load;
  const int64_t q = nA / workers, r = nA % workers;
  for (int w = 0; w < workers; ++w) load.push((q + (w < r ? 1 : 0)) * a);
  for (int64_t i = 0; i < nB; ++i) {
    const int64_t l = load.top();
    load.pop();
    load.push(l + b);
  }
  int64_t mx = 0;
  while (!load.empty()) { mx = std::max(mx, load.top()); load.pop(); }
  return mx;
}

// Estimated tiles of height bm and width tn for a problem: its rows' tiles
// plus, for grouped rows (group sizes are known only on the device), half a
// ragged tile per group.
static int64_t est_tiles(const GemmProblem &q, int bm, int tn) {
  const int64_t m = (q.a_rows + bm - 1) / bm + (q.offsets ? q.n_groups / 2 : 0);
  return m * ((q.N + tn - 1) / tn);
}

// Two MMAs per k-step on a CTA pair (256 x 512 or 256 x 384 tiles) for
// ungated GEMMs with long K (the down projections): the MMA width per output
// tile, or 0 to keep the narrow tiles (`bn` wide on one SM, or on a pair when
// `pair`). Measured on B200, the wide tiles run about 1.25x the MMA work per
// unit time of the one-SM kernel and about 1.1x that of the narrow pair
// tiles, but their coarser grain costs more in ragged group ends and in the
// last wave; they are used when the estimated makespans say so.
static int pick_wide(const GemmProblem *probs, int n_probs, int act, int bn, bool pair) {
  if (act != kActNone) return 0;
  int64_t rows = 0, groups = 0;
  bool w256 = true, w192 = true;
  for (int i = 0; i < n_probs; ++i) {
    if (probs[i].K < 2048) return 0;
    w256 = w256 && probs[i].N % 512 == 0;
    w192 = w192 && probs[i].N % 384 == 0;
    rows += probs[i].a_rows;
    groups += probs[i].offsets ? probs[i].n_groups : 1;
  }
  if (groups == 0 || rows < 256 * groups) return 0;
  const int wbn = w256 ? 256 : w192 ? 192 : 0;
  if (wbn == 0) return 0;
  int64_t tn[2], tw[2], kb[2];
  for (int i = 0; i < n_probs; ++i) {
    kb[i] = (probs[i].K + BK - 1) / BK;
    tn[i] = est_tiles(probs[i], pair ? 2 * BM : BM, bn);
    tw[i] = est_tiles(probs[i], 2 * BM, 2 * wbn);
  }
  const int sms = num_sms();
  // Time per worker in units of one SM's MMA clocks per K block of a
  // 128 x 1 tile slice: a narrow tile gives each of its SMs 128 x bn, a
  // wide one 128 x 2*wbn.
  const double t_narrow = (double)lpt_makespan(tn, kb, n_probs, pair ? sms / 2 : sms) * bn;
  const double t_wide = (double)lpt_makespan(tw, kb, n_probs, sms / 2) * 2 * wbn;
  const double gain = pair ? 1.10 : 1.25;
  return t_wide < t_narrow * gain ? wbn : 0;
}

int launch_grouped_gemm_bf16(const GemmProblem *probs, int n_probs, int act, bool out_f32,
                             int32_t *dev_status, cudaStream_t stream, const GemmProblem *also) {
  if (n_probs < 1 || n_probs > 2) return MOE_ERR_INVALID_ARG;
  if (out_f32) return MOE_ERR_UNSUPPORTED;  // bf16 layers keep every GEMM output in bf16
  GemmProblem rule[3];
  int n_rule = 0;
  for (int i = 0; i < n_probs; ++i) rule[n_rule++] = probs[i];
  if (also) rule[n_rule++] = *also;
  const int bn = pick_bn(rule, n_rule, act);
  const bool pair = use_pair(rule, n_rule, bn);
  const int wide = pick_wide(probs, n_probs, act, bn, pair);
  if (wide == 256) return run_tc_pair<256, kActNone, false, 2>(probs, n_probs, dev_status, stream);
  if (wide == 192) return run_tc_pair<192, kActNone, false, 2>(probs, n_probs, dev_status, stream);
#define MOE_RUN(BN_, ACT_) \
  return pair ? run_tc_pair<BN_, ACT_, false>(probs, n_probs, dev_status, stream) \
              : run_tc<BN_, ACT_, false>(probs, n_probs, dev_status, stream)
  if (act == kActGelu) {
    if (bn == 256) MOE_RUN(256, kActGelu);
    if (bn == 192) MOE_RUN(192, kActGelu);
    MOE_RUN(128, kActGelu);
  }
  if (act == kActSwiglu) {
    if (bn == 256) MOE_RUN(256, kActSwiglu);
    MOE_RUN(128, kActSwiglu);
  }
  if (act == kActNone) {
    if (bn == 256) MOE_RUN(256, kActNone);
    if (bn == 192) MOE_RUN(192, kActNone);
    MOE_RUN(128, kActNone);
  }
#undef MOE_RUN
  return MOE_ERR_UNSUPPORTED;
}

}  // namespace moe
