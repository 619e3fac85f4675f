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
//   warps 2..5   epilogue: tcgen05.ld of the accumulator (one TMEM lane
//                quadrant per warp), activation, rounding, global store;
//                overlaps the next tile's MMAs
// SwiGLU: the B tile holds BN/2 gate rows and the matching BN/2 up rows, so
// one accumulator carries both halves and the epilogue forms
// silu(gate) * up without another pass.
// Every mbarrier wait is bounded: on expiry the kernel flags
// MOE_DEV_TIMEOUT, lets its in-flight copies and MMAs finish (again with a
// bound), frees its tensor memory and returns.
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;  // 64 bf16 = 128 bytes = one swizzle atom row
constexpr int kThreads = 192;
constexpr int kMaxEntries = 2 * MOE_MAX_EXPERTS + 2;
constexpr uint64_t kTimeoutNs = 2000000000ull;  // 2 s per wait

struct ProbDev {
  const int32_t *offsets;
  int n_groups;
  int64_t a_rows;
  int b_rows_per_group;
  int N, K;
  void *out;
  int64_t ld_out;
};
struct ParamsDev {
  int n_probs;
  ProbDev pr[2];
  int32_t *status;
};

struct Sched {
  int n_entries;
  int total_tiles;
  int tile_start[kMaxEntries + 1];
  int prob[kMaxEntries];
  int group[kMaxEntries];
  int row0[kMaxEntries];
  int row_end[kMaxEntries];
};

// ---------------------------------------------------------------- PTX
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait. Returns false if the kernel is aborting (another role gave
// up) or this wait expired (then it raises the abort itself).
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                       int32_t *status, bool watch_abort = true) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t spin = 1;; ++spin) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((spin & 63u) == 0) {
      if (watch_abort && *abort_flag) return false;
      if (global_timer_ns() - t0 > kTimeoutNs) {
        *abort_flag = 1;
        set_status(status, MOE_DEV_TIMEOUT);
        return false;
      }
    }
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
// D[tmem] (+)= A[smem] . B[smem]^T, M=128, N from the instruction descriptor, K=16.
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle,
// 8-row core groups 1024 bytes apart (SBO), descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);        // start address
  d |= (uint64_t)1u << 16;                        // leading byte offset (unused for SW128 K-major)
  d |= (uint64_t)(1024u >> 4) << 32;              // stride byte offset
  d |= (uint64_t)1u << 46;                        // version (sm_100)
  d |= (uint64_t)2u << 61;                        // layout: SWIZZLE_128B
  return d;
}

// Instruction descriptor: bf16 x bf16 -> fp32, both K-major, M=128, N=n.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int n) {
  return (1u << 4)                       // D format f32
         | (1u << 7)                     // A format bf16
         | (1u << 10)                    // B format bf16
         | ((uint32_t)(n >> 3) << 17)    // N / 8
         | ((uint32_t)(BM >> 4) << 24);  // M / 16
}

__device__ __forceinline__ int find_entry(const Sched &s, int t) {
  int lo = 0, hi = s.n_entries - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (s.tile_start[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int BN, int ACT, bool OUT_F32, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                       const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                       const ParamsDev p) {
  constexpr int BNO = (ACT == kActSwiglu) ? BN / 2 : BN;  // output columns per tile
  constexpr uint32_t A_BYTES = BM * BK * 2;
  constexpr uint32_t B_BYTES = BN * BK * 2;
  constexpr uint32_t STAGE_TX = A_BYTES + B_BYTES;
  constexpr uint32_t TMEM_COLS = (2 * BN <= 256) ? 256 : 512;
  constexpr uint32_t IDESC = idesc_bf16_f32(BN);

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
      mbar_init(tempty0 + 8 * a, 4);
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
    }
    if (lane == 0) {
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
    const int quad = warp & 3;
    const int lrow = quad * 32 + lane;
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
      // Warp-uniform: tcgen05.ld below is .sync.aligned, so either every
      // lane proceeds or every lane leaves.
      const bool ready = mbar_wait(tfull0 + 8 * acc, acc_phase, &abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ready)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * BN);
#pragma unroll 1
      for (int c = 0; c < BNO; c += 32) {
        float v[32];
        tmem_ld32(taddr + c, v);
        if (ACT == kActSwiglu) {
          float u[32];
          tmem_ld32(taddr + BN / 2 + c, u);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = silu(v[i]) * u[i];
        } else if (ACT == kActGelu) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = gelu_erf(v[i]);
        }
        if (valid) {
          const int col = col0 + c;
          if (OUT_F32) {
            float *o = static_cast<float *>(pr.out) + (int64_t)row * pr.ld_out + col;
            if (col + 32 <= pr.N) {
#pragma unroll
              for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4 *>(o + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
            } else {
              for (int i = 0; i < 32 && col + i < pr.N; ++i) o[i] = v[i];
            }
          } else {
            __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(pr.out) + (int64_t)row * pr.ld_out + col;
            if (col + 32 <= pr.N) {
#pragma unroll
              for (int i = 0; i < 32; i += 8) {
                uint4 u4;
                __nv_bfloat162 *h2 = reinterpret_cast<__nv_bfloat162 *>(&u4);
#pragma unroll
                for (int j = 0; j < 4; ++j) h2[j] = __floats2bfloat162_rn(v[i + 2 * j], v[i + 2 * j + 1]);
                *reinterpret_cast<uint4 *>(o + i) = u4;
              }
            } else {
              for (int i = 0; i < 32 && col + i < pr.N; ++i) o[i] = __float2bfloat16_rn(v[i]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
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

// ------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
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

template <int BN, int ACT, bool OUT_F32>
int run_tc(const GemmProblem *probs, int n_probs, int32_t *status, cudaStream_t stream) {
  constexpr uint32_t STAGE_BYTES = (BM + BN) * BK * 2;
  constexpr int STAGES = (200 * 1024) / STAGE_BYTES > 8 ? 8 : (200 * 1024) / STAGE_BYTES;
  constexpr int BNO = (ACT == kActSwiglu) ? BN / 2 : BN;
  const size_t smem = 1024 + (size_t)STAGES * STAGE_BYTES;

  CUtensorMap maps[4];
  memset(maps, 0, sizeof(maps));
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
    max_tiles += max_m_tiles(q, BM) * ((q.N + BNO - 1) / BNO);
  }
  if (n_probs == 1) { maps[2] = maps[0]; maps[3] = maps[1]; }
  if (max_tiles == 0) return MOE_OK;
  auto kern = grouped_gemm_tc_kernel<BN, ACT, OUT_F32, STAGES>;
  MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  int grid = num_sms();
  if (max_tiles < grid) grid = (int)max_tiles;
  kern<<<grid, kThreads, smem, stream>>>(maps[0], maps[1], maps[2], maps[3], pd);
  return last_launch_status();
}

}  // namespace

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

int launch_grouped_gemm_bf16(const GemmProblem *probs, int n_probs, int act, bool out_f32,
                             int32_t *dev_status, cudaStream_t stream) {
  if (n_probs < 1 || n_probs > 2) return MOE_ERR_INVALID_ARG;
  const int bn = pick_bn(probs, n_probs, act);
  if (!out_f32) {
    if (act == kActGelu) {
      if (bn == 256) return run_tc<256, kActGelu, false>(probs, n_probs, dev_status, stream);
      if (bn == 192) return run_tc<192, kActGelu, false>(probs, n_probs, dev_status, stream);
      return run_tc<128, kActGelu, false>(probs, n_probs, dev_status, stream);
    }
    if (act == kActSwiglu) {
      if (bn == 256) return run_tc<256, kActSwiglu, false>(probs, n_probs, dev_status, stream);
      return run_tc<128, kActSwiglu, false>(probs, n_probs, dev_status, stream);
    }
    return MOE_ERR_UNSUPPORTED;
  }
  if (act != kActNone) return MOE_ERR_UNSUPPORTED;
  if (bn == 256) return run_tc<256, kActNone, true>(probs, n_probs, dev_status, stream);
  if (bn == 192) return run_tc<192, kActNone, true>(probs, n_probs, dev_status, stream);
  return run_tc<128, kActNone, true>(probs, n_probs, dev_status, stream);
}

}  // namespace moe
