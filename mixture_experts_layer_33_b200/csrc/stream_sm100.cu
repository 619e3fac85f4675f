// Weight-streaming expert MLP for small blocks of tokens (<= 128).
//
// Dynamic Expert Sharing: Decoupling Memory from Parallelism in
// Mixture-of-Experts Diffusion LLMs, section 2.1: one expert serving c
// tokens costs f(c) = a*c + b, where b, the fetch of the expert's weights
// from HBM, dominates; a block's MoE latency is governed by b times the
// number of distinct experts it touches. So this kernel's job is to read
// every used expert's weights from HBM exactly once, back to back, at full
// bandwidth.
//
// Swap-AB on tcgen05: the weights are the M operand (128 rows of an
// expert's weight matrix per unit), the expert's tokens the N operand
// (NB = 32/64/128 columns, padded), so D^T = W . X^T lands in TMEM with one
// output feature per lane. One persistent, co-resident CTA per SM walks a
// single list of units: first every (expert, 128 hidden units) block of the
// up projection, then every (expert, 128 output features) block of the down
// projection, so the weight stream never pauses between the two. A down
// unit of expert e waits (bounded) on a per-expert counter that the up
// units of e release once their hidden activations are stored.
//   warp 0      TMA producer: a ring of 40 KB stages [A0 | A1 | B0 | B1]
//               (two 128x64 weight tiles, two NBx64 token tiles)
//   warp 1      one thread issues tcgen05.mma, 8 per stage
//   warps 2..5  epilogue, one TMEM lane quadrant each (outputs in bf16)
// Stage use: SwiGLU up: A0 = gate rows, A1 = up rows, both against B0, into
// two accumulators, so the same thread forms silu(gate) * up. GELU up and
// down: A0/B0 and A1/B1 are two consecutive 64-wide k-blocks of one
// product (split along K inside the stage).
// Every wait is bounded (MOE_DEV_TIMEOUT) as in the grouped GEMM.
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace moe {
namespace {

using namespace tc;

constexpr int BMW = 128;  // weight rows per unit (MMA M)
constexpr int BK = 64;
constexpr int kThreads = 192;
constexpr int kMaxEntries = 2 * MOE_MAX_EXPERTS + 1;

struct PassDev {
  int w_rows_per_group;  // weight rows per group (2N for SwiGLU: gate rows then up rows)
  int N, K;              // output features per token, reduction length
  void *out;
  int64_t ld_out;
};
struct StreamParams {
  const int32_t *offsets;  // [n_groups + 1] token-row offsets, or NULL: one group of t_rows
  int n_groups;
  int t_rows;
  PassDev up, down;
  int32_t *done;           // [n_groups] epilogue-warp arrivals of finished up units (zeroed before launch)
  int32_t *status;
};

struct Units {
  int n_entries;
  int total;
  int start[kMaxEntries + 1];
  int group[kMaxEntries];  // >= 0: up units of group; < 0: down units of group ~g
  int row0[kMaxEntries];
  int cnt[kMaxEntries];
};

__device__ __forceinline__ int find_unit_entry(const Units &u, int t) {
  int lo = 0, hi = u.n_entries - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (u.start[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ int ld_acquire(const int32_t *p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bounded wait until *p >= target (written by other CTAs of this grid).
__device__ __noinline__ bool wait_counter(const int32_t *p, int target, volatile int *abort_flag,
                                          int32_t *status) {
  if (ld_acquire(p) >= target) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t spin = 1;; ++spin) {
    if (ld_acquire(p) >= target) return true;
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

template <int NB, int ACT>
__global__ void __launch_bounds__(kThreads, 1)
expert_stream_kernel(const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmX,
                     const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ CUtensorMap tmH,
                     const StreamParams p) {
  constexpr bool GATED = ACT == kActSwiglu;
  constexpr uint32_t A_BYTES = BMW * BK * 2;  // 16 KB
  constexpr uint32_t B_BYTES = NB * BK * 2;
  constexpr uint32_t STAGE_BYTES = 2 * A_BYTES + 2 * B_BYTES;
  constexpr int STAGES0 = (200 * 1024) / STAGE_BYTES;
  constexpr int STAGES = STAGES0 > 8 ? 8 : STAGES0;
  constexpr int ACC_COLS = 2 * NB;  // accumulator set: D0 and (gated up) D1
  constexpr uint32_t TMEM_COLS = 2 * ACC_COLS <= 32 ? 32 : 2 * ACC_COLS <= 64 ? 64
                                 : 2 * ACC_COLS <= 128 ? 128 : 2 * ACC_COLS <= 256 ? 256 : 512;
  constexpr uint32_t IDESC = idesc_bf16_f32(BMW, NB);

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[2 * STAGES + 5];
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ Units units;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~(uintptr_t)1023);
  const uint32_t s0 = smem_u32(base);
  const uint32_t full0 = smem_u32(&bars[0]);
  const uint32_t empty0 = smem_u32(&bars[STAGES]);
  const uint32_t tfull0 = smem_u32(&bars[2 * STAGES]);
  const uint32_t tempty0 = smem_u32(&bars[2 * STAGES + 2]);
  const uint32_t drain = smem_u32(&bars[2 * STAGES + 4]);
  const int up_blocks = (p.up.N + BMW - 1) / BMW;
  const int down_blocks = (p.down.N + BMW - 1) / BMW;

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
    // Entries 0..G-1: up units of group g; entries G..2G-1: its down units.
    int run = 0;
    for (int pass = 0; pass < 2; ++pass) {
      const int blocks = pass == 0 ? up_blocks : down_blocks;
      for (int g0 = 0; g0 < p.n_groups; g0 += 32) {
        const int g = g0 + lane;
        int lo = 0, hi = 0;
        if (g < p.n_groups) {
          lo = p.offsets ? p.offsets[g] : 0;
          hi = p.offsets ? p.offsets[g + 1] : p.t_rows;
          check_group_rows(lo, hi, p.t_rows, p.status, NB);  // a group spans <= NB token columns
        }
        const int n = (g < p.n_groups && hi > lo) ? blocks : 0;
        const int inc = warp_inclusive_scan(n);
        if (g < p.n_groups) {
          const int e = pass * p.n_groups + g;
          units.start[e] = run + inc - n;
          units.group[e] = pass == 0 ? g : ~g;
          units.row0[e] = lo;
          units.cnt[e] = hi - lo;
        }
        run += __shfl_sync(0xffffffffu, inc, 31);
      }
    }
    if (lane == 0) {
      units.n_entries = 2 * p.n_groups;
      units.total = run;
      units.start[2 * p.n_groups] = run;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  const int total = units.total;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmW1)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmW2)) : "memory");
    int stage = 0;
    uint32_t phase = 0, armed = 0, armed_parity = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
      const int e = find_unit_entry(units, t);
      const int gcode = units.group[e];
      const bool up = gcode >= 0;
      const int g = up ? gcode : ~gcode;
      const int blk = t - units.start[e];
      const int x_row = units.row0[e];
      const PassDev &pd = up ? p.up : p.down;
      const CUtensorMap *mW = up ? &tmW1 : &tmW2;
      const CUtensorMap *mB = up ? &tmX : &tmH;
      const int w_row = g * pd.w_rows_per_group + blk * BMW;
      const int nkb = (pd.K + BK - 1) / BK;
      const bool paired = up && GATED;
      const int nst = paired ? nkb : (nkb + 1) / 2;
      if (!up) {
        // The hidden activations of group g come from other CTAs' up units.
        if (!wait_counter(p.done + g, 4 * up_blocks, &abort_flag, p.status)) { ok = false; break; }
        asm volatile("fence.proxy.async.global;" ::: "memory");
      }
      for (int st = 0; st < nst; ++st) {
        if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, &abort_flag, p.status)) { ok = false; break; }
        const uint32_t fb = full0 + 8 * stage;
        const uint32_t a0 = s0 + stage * STAGE_BYTES;
        const uint32_t a1 = a0 + A_BYTES, b0 = a0 + 2 * A_BYTES, b1 = b0 + B_BYTES;
        if (paired) {
          mbar_arrive_expect_tx(fb, 2 * A_BYTES + B_BYTES);
          tma_load_2d(a0, mW, st * BK, w_row, fb);
          tma_load_2d(a1, mW, st * BK, w_row + pd.N, fb);
          tma_load_2d(b0, mB, st * BK, x_row, fb);
        } else {
          const bool two = 2 * st + 1 < nkb;
          mbar_arrive_expect_tx(fb, (two ? 2u : 1u) * (A_BYTES + B_BYTES));
          tma_load_2d(a0, mW, 2 * st * BK, w_row, fb);
          tma_load_2d(b0, mB, 2 * st * BK, x_row, fb);
          if (two) {
            tma_load_2d(a1, mW, (2 * st + 1) * BK, w_row, fb);
            tma_load_2d(b1, mB, (2 * st + 1) * BK, x_row, fb);
          }
        }
        armed |= 1u << stage;
        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    for (int s = 0; s < STAGES; ++s)
      if (armed & (1u << s))
        mbar_wait(full0 + 8 * s, (armed_parity >> s) & 1u, &abort_flag, p.status, false);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    int stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
      const int e = find_unit_entry(units, t);
      const bool up = units.group[e] >= 0;
      const int K = up ? p.up.K : p.down.K;
      const int nkb = (K + BK - 1) / BK;
      const bool paired = up && GATED;
      const int nst = paired ? nkb : (nkb + 1) / 2;
      if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1u, &abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t d0 = tmem_base + (uint32_t)(acc * ACC_COLS);
      for (int st = 0; st < nst; ++st) {
        if (!mbar_wait(full0 + 8 * stage, phase, &abort_flag, p.status)) { ok = false; break; }
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
    mbar_wait(drain, 0, &abort_flag, p.status, false);
  } else if (warp >= 2) {
    // ---------------- epilogue: lane j of quadrant q holds feature blk*128 + 32q + j
    const int quad = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const int e = find_unit_entry(units, t);
      const int gcode = units.group[e];
      const bool up = gcode >= 0;
      const int g = up ? gcode : ~gcode;
      const int blk = t - units.start[e];
      const PassDev &pd = up ? p.up : p.down;
      const int feat = blk * BMW + quad * 32 + lane;
      const bool valid = feat < pd.N;
      const int row0 = units.row0[e];
      const int cnt = units.cnt[e];
      const bool ready = mbar_wait(tfull0 + 8 * acc, acc_phase, &abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ready)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * ACC_COLS);
#pragma unroll 1
      for (int c = 0; c < NB; c += 32) {
        float v[32];
        tmem_ld32(taddr + c, v);
        if (up && GATED) {
          float u[32];
          tmem_ld32(taddr + NB + c, u);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = silu(v[i]) * u[i];
        } else if (up) {
#pragma unroll
          for (int i = 0; i < 32; i += 2) gelu_erf_x2(v[i], v[i + 1]);
        }
        if (valid) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (c + i < cnt) {
              const int64_t o = (int64_t)(row0 + c + i) * pd.ld_out + feat;
              static_cast<__nv_bfloat16 *>(pd.out)[o] = __float2bfloat16_rn(v[i]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
      if (up) {
        // Publish this warp's quarter of the unit's hidden activations: each
        // lane fences its own stores, then one lane counts the warp in. A
        // group's down units wait for 4 arrivals per up unit (no barrier
        // between the epilogue warps, so a warp that aborts blocks no other).
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(p.done + g, 1);
      }
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

template <int NB, int ACT>
int run_stream(const GemmProblem &up, const GemmProblem &down, int32_t *done, bool zeroed,
               int32_t *status, cudaStream_t stream) {
  constexpr uint32_t STAGE_BYTES = 2 * BMW * BK * 2 + 2 * NB * BK * 2;
  constexpr int S0 = (200 * 1024) / STAGE_BYTES;
  constexpr int STAGES = S0 > 8 ? 8 : S0;
  const size_t smem = 1024 + (size_t)STAGES * STAGE_BYTES;
  if (up.n_groups > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
  CUtensorMap mW1, mX, mW2, mH;
  if (!make_tma_2d_bf16(&mW1, up.B, (int64_t)up.n_groups * up.b_rows_per_group, up.K, BMW) ||
      !make_tma_2d_bf16(&mX, up.A, up.a_rows, up.K, NB) ||
      !make_tma_2d_bf16(&mW2, down.B, (int64_t)down.n_groups * down.b_rows_per_group, down.K, BMW) ||
      !make_tma_2d_bf16(&mH, down.A, down.a_rows, down.K, NB))
    return MOE_ERR_CUDA;
  StreamParams sp;
  memset(&sp, 0, sizeof(sp));
  sp.offsets = up.offsets;
  sp.n_groups = up.n_groups;
  sp.t_rows = (int)up.a_rows;
  sp.up = PassDev{up.b_rows_per_group, up.N, up.K, up.out, up.ld_out};
  sp.down = PassDev{down.b_rows_per_group, down.N, down.K, down.out, down.ld_out};
  sp.done = done;
  sp.status = status;
  const int64_t max_units = (int64_t)up.n_groups *
                            ((up.N + BMW - 1) / BMW + (down.N + BMW - 1) / BMW);
  if (max_units == 0 || up.a_rows == 0) return MOE_OK;
  if (!zeroed) MOE_CUDA_TRY(cudaMemsetAsync(done, 0, (size_t)up.n_groups * sizeof(int32_t), stream));
  auto kern = expert_stream_kernel<NB, ACT>;
  MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  int grid = num_sms();
  if (max_units < grid) grid = (int)max_units;
  // Cooperative launch: every CTA is resident, so a down unit's wait on up
  // units owned by other CTAs always ends.
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  MOE_CUDA_TRY(cudaLaunchKernelEx(&cfg, kern, mW1, mX, mW2, mH, sp));
  return last_launch_status();
}

}  // namespace

bool stream_mlp_supported(int T) { return T > 0 && T <= 128; }

size_t stream_mlp_workspace_bytes(int n_groups) { return (size_t)(n_groups > 0 ? n_groups : 1) * 4; }

int launch_stream_mlp(const GemmProblem &up, int act, const GemmProblem &down, int max_tokens,
                      int32_t *done, bool counters_zeroed, int32_t *dev_status,
                      cudaStream_t stream) {
  const bool gated = act == kActSwiglu;
  if (max_tokens <= 32)
    return gated ? run_stream<32, kActSwiglu>(up, down, done, counters_zeroed, dev_status, stream)
                 : run_stream<32, kActGelu>(up, down, done, counters_zeroed, dev_status, stream);
  if (max_tokens <= 64)
    return gated ? run_stream<64, kActSwiglu>(up, down, done, counters_zeroed, dev_status, stream)
                 : run_stream<64, kActGelu>(up, down, done, counters_zeroed, dev_status, stream);
  if (max_tokens <= 128)
    return gated ? run_stream<128, kActSwiglu>(up, down, done, counters_zeroed, dev_status, stream)
                 : run_stream<128, kActGelu>(up, down, done, counters_zeroed, dev_status, stream);
  return MOE_ERR_UNSUPPORTED;
}

}  // namespace moe
