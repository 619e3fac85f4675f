// Device helpers shared by the kernels of libmoe.so (sm_100a only).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libmoe targets sm_100a (B200) only"
#endif

namespace moe {

constexpr int kWarp = 32;

// Kinds of experts and the per-id index among the constant experts, passed
// to kernels by value (no global state).
struct KindTable {
  int8_t kind[MOE_MAX_EXPERTS];
  int16_t cidx[MOE_MAX_EXPERTS];
};

__device__ __forceinline__ void set_status(int32_t *st, uint32_t bits) {
  if (st) atomicOr(reinterpret_cast<unsigned int *>(st), bits);
}

// MOE_DEBUG builds range-check indices that callers hand in (row offsets,
// rows, token lists); other builds trust them (moe_dispatch writes them).
#ifndef MOE_DEBUG
#define MOE_DEBUG 0
#endif

// The rows [lo, hi) of a group read from caller offsets: in MOE_DEBUG
// builds a group outside 0 <= lo <= hi <= rows, or with more than max_cnt
// rows, is flagged (MOE_DEV_BAD_INDEX) and treated as empty.
template <typename I>
__device__ __forceinline__ void check_group_rows(I &lo, I &hi, int64_t rows, int32_t *status,
                                                 int64_t max_cnt = INT64_MAX) {
#if MOE_DEBUG
  if (lo < 0 || hi < lo || (int64_t)hi > rows || (int64_t)(hi - lo) > max_cnt) {
    set_status(status, MOE_DEV_BAD_INDEX);
    lo = hi = 0;
  }
#else
  (void)lo; (void)hi; (void)rows; (void)status; (void)max_cnt;
#endif
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// (value, id) "better than": larger value, or equal value and lower id.
// IEEE comparison, so -0 == +0 is a tie.
__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

// Warp-wide argmax of (value, id) pairs under `better`; every lane gets it.
__device__ __forceinline__ void warp_argmax(float &bv, int &bi) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float ov = __shfl_xor_sync(0xffffffffu, bv, o);
    int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
  }
}

// Inclusive warp scan of ints.
__device__ __forceinline__ int warp_inclusive_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

// Exclusive block scan of one int per thread. `scratch` holds >= 33 ints.
// All threads of the block must call it. Returns the exclusive prefix and
// writes the block total to *total.
__device__ __forceinline__ int block_exclusive_scan(int v, int *scratch, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = (blockDim.x + 31) >> 5;
  int inc = warp_inclusive_scan(v);
  if (lane == 31) scratch[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int t = lane < nwarps ? scratch[lane] : 0;
    int ti = warp_inclusive_scan(t);
    scratch[lane] = ti - t;
    if (lane == 31) scratch[32] = ti;
  }
  __syncthreads();
  int out = scratch[warp] + inc - v;
  *total = scratch[32];
  __syncthreads();
  return out;
}

// 8 consecutive elements <-> 8 floats.
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&f)[8]) {
  uint4 u = *reinterpret_cast<const uint4 *>(p);
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ void load8(const float *p, float (&f)[8]) {
  float4 a = *reinterpret_cast<const float4 *>(p);
  float4 b = *reinterpret_cast<const float4 *>(p + 4);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void store8(__nv_bfloat16 *p, const float (&f)[8]) {
  uint4 u;
  __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  *reinterpret_cast<uint4 *>(p) = u;
}
__device__ __forceinline__ void store8(float *p, const float (&f)[8]) {
  *reinterpret_cast<float4 *>(p) = make_float4(f[0], f[1], f[2], f[3]);
  *reinterpret_cast<float4 *>(p + 4) = make_float4(f[4], f[5], f[6], f[7]);
}

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

// Packed fp32x2 arithmetic (sm_100: two fp32 FMAs per issue slot).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t r, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}
__device__ __forceinline__ uint64_t f2_splat(float x) { return f2_pack(x, x); }
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
// GELU(u) = u Phi(u) = 0.5 u (1 + erf(u / sqrt 2)), the exact (erf) form,
// two values at a time on packed fp32x2 arithmetic (the GEMM epilogues'
// issue slots are the scarce resource). erf by Abramowitz & Stegun,
// Handbook of Mathematical Functions (1964), formula 7.1.26: for a >= 0,
// erf(a) = 1 - P(t) exp(-a^2), P(t) = a1 t + ... + a5 t^5, t = 1/(1 + p a),
// |error| <= 1.5e-7. With a = |v|/sqrt 2:
//   GELU(v) = 0.5 v (1 + sign(v) erf(a)) = max(v, 0) - 0.5 |v| P(t) exp(-v^2/2),
// with -0.5 folded into P's coefficients, 1/sqrt 2 into p, and
// exp(-v^2/2) = 2^(v^2 (-0.5 log2 e)); branch-free, no cancellation for
// v < 0 (one reciprocal and one exponential per value, the rest packed).
// Evaluated in fp32: |error| <= 4e-7 max(1, |v|), far below bf16 rounding
// and the fp32 layer tolerance.
__device__ __forceinline__ void gelu_erf_x2(float &v0, float &v1) {
  const uint64_t ax = f2_pack(fabsf(v0), fabsf(v1)), v = f2_pack(v0, v1);
  float d0, d1;
  f2_unpack(f2_fma(ax, f2_splat(0.23164189f), f2_splat(1.0f)), d0, d1);
  const uint64_t t = f2_pack(rcp_approx(d0), rcp_approx(d1));
  uint64_t q = f2_fma(f2_splat(-0.5307027145f), t, f2_splat(0.7265760135f));
  q = f2_fma(q, t, f2_splat(-0.7107068705f));
  q = f2_fma(q, t, f2_splat(0.142248368f));
  q = f2_fma(q, t, f2_splat(-0.127414796f));
  q = f2_mul(f2_mul(q, t), ax);
  float s0, s1;
  f2_unpack(f2_mul(f2_mul(v, v), f2_splat(-0.72134752044f)), s0, s1);
  const uint64_t e = f2_pack(ex2_approx(s0), ex2_approx(s1));
  f2_unpack(f2_fma(q, e, f2_pack(fmaxf(v0, 0.f), fmaxf(v1, 0.f))), v0, v1);
}
__device__ __forceinline__ float gelu_erf(float v) {
  float a = v, b = v;
  gelu_erf_x2(a, b);
  return a;
}
// SiLU(u) = u / (1 + exp(-u)), with the accurate expf (a few ulps at any u).
__device__ __forceinline__ float silu(float v) { return __fdividef(v, 1.0f + expf(-v)); }

// DES-Vote fixed point: q(p) = round-half-even(p * 2^40) as int64. The
// product is exact in double and rounded once, so integer sums of votes
// are exact and independent of the order they are added in.
__device__ __forceinline__ long long vote_quantum(float p) {
  return __double2ll_rn((double)p * 1099511627776.0);
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

}  // namespace moe
