// Grouped expert GEMM in fp32 on CUDA cores, for fp32 layers.
//
// MMOE: Modernizing Diffusion Transformers with Efficient Expert Design,
// "MoE++ expert layer": heavy experts are standard MLPs. This is the same
// grouped GEMM D = act(A . B_g^T) as the tcgen05 kernel, kept in true fp32
// (the tensor cores' fp32-input mode is tf32, which would not meet an fp32
// tolerance). fp32 layers here are small and latency-bound.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kBM = 64, kBN = 64, kBK = 16, kThreads = 256;

template <int ACT>
__global__ void __launch_bounds__(kThreads) grouped_gemm_f32_kernel(GemmProblem p) {
  __shared__ float As[kBK][kBM + 4];
  __shared__ float Bs[kBK][kBN + 4];
  __shared__ float Bu[ACT == kActSwiglu ? kBK : 1][kBN + 4];
  __shared__ int s_group, s_row0, s_row_end;

  const float *A = static_cast<const float *>(p.A);
  const float *B = static_cast<const float *>(p.B);
  float *out = static_cast<float *>(p.out);
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;

  if (tid == 0) {
    int g = -1, r0 = 0, r1 = 0;
    int64_t t = blockIdx.y;
    for (int gi = 0; gi < p.n_groups; ++gi) {
      int64_t lo = p.offsets ? p.offsets[gi] : 0;
      int64_t hi = p.offsets ? p.offsets[gi + 1] : p.a_rows;
      check_group_rows(lo, hi, p.a_rows, p.status);
      int64_t mt = (hi - lo + kBM - 1) / kBM;
      if (t < mt) { g = gi; r0 = (int)(lo + t * kBM); r1 = (int)hi; break; }
      t -= mt;
    }
    s_group = g; s_row0 = r0; s_row_end = r1;
  }
  __syncthreads();
  const int g = s_group;
  if (g < 0) return;
  const int row0 = s_row0, row_end = s_row_end;
  const int n0 = blockIdx.x * kBN;
  const int64_t brow = (int64_t)g * p.b_rows_per_group;
  const int K = p.K, N = p.N;

  float acc[4][4] = {}, accu[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kBK) {
    for (int i = tid; i < kBM * kBK; i += kThreads) {
      int r = i / kBK, c = i % kBK, gr = row0 + r, gk = k0 + c;
      As[c][r] = (gr < row_end && gk < K) ? A[(int64_t)gr * K + gk] : 0.f;
      int n = n0 + r;
      Bs[c][r] = (n < N && gk < K) ? B[(brow + n) * K + gk] : 0.f;
      if (ACT == kActSwiglu) Bu[c][r] = (n < N && gk < K) ? B[(brow + N + n) * K + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kBK; ++kk) {
      float a[4], b[4], u[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty * 4 + i];
        b[i] = Bs[kk][tx * 4 + i];
        if (ACT == kActSwiglu) u[i] = Bu[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
          if (ACT == kActSwiglu) accu[i][j] = fmaf(a[i], u[j], accu[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int r = row0 + ty * 4 + i;
    if (r >= row_end) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v = acc[i][j];
      if (ACT == kActGelu) v = gelu_erf(v);
      if (ACT == kActSwiglu) v = silu(v) * accu[i][j];
      out[(int64_t)r * p.ld_out + n] = v;
    }
  }
}

}  // namespace

int launch_grouped_gemm_f32(const GemmProblem &p, int act, cudaStream_t stream) {
  const int64_t mt = max_m_tiles(p, kBM);
  if (mt == 0 || p.a_rows == 0) return MOE_OK;
  dim3 grid((p.N + kBN - 1) / kBN, (unsigned)mt);
  if (act == kActGelu) grouped_gemm_f32_kernel<kActGelu><<<grid, kThreads, 0, stream>>>(p);
  else if (act == kActSwiglu) grouped_gemm_f32_kernel<kActSwiglu><<<grid, kThreads, 0, stream>>>(p);
  else grouped_gemm_f32_kernel<kActNone><<<grid, kThreads, 0, stream>>>(p);
  return last_launch_status();
}

}  // namespace moe
