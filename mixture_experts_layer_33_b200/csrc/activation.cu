// The elementwise activations of the expert MLPs, exposed on their own.
//
// MMOE: Modernizing Diffusion Transformers with Efficient Expert Design,
// "MoE++ expert layer": heavy experts are standard MLPs; the GELU (exact,
// erf form) and the SiLU gate of SwiGLU below are the same device
// functions the grouped-GEMM and weight-streaming epilogues apply, so
// testing them here tests the epilogues' arithmetic.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

__global__ void activation_kernel(const float *__restrict__ x, float *__restrict__ y, int64_t n,
                                  int act) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    y[i] = act == MOE_SWIGLU ? silu(x[i]) : gelu_erf(x[i]);
}

}  // namespace

int launch_activation(const float *x, float *y, int64_t n, int act, cudaStream_t stream) {
  if (n == 0) return MOE_OK;
  int64_t blocks = (n + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  activation_kernel<<<(int)blocks, 256, 0, stream>>>(x, y, n, act);
  return last_launch_status();
}

}  // namespace moe
