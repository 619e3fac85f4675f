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

// One thread per pair of elements (the epilogues' packed GELU takes two).
// y may alias x: both inputs of a pair are read before either is written.
__global__ void activation_kernel(const float *x, float *y, int64_t n, int act) {
  const int64_t np = (n + 1) >> 1;
  for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < np;
       p += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = 2 * p;
    const bool two = i + 1 < n;
    float a = x[i], b = two ? x[i + 1] : 0.f;
    if (act == MOE_SWIGLU) {
      a = silu(a);
      b = silu(b);
    } else {
      gelu_erf_x2(a, b);
    }
    y[i] = a;
    if (two) y[i + 1] = b;
  }
}

}  // namespace

int launch_activation(const float *x, float *y, int64_t n, int act, cudaStream_t stream) {
  if (n == 0) return MOE_OK;
  int64_t blocks = ((n + 1) / 2 + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  activation_kernel<<<(int)blocks, 256, 0, stream>>>(x, y, n, act);
  return last_launch_status();
}

}  // namespace moe
