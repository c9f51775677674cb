// testbuild_probes.cu -- entry points that exist only in the test build of the
// library (EXATTN_TEST_BUILD; see build.py), for tests that need a device
// function of the kernels evaluated on its own.  The product library compiles
// this file to nothing and exports none of it.
#ifdef EXATTN_TEST_BUILD

#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace exattn {
namespace {

// y[i] = the kernels' FMA-pipe 2^x (exp2_poly2) at x[i]; ref[i] = CUDA's exp2f
// at x[i].  Pairs go through the packed two-wide form the softmax uses.
__global__ void exp2_poly_probe_kernel(const float *__restrict__ x, float *__restrict__ y,
                                       float *__restrict__ ref, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float x0 = x[i], x1 = i + 1 < n ? x[i + 1] : 0.f;
  const float2 p = exp2_poly2(make_float2(x0, x1));
  y[i] = p.x;
  ref[i] = exp2f(x0);
  if (i + 1 < n) {
    y[i + 1] = p.y;
    ref[i + 1] = exp2f(x1);
  }
}

}  // namespace
}  // namespace exattn

extern "C" __attribute__((visibility("default"))) attn_status_t attn_test_exp2_poly(
    const float *x, float *y, float *ref, int n, attn_stream_t stream) {
  if (!x || !y || !ref || n < 0) return ATTN_ERR_INVALID_ARG;
  if (n == 0) return ATTN_OK;
  const int pairs = (n + 1) / 2;
  exattn::exp2_poly_probe_kernel<<<(pairs + 255) / 256, 256, 0,
                                   reinterpret_cast<cudaStream_t>(stream)>>>(x, y, ref, n);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

#endif  // EXATTN_TEST_BUILD
