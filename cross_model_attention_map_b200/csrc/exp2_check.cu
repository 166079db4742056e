// iamap_selftest_exp2: the FMA-pipe 2^x of exp2_fma.cuh beside ex2.approx on the MUFU unit, for
// element-wise tests of the polynomial against the hardware exponential and exact values.
#include <algorithm>

#include "internal.h"
#include "exp2_fma.cuh"

namespace iamap {
namespace {

__global__ void exp2_pair_kernel(const float* __restrict__ x, float* __restrict__ y_fma,
                                 float* __restrict__ y_mufu, int64_t n) {
  // two elements per thread, as the packed form computes them
  for (int64_t k = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x); k < n;
       k += 2 * (int64_t)gridDim.x * blockDim.x) {
    const float a = x[k], b = k + 1 < n ? x[k + 1] : 0.f;
    float ya, yb;
    f2_unpack(exp2_fma_x2(f2_pack(a, b)), ya, yb);
    y_fma[k] = ya;
    y_mufu[k] = ex2(a);
    if (k + 1 < n) {
      y_fma[k + 1] = yb;
      y_mufu[k + 1] = ex2(b);
    }
  }
}

}  // namespace
}  // namespace iamap

extern "C" int iamap_selftest_exp2(const float* x, float* y_fma, float* y_mufu, int64_t n,
                                   void* stream) {
  iamap::clear_error();
  if (n < 0) return iamap::set_error(IAMAP_ERR_INVALID_ARG, "n < 0");
  if (n == 0) return IAMAP_OK;
  if (!x || !y_fma || !y_mufu) return iamap::set_error(IAMAP_ERR_INVALID_ARG, "null pointer");
  const int64_t pairs = (n + 1) / 2;
  const int blocks = (int)std::min<int64_t>((pairs + 255) / 256, 148 * 8);
  iamap::exp2_pair_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y_fma, y_mufu, n);
  IAMAP_LAUNCH_CHECK("exp2_pair_kernel");
  return IAMAP_OK;
}
