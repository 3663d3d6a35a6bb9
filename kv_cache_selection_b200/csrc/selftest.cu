// Self-test entry points of device functions that have no reference of their
// own in the CUDA library: the tests compare them with CUDA's functions.
#include <cuda_runtime.h>

#include "statekv.h"
#include "kernels.h"
#include "tc_common.cuh"

namespace skv {
namespace {

__global__ void exp2_fma_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) y[i] = tc::exp2_fma(x[i]);
}

}  // namespace
}  // namespace skv

extern "C" int statekv_selftest_exp2(const float* x, float* y, int n, void* stream) {
  if (!x || !y || n < 0) {
    skv::set_free_error("statekv_selftest_exp2: null pointer or negative n");
    return STATEKV_ERR_INVALID_ARG;
  }
  if (n == 0) return STATEKV_OK;
  skv::exp2_fma_kernel<<<(n + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    skv::set_free_error(cudaGetErrorString(e));
    return STATEKV_ERR_CUDA;
  }
  return STATEKV_OK;
}
