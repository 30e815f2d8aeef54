// Test hook for the FMA-pipe exponential used by the selection kernels.
#include "../../include/std_b200.h"
#include "common.cuh"

namespace {
__global__ void probe_exp2_kernel(const float* x, float* y_fma, float* y_sfu, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    y_fma[i] = stdb::exp2_fma(x[i]);
    y_sfu[i] = stdb::ex2(x[i]);
  }
}
}  // namespace

extern "C" int std_probe_exp2(const float* x, float* y_fma, float* y_sfu, int n, std_stream_t stream) {
  if (!x || !y_fma || !y_sfu || n < 0) return STD_ERR_INVALID_ARG;
  if (n == 0) return STD_OK;
  probe_exp2_kernel<<<(n + 255) / 256, 256, 0, stream>>>(x, y_fma, y_sfu, n);
  return cudaGetLastError() == cudaSuccess ? STD_OK : STD_ERR_CUDA;
}
