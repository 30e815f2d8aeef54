// Test hooks: the FMA-pipe exponential used by the selection kernels, and a
// bounded wait that nothing completes.
#include "../../include/std_b200.h"
#include "common.cuh"
#include "tc100.cuh"

namespace {
// Each thread evaluates a pair (2i, 2i + 1) through the packed polynomial.
__global__ void probe_exp2_kernel(const float* x, float* y_fma, float* y_sfu, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float x0 = x[i], x1 = i + 1 < n ? x[i + 1] : 0.f;
  float e0, e1;
  stdb::f2_split(stdb::exp2_fma2(stdb::f2_make(x0, x1)), e0, e1);
  y_fma[i] = e0;
  y_sfu[i] = stdb::ex2(x0);
  if (i + 1 < n) {
    y_fma[i + 1] = e1;
    y_sfu[i + 1] = stdb::ex2(x1);
  }
}

// Thread 0 waits, through the bounded mbarrier wait of the tensor-core kernels, on a
// barrier that no thread arrives on; the wait gives up after its time limit, raises the
// CTA's abort flag and STD_DEVERR_TIMEOUT in the device error word, and the kernel returns.
// completed[0] = 1 if the wait completed, 0 if it gave up.
__global__ void probe_wait_kernel(int* err, int* completed) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    stdb::tc::mbar_init(&bar, 1);
    abort_flag = 0;
    stdb::tc::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) completed[0] = stdb::tc::mbar_wait(&bar, 0, &abort_flag, err) ? 1 : 0;
}
}  // namespace

namespace stdb {
cudaError_t launch_probe_wait(int* err, int* completed, cudaStream_t s) {
  probe_wait_kernel<<<1, 32, 0, s>>>(err, completed);
  return cudaGetLastError();
}
}  // namespace stdb

extern "C" int std_probe_exp2(const float* x, float* y_fma, float* y_sfu, int n, std_stream_t stream) {
  if (!x || !y_fma || !y_sfu || n < 0) return STD_ERR_INVALID_ARG;
  if (n == 0) return STD_OK;
  probe_exp2_kernel<<<(n + 511) / 512, 256, 0, stream>>>(x, y_fma, y_sfu, n);
  return cudaGetLastError() == cudaSuccess ? STD_OK : STD_ERR_CUDA;
}
