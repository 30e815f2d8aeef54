// Combination of attention partials computed over disjoint key ranges: the one
// exchange a decode attention needs when its KV cache is split by position over
// several devices (each device attends its own rows, the partials are gathered,
// then merged here).  The gist.science summary keeps all KV caches in one GPU's
// HBM ("Bedeutung"); splitting them is the plain decomposition of the softmax:
//   M = max_k m_k,  w_k = exp(m_k - M),  o = sum_k w_k o_k / sum_k w_k l_k.
#include "common.cuh"
#include "internal.h"

namespace stdb {
namespace {

// One thread per 4 output columns of one row; the partials of that item are read
// part by part (n_parts is small: one per device).
__global__ void __launch_bounds__(256)
merge_partials_kernel(int64_t rows, int d, int n_parts, const float* o_parts, const float* ml_parts, float* o) {
  pdl_wait();  // memory of earlier kernels in the stream is visible from here on
  pdl_trigger();
  const int64_t items = rows * (d / 4);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < items; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / (d / 4);
    const int col = (int)(i % (d / 4)) * 4;
    float M = -INFINITY;
    for (int k = 0; k < n_parts; ++k) M = fmaxf(M, __ldg(ml_parts + ((size_t)k * rows + r) * 2));
    const float ref = M == -INFINITY ? 0.f : M;
    float L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k = 0; k < n_parts; ++k) {
      const float2 ml = __ldg(reinterpret_cast<const float2*>(ml_parts + ((size_t)k * rows + r) * 2));
      const float w = ex2((ml.x - ref) * kLog2e);  // exp(m_k - M); 0 for an empty range
      L += w * ml.y;
      const float4 x = __ldg(reinterpret_cast<const float4*>(o_parts + ((size_t)k * rows + r) * d + col));
      acc.x += w * x.x;
      acc.y += w * x.y;
      acc.z += w * x.z;
      acc.w += w * x.w;
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    *reinterpret_cast<float4*>(o + r * d + col) = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  }
}

}  // namespace

cudaError_t launch_merge_partials(int64_t rows, int d, int n_parts, const float* o_parts, const float* ml_parts,
                                  float* o, int sms, cudaStream_t s) {
  const int64_t items = rows * (d / 4);
  int64_t blocks = (items + 255) / 256;
  if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
  if (blocks < 1) blocks = 1;
  return launch_pdl(merge_partials_kernel, dim3((unsigned)blocks), dim3(256), 0, s, rows, d, n_parts, o_parts,
                    ml_parts, o);
}

}  // namespace stdb
