// Index set of the "Streaming" draft baseline.
//
// The gist.science summary ("Experimentelle Ergebnisse", item "Vergleich")
// compares Sparse-to-Dense with a baseline named Streaming that drafts with
// streaming attention, and prints no detail of it.  Read plainly, streaming
// attention keeps a fixed set of positions instead of choosing by attention: the
// first n_sink visual positions (attention sinks) and the most recent
// K - n_sink visual positions.  The text and generated rows follow in the sparse
// cache as for top-K, so the same gather, draft and verify calls run on it.
#include "common.cuh"
#include "internal.h"

namespace stdb {
namespace {

__global__ void __launch_bounds__(256)
streaming_idx_kernel(const int32_t* nvis, int B, int Hkv, int K, int n_sink, int32_t* idx, int* err) {
  pdl_wait();  // memory of earlier kernels in the stream is visible from here on
  pdl_trigger();
  const int h = blockIdx.y, lb = blockIdx.z, b = lb % B;
  const int prob = lb * Hkv + h;
  const int nv = nvis[b];
  if (K > nv) {  // the window does not fit: the problem is skipped and flagged
    if (blockIdx.x == 0 && threadIdx.x == 0) flag_error(err, STD_DEVERR_K_RANGE);
    return;
  }
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < K; j += gridDim.x * blockDim.x)
    idx[(size_t)prob * K + j] = j < n_sink ? j : nv - K + j;  // sinks, then the last K - n_sink positions
}

}  // namespace

cudaError_t launch_streaming_indices(const int32_t* nvis, int L, int B, int Hkv, int K, int n_sink, int32_t* idx,
                                     int* err, cudaStream_t s) {
  const int bx = (K + 255) / 256 < 64 ? (K + 255) / 256 : 64;
  return launch_pdl(streaming_idx_kernel, dim3(bx, Hkv, L * B), dim3(256), 0, s, nvis, B, Hkv, K, n_sink, idx,
                    err);
}

}  // namespace stdb
