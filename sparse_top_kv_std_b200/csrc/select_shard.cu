// Selection over a cache split by position (one part per GPU): the steps around the
// score passes that combine the parts.  The selection score of a visual key is the mean
// over text rows of softmax(q . k / sqrt(d)) ("Methodik" item 4 of the gist.science
// summary); split over parts, each part's pass 1 gives every row's max and sum over its
// own keys, the parts' statistics merge into the whole row's (max of the maxima, sums
// rescaled to it), each part's pass 2 then scores its keys against the merged
// statistics -- the same scores as one pass over all keys -- and keeps its own top-K as
// candidates; the global top-K is the top-K of the candidates, since every key of it is
// among its own part's top-K.
#include "common.cuh"
#include "internal.h"

namespace stdb {
namespace {

// One thread per (problem, row): M = max_i m_i, L = sum_i l_i 2^(m_i - M), parts in order.
__global__ void merge_rowstats_kernel(const float* m_parts, const float* l_parts, int n_parts, int64_t n, float* m_out,
                                      float* l_out) {
  pdl_wait();
  pdl_trigger();
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    float M = -INFINITY;
    for (int k = 0; k < n_parts; ++k) M = fmaxf(M, m_parts[k * n + i]);
    float L = 0.f;
    if (M != -INFINITY) {
      for (int k = 0; k < n_parts; ++k) {
        const float l = l_parts[k * n + i];
        if (l > 0.f) L += l * ex2(m_parts[k * n + i] - M);
      }
    }
    m_out[i] = M;
    l_out[i] = L;
  }
}

// cand_score[p][j] = scores[p * stride + idx[p][j]] (an index outside the row gives -inf)
__global__ void candidate_scores_kernel(const float* scores, int64_t stride, const int32_t* idx, int probs, int K,
                                        float* cand_score) {
  pdl_wait();
  pdl_trigger();
  const int64_t n = (int64_t)probs * K;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t p = i / K;
    const int j = idx[i];  // from the top-K, which leaves idx unwritten when it flags an error
    cand_score[i] = (j >= 0 && j < stride) ? scores[p * stride + j] : -INFINITY;
  }
}

// cat[p][k * K + j] = part_score[k][p][j]: each problem's candidates in part order, so a
// position in cat increases with the global index (parts hold increasing positions and
// each part's candidates are ascending)
__global__ void concat_candidates_kernel(const float* part_score, int n_parts, int probs, int K, float* cat) {
  pdl_wait();
  pdl_trigger();
  const int64_t n = (int64_t)n_parts * probs * K;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t k = i / ((int64_t)probs * K), r = i % ((int64_t)probs * K);
    const int64_t p = r / K, j = r % K;
    cat[(p * n_parts + k) * K + j] = part_score[i];
  }
}

// idx_out[p][j] = part_idx[k][p][c] + part_offset[k][b] for pos[p][j] = k * K + c
__global__ void map_candidates_kernel(const int32_t* pos, const int32_t* part_idx, const int32_t* part_offset,
                                      int n_parts, int probs, int K, int B, int Hkv, int32_t* idx_out, int* err) {
  pdl_wait();
  pdl_trigger();
  const int64_t n = (int64_t)probs * K;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int p = (int)(i / K);
    const int b = (p / Hkv) % B;
    const int q = pos[i];
    if (q < 0 || q >= n_parts * K) {
      flag_error(err, STD_DEVERR_K_RANGE);
      idx_out[i] = 0;
      continue;
    }
    const int k = q / K, c = q % K;
    idx_out[i] = part_idx[((int64_t)k * probs + p) * K + c] + part_offset[k * B + b];
  }
}

int grid_for(int64_t n) { return (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096); }

}  // namespace

cudaError_t launch_merge_rowstats(const float* m_parts, const float* l_parts, int n_parts, int64_t n, float* m_out,
                                  float* l_out, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  return launch_pdl(merge_rowstats_kernel, dim3(grid_for(n)), dim3(256), 0, s, m_parts, l_parts, n_parts, n, m_out, l_out);
}

cudaError_t launch_candidate_scores(const float* scores, int64_t stride, const int32_t* idx, int probs, int K,
                                    float* cand_score, cudaStream_t s) {
  return launch_pdl(candidate_scores_kernel, dim3(grid_for((int64_t)probs * K)), dim3(256), 0, s, scores, stride, idx,
                    probs, K, cand_score);
}

cudaError_t launch_concat_candidates(const float* part_score, int n_parts, int probs, int K, float* cat,
                                     cudaStream_t s) {
  return launch_pdl(concat_candidates_kernel, dim3(grid_for((int64_t)n_parts * probs * K)), dim3(256), 0, s, part_score,
                    n_parts, probs, K, cat);
}

cudaError_t launch_map_candidates(const int32_t* pos, const int32_t* part_idx, const int32_t* part_offset, int n_parts,
                                  int probs, int K, int B, int Hkv, int32_t* idx_out, int* err, cudaStream_t s) {
  return launch_pdl(map_candidates_kernel, dim3(grid_for((int64_t)probs * K)), dim3(256), 0, s, pos, part_idx,
                    part_offset, n_parts, probs, K, B, Hkv, idx_out, err);
}

}  // namespace stdb
