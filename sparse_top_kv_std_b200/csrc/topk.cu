// Exact top-K of the selection scores ("Methodik" item 4 of the gist.science
// summary: keep the K visual KV entries with the highest averaged text-to-
// visual attention), one CTA of 1024 threads per (layer, sequence, KV head).
//
// 1. Radix select on an order-preserving 32-bit key of each float (4 passes of
//    8-bit digits, shared-memory histograms) finds the K-th largest key tau and
//    how many entries equal to tau are still needed.
// 2. Compaction: every warp owns a contiguous index range; warp ballots count
//    the entries above tau and equal to tau, a scan over the 32 warps decides
//    which equal entries are taken (the lowest positions) and where each warp
//    writes, and a second sweep writes the positions in ascending order.
// Deterministic: the result does not depend on scheduling.
#include "common.cuh"
#include "internal.h"

namespace stdb {
namespace {

constexpr int TOPK_THREADS = 1024;
constexpr int TOPK_WARPS = TOPK_THREADS / 32;

__device__ __forceinline__ uint32_t order_key(float x) { return score_order_key(x); }

// hist0 (optional): [rows][256] counts of the top 8 key bits of every row's n entries, made
// while the scores were written; the first radix pass then reads it instead of the scores.
__global__ void __launch_bounds__(TOPK_THREADS)
topk_kernel(const float* scores, int64_t stride, const int32_t* n_dev, int n_const, int n_div,
            int n_mod, int K, int32_t* idx, const uint32_t* hist0, int* err) {
  pdl_wait();  // memory of earlier kernels in the stream is visible from here on
  pdl_trigger();
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int s_remaining;
  __shared__ int w_gt[TOPK_WARPS], w_eq[TOPK_WARPS], w_eq_before[TOPK_WARPS], w_out_before[TOPK_WARPS];

  const int p = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = n_dev ? n_dev[(p / n_div) % n_mod] : n_const;
  const float* row = scores + (size_t)p * stride;
  int32_t* out = idx + (size_t)p * K;
  if (n > stride) {  // a device length above the host-side bound the buffer was sized for
    if (tid == 0) flag_error(err, STD_DEVERR_NVIS_MAX);
    return;
  }
  if (n < K || n <= 0) {
    if (tid == 0) flag_error(err, STD_DEVERR_K_RANGE);
    return;
  }
  if (tid == 0) {
    s_prefix = 0u;
    s_mask = 0u;
    s_remaining = K;
  }
  // ---- radix select of the K-th largest key
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += TOPK_THREADS) hist[i] = 0u;
    __syncthreads();
    const uint32_t prefix = s_prefix, mask = s_mask;
    if (shift == 24 && hist0) {
      for (int i = tid; i < 256; i += TOPK_THREADS) hist[i] = hist0[(size_t)p * 256 + i];
    } else {
      for (int i = tid; i < n; i += TOPK_THREADS) {
        const uint32_t k = order_key(row[i]);
        if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
      }
    }
    __syncthreads();
    if (tid == 0) {
      int rem = s_remaining;
      int digit = 255;
      for (; digit > 0; --digit) {
        const int cnt = (int)hist[digit];
        if (cnt >= rem) break;
        rem -= cnt;
      }
      s_remaining = rem;
      s_prefix = prefix | ((uint32_t)digit << shift);
      s_mask = mask | (255u << shift);
    }
    __syncthreads();
  }
  const uint32_t tau = s_prefix;
  const int need_eq = s_remaining;  // entries equal to tau to take, lowest positions first

  // ---- compaction, pass A: per-warp counts over a contiguous range
  const int per_warp = ((n + TOPK_WARPS - 1) / TOPK_WARPS + 31) / 32 * 32;
  const int w_begin = warp * per_warp;
  const int w_end = min(n, w_begin + per_warp);
  int gt = 0, eq = 0;
  for (int base = w_begin; base < w_end; base += 32) {
    const int i = base + lane;
    const uint32_t k = i < w_end ? order_key(row[i]) : 0u;
    const bool valid = i < w_end;
    gt += __popc(__ballot_sync(0xffffffffu, valid && k > tau));
    eq += __popc(__ballot_sync(0xffffffffu, valid && k == tau));
  }
  if (lane == 0) {
    w_gt[warp] = gt;
    w_eq[warp] = eq;
  }
  __syncthreads();
  if (tid == 0) {
    int eq_acc = 0, out_acc = 0;
    for (int w = 0; w < TOPK_WARPS; ++w) {
      w_eq_before[w] = eq_acc;
      w_out_before[w] = out_acc;
      const int take_eq = max(0, min(w_eq[w], need_eq - eq_acc));
      out_acc += w_gt[w] + take_eq;
      eq_acc += w_eq[w];
    }
  }
  __syncthreads();
  // ---- pass B: write selected positions in ascending order
  int eq_seen = w_eq_before[warp];
  int out_pos = w_out_before[warp];
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int base = w_begin; base < w_end; base += 32) {
    const int i = base + lane;
    const bool valid = i < w_end;
    const uint32_t k = valid ? order_key(row[i]) : 0u;
    const bool is_eq = valid && k == tau;
    const uint32_t eq_bits = __ballot_sync(0xffffffffu, is_eq);
    const int eq_rank = eq_seen + __popc(eq_bits & lt_mask);
    const bool take = valid && (k > tau || (is_eq && eq_rank < need_eq));
    const uint32_t take_bits = __ballot_sync(0xffffffffu, take);
    if (take && STD_DCHECK(out_pos + __popc(take_bits & lt_mask) < K && i < n, err))
      out[out_pos + __popc(take_bits & lt_mask)] = i;
    out_pos += __popc(take_bits);
    eq_seen += __popc(eq_bits);
  }
  // every warp's output run ends where the next one starts, the last one at K
  (void)STD_DCHECK(out_pos == (warp + 1 < TOPK_WARPS ? w_out_before[warp + 1] : K), err);
}

}  // namespace

cudaError_t launch_topk(const float* scores, int64_t stride, int rows, const int32_t* n_dev,
                        int n_const, int n_div, int n_mod, int K, int32_t* idx, const uint32_t* hist0, int* err,
                        cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  return launch_pdl(topk_kernel, dim3(rows), dim3(TOPK_THREADS), 0, s, scores, stride, n_dev, n_const, n_div, n_mod, K,
                    idx, hist0, err);
}

}  // namespace stdb
