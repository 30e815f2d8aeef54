// Host-side launchers shared between the C ABI layer and the kernel files.
#pragma once

#include <atomic>
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace stdb {

// Launch `kern` on `s` with programmatic stream serialization (the kernel may
// begin while its predecessor finishes; it waits with griddepcontrol.wait).
// Kernel launches the library has issued (std_launch_count); launch_pdl counts each.
extern std::atomic<unsigned long long> g_launch_count;

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  if (e == cudaSuccess) g_launch_count.fetch_add(1, std::memory_order_relaxed);
  return e;
}

// The same with the CTAs grouped into thread-block clusters of `cluster` consecutive CTAs
// (gridDim.x a multiple of it).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                               unsigned cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  if (e == cudaSuccess) g_launch_count.fetch_add(1, std::memory_order_relaxed);
  return e;
}

// One decode-attention launch: query row r of a KV head (r = g * nq + i, g the
// query head in the group, i the query position) attends to keys
// j < len[b] + len_off + i.
struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  float* o;
  const int32_t* len;
  int len_off;
  int L, B, Hq, Hkv, G, nq, rows, d, dtype;
  int64_t cap;
  int splits;
  // Problem-aligned split (keys-on-lanes kernel; 0: stream-K over the flat tile sequence):
  // CTA c takes part c % parts of problem c / parts, an equal share of that problem's
  // tiles, so no CTA's range straddles two problems; splits = problems x parts.
  int parts;
  // With parts: the parts of a problem form one thread-block cluster of `cluster` CTAs
  // and merge their partials through distributed shared memory (set by the launch;
  // 0: the global partials and the arrival counter).
  int cluster;
  float* ws;  // partials: [prob][split][rows_pad][d] then [prob][split][rows_pad][2]
  int* err;
  uint32_t epoch;  // per-call tag of the merge counters (tensor-core kernel)
  // Fused append (tensor-core kernel; k_new == nullptr: none): rows r < new_rows of
  // k_new / v_new [L][B][Hkv][new_rows][d] are written to cache positions
  // len[b] + new_off + r before those positions are read.
  const void* k_new;
  const void* v_new;
  int new_rows, new_off;
  // Early start (tensor-core kernel), bits of STD_ATTN_EARLY_*: the kernel just before
  // this one in the stream is one of this library's (launched after every earlier write
  // to these buffers) and writes neither len nor any K/V row below len[b] + new_off - 1
  // (bit 1), nor q (bit 2).  The kernel then reads the lengths, loads the K/V tiles
  // below that row (and Q) and runs their softmax before griddepcontrol.wait, overlapping
  // the previous kernel's tail, and waits only before the tiles above that row, before
  // Q (without bit 2) and before its first global write.
  int early;
  // Key range (tensor-core kernel): only cache rows [row_begin, row_end) are attended
  // (plan_attn sets 0 and cap).  partial != 0: instead of the normalised output, write
  // o = sum_j 2^(x_j - m) v_j unnormalised to `o` and (m, l) to `ml` [rows][2] (m in
  // natural-log units of the scaled logits, l = sum_j 2^(x_j - m)); a query row that
  // attends no key gets o = 0, m = -inf, l = 0, and no length check is flagged.
  int row_begin, row_end;
  int partial;
  float* ml;
};

// Split-K kernels (fp32 operands; bf16 when the tensor-core kernel does not apply):
// rows padded to the kernel's row tile, and the workspace floats for `splits`.
int attn_rows_pad(int rows, int dtype);
size_t attn_ws_floats(int probs, int splits, int rows, int d, int dtype);
cudaError_t launch_decode_attn(const AttnArgs& a, cudaStream_t s);

// Tensor-core kernel (bf16, d in {64, 128}, rows <= 128, B <= 64): persistent
// stream-K over 128-key tiles, a.splits = number of CTAs; workspace holds
// (problems + CTAs) partial slots.
bool attn_tc_supported(const AttnArgs& a);
// The tensor-core call runs the keys-on-lanes kernel (d = 128, at most 16 query rows per
// problem), the one that honours AttnArgs::parts.
bool attn_tc_keys_on_lanes(const AttnArgs& a);
size_t attn_tc_ws_floats(int probs, int ctas, int rows, int d);
cudaError_t launch_decode_attn_tc(const AttnArgs& a, cudaStream_t s);

// 2D bf16 tensor map over `rows` rows of `inner` elements, box 64 x box_rows, 128-byte swizzle.
bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows);

struct ScoreArgs {
  const void* q_text;   // [L][B][Hq][T][d]
  const void* k_full;   // [L][B][Hkv][cap][d]
  const int32_t* nvis;  // device [B]
  int nvis_max;
  int L, B, Hq, Hkv, G, T, d, dtype;
  int64_t cap;
  float* row_m;   // [prob][G*T]  max of the scaled log2 logits
  float* row_l;   // [prob][G*T]  sum of 2^(x - m)
  float* scores;  // [prob][nvis_max]
  int* err;
  int causal_text;  // nonzero: text keys 0..t join row (g, t)'s softmax (launch_text_rowstats after pass 1)
  int prefix;       // prompt rows before the visual block (a system prompt): cache = [prefix | visual | text]
  // [prob][256]: counts of the top 8 bits of score_order_key over each problem's scores,
  // made by the tensor-core score pass as it writes the scores (the top-K's first radix pass)
  uint32_t* hist;
  // which passes run: bit 0 the row statistics (into row_m / row_l), bit 1 the scores from
  // the row statistics already there; 0 means both
  int passes;
  // nonzero: the buffer holds no text rows after the visual keys (one part of a cache split
  // by position): the extent check is prefix + nvis <= cap (the default score reads no text key)
  int keys_only;
};
// *hist_done: whether the path that ran filled a.hist (the tensor-core path does).
cudaError_t launch_select_scores(const ScoreArgs& a, cudaStream_t s, bool* hist_done);
// Causal full-row variant: merge each text row's visible text keys into pass 1's (row_m, row_l).
cudaError_t launch_text_rowstats(const ScoreArgs& a, cudaStream_t s);
// tcgen05 version for bf16 operands; cudaErrorNotSupported for shapes it does not cover.
cudaError_t launch_select_scores_tc(const ScoreArgs& a, cudaStream_t s);

// Top-K of `rows` rows of scores at scores + p * stride.  Row p has
// n_dev[(p / n_div) % n_mod] valid entries (n_const if n_dev is NULL).  idx [rows][K].
// hist0: NULL, or each row's histogram of the top 8 key bits (ScoreArgs::hist).
cudaError_t launch_topk(const float* scores, int64_t stride, int rows, const int32_t* n_dev,
                        int n_const, int n_div, int n_mod, int K, int32_t* idx, const uint32_t* hist0, int* err,
                        cudaStream_t s);

struct GatherArgs {
  const void* k_full;
  const void* v_full;
  void* k_sp;
  void* v_sp;
  const int32_t* idx;  // [prob][K]
  const int32_t* nvis;
  int32_t* len_sparse;
  int L, B, Hkv, T, K, row_bytes;
  int prefix;  // prompt rows before the visual block, copied first
  int64_t cap_full, cap_sparse;
  int* err;
  // part_rows > 0: k_full / v_full hold only global cache positions [part_pos0, part_pos0 +
  // part_rows) (cap_full is then that buffer's capacity); sparse rows whose source lies
  // elsewhere are written as zeros, so that the parts' sparse caches sum to the whole one
  int64_t part_pos0, part_rows;
};
cudaError_t launch_gather(const GatherArgs& a, cudaStream_t s);
// Selection split by position: merge of the parts' row statistics ([n_parts][n] each, exp2
// domain: M = max m_i, L = sum l_i 2^(m_i - M)); each part's top-K candidates' scores
// (cand_score[p][j] = scores[p * stride + idx[p][j]]); the parts' candidate scores laid out
// per problem in part order (cat[p][i * K + j] = part_score[i][p][j]); and the merged
// selection's positions in that layout mapped back to global visual indices.
cudaError_t launch_merge_rowstats(const float* m_parts, const float* l_parts, int n_parts, int64_t n, float* m_out,
                                  float* l_out, cudaStream_t s);
cudaError_t launch_candidate_scores(const float* scores, int64_t stride, const int32_t* idx, int probs, int K,
                                    float* cand_score, cudaStream_t s);
cudaError_t launch_concat_candidates(const float* part_score, int n_parts, int probs, int K, float* cat,
                                     cudaStream_t s);
cudaError_t launch_map_candidates(const int32_t* pos, const int32_t* part_idx, const int32_t* part_offset, int n_parts,
                                  int probs, int K, int B, int Hkv, int32_t* idx_out, int* err, cudaStream_t s);
// Sink + recent-window index set: idx[prob][j] = j (j < n_sink), else nvis[b] - K + j.
cudaError_t launch_streaming_indices(const int32_t* nvis, int L, int B, int Hkv, int K, int n_sink, int32_t* idx,
                                     int* err, cudaStream_t s);

cudaError_t launch_append(void* k_cache, void* v_cache, int64_t cap, const int32_t* len, int off,
                          const void* k_new, const void* v_new, int n_new, int L, int B, int Hkv,
                          int row_bytes, int* err, cudaStream_t s);

cudaError_t launch_commit(void* k_full, void* v_full, void* k_sp, void* v_sp, int32_t* len_full,
                          int32_t* len_sp, const int32_t* n_plus_1, int max_n, int L, int B,
                          int Hkv, int row_bytes, int64_t cap_full, int64_t cap_sparse, int* err,
                          cudaStream_t s);

// o[r] = merge of n_parts partials (o_parts [n_parts][rows][d], ml_parts [n_parts][rows][2]).
cudaError_t launch_merge_partials(int64_t rows, int d, int n_parts, const float* o_parts, const float* ml_parts,
                                  float* o, int sms, cudaStream_t s);

cudaError_t launch_accept(int B, int gamma, const int32_t* draft, const int32_t* dense,
                          int32_t* n_plus_1, int32_t* accepted, cudaStream_t s);

}  // namespace stdb
