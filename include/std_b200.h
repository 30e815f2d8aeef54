/*
 * std_b200.h -- C ABI of the Sparse-to-Dense (StD) decoding hot path on B200 (sm_100a).
 *
 * Sparse-to-Dense accelerates Video-LLM decoding without changing its output:
 * a sparse mode of the model (attention over a top-K subset of the visual KV)
 * drafts gamma tokens, and the dense mode (attention over the whole cache)
 * verifies them in one pass; the longest agreeing prefix plus one bonus token
 * is kept.  Sources: "Sparse-to-Dense: A Free Lunch for Lossless Acceleration
 * of Video Understanding in LLMs" -- the gist.science technical summary
 * (sections "Methodik" 2-4) and the paper abstract.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All tensor arguments are DEVICE pointers owned by the caller; the library
 *    never allocates, frees or keeps them.  Scratch space is a caller-provided
 *    device workspace whose size a *_workspace_size() query returns.
 *  - Layouts are dense, row-major, head dimension innermost:
 *        caches   [L][B][Hkv][cap][d]       (cap = dims->cap_full or cap_sparse)
 *        queries  [L][B][Hq][rows][d]
 *        outputs  [L][B][Hq][rows][d]  float32
 *    Query head hq reads KV head hq / G with G = Hq / Hkv (standard grouped-
 *    query attention; consecutive query heads share a KV head).
 *  - Element type of Q/K/V is dims->dtype: STD_F32 (float) or STD_BF16
 *    (bfloat16 bits).  Arithmetic is float32 in every kernel; bf16 operands go
 *    through the tensor cores with float32 accumulation.
 *  - Lengths (len_full, len_sparse, nvis) are int32 arrays on the DEVICE, one
 *    entry per sequence, so whole rounds run without host synchronisation and
 *    can be captured in a CUDA graph.
 *  - Every call is asynchronous on `stream` (NULL = the legacy default stream).
 *  - Return value: STD_OK (0) or a negative STD_ERR_* code.  Arguments that
 *    the host can check are checked before anything is launched; nothing is
 *    launched on error.  std_last_error() gives a message (thread-local).
 *    Conditions that depend on device-resident lengths are checked by the
 *    kernels: the offending (sequence, head) is skipped and a bit is OR-ed
 *    into a per-device error word, read with std_get_device_error().
 *  - No kernel waits on another kernel, CTA or device.  The tensor-core kernels
 *    wait only on their own CTA's mbarriers (TMA arrivals, MMA commits, warp
 *    hand-offs); every such wait gives up after 0.5 s, sets
 *    STD_DEVERR_TIMEOUT, drains its copies in flight, frees its tensor memory
 *    and returns.
 */
#ifndef STD_B200_H
#define STD_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (the runtime's CUstream_st*); NULL is the legacy default stream. */
typedef struct CUstream_st* std_stream_t;

enum std_status {
  STD_OK = 0,
  STD_ERR_INVALID_ARG = -1, /* null pointer, bad size or shape */
  STD_ERR_UNSUPPORTED = -2, /* dtype / head dim / group shape the library has no kernel for */
  STD_ERR_CAPACITY = -3,    /* a host-checkable size exceeds a cache capacity */
  STD_ERR_CUDA = -4,        /* a CUDA runtime call or launch failed */
  STD_ERR_DEVICE = -5,      /* std_get_device_error found flags set */
  STD_ERR_TIMEOUT = -6,     /* reserved; a timed-out wait inside a kernel shows as STD_DEVERR_TIMEOUT */
  STD_ERR_WORKSPACE = -7    /* workspace missing or smaller than the size query returned */
};

enum std_dtype { STD_F32 = 0, STD_BF16 = 1 };

/* Bits of the per-device error word (std_get_device_error). */
enum std_device_error {
  STD_DEVERR_CAPACITY = 1,  /* an append / commit / verify would pass the cache capacity */
  STD_DEVERR_LENGTH = 2,    /* a device length was <= 0 or beyond the capacity in attention */
  STD_DEVERR_K_RANGE = 4,   /* select: K > nvis[b], or nvis[b] + T > cap_full */
  STD_DEVERR_NVIS_MAX = 8,  /* select: nvis[b] > the host-side nvis_max bound */
  STD_DEVERR_TIMEOUT = 16,  /* a bounded wait inside a kernel gave up; that CTA's output is missing */
  STD_DEVERR_DEBUG = 32     /* debug build only (libstd_b200_debug.so, compiled with STD_DEBUG): an index
                               or cache row outside its buffer was caught and that access skipped */
};

/* Shape of the model slice a call works on.  cap_full / cap_sparse are the row
 * capacities of the full and the sparse (compacted) caches. */
typedef struct std_dims {
  int32_t L, B, Hq, Hkv, d, dtype;
  int64_t cap_full, cap_sparse;
} std_dims;

/* ---------------------------------------------------------------- library */

/* Library version as major * 10000 + minor * 100 + patch. */
int std_version(void);

/* Kernel launches this process has issued through the library so far (all
 * devices and threads), for accounting: the difference around a region counts
 * the library's kernels launched in it. */
unsigned long long std_launch_count(void);

/* Message describing the last error returned on this host thread ("" if none). */
const char* std_last_error(void);

/* Read the current device's error word into *flags (may be NULL), optionally
 * clearing it.  Orders after all work already queued on `stream` and blocks
 * the host until that work is done.  Returns STD_ERR_DEVICE if any bit was
 * set, else STD_OK (or STD_ERR_CUDA). */
int std_get_device_error(int32_t* flags, int clear, std_stream_t stream);

/* ---------------------------------------------------------------- prefill selection
 *
 * "Methodik" item 4 of the summary: the top-K visual KV entries are chosen
 * once, at prefill, from the attention scores from text tokens to visual
 * tokens, averaged; the choice differs per layer and head.  Item 2: the
 * sparse model attends only to those entries.
 *
 * For every (layer l, sequence b, KV head h):
 *   score[n] = 1/(G*T) * sum over the G query heads g of the group and the
 *              T text rows t of softmax_{n < nvis[b]}( q_text[g,t] . k_n / sqrt(d) )
 *   idx      = the K highest scores, ties to the lower position, ascending
 *   sparse cache rows [0, K)     = full rows idx[0..K)   (K and V)
 *   sparse cache rows [K, K + T) = full rows [nvis[b], nvis[b] + T) (the text)
 *   len_sparse[b] = K + T
 * The softmax runs over the visual keys only.
 */

/* Device workspace bytes std_select_topk needs for these shapes. */
size_t std_select_workspace_size(const std_dims* dims, int T, int nvis_max);

/*
 * q_text      [L][B][Hq][T][d]          text-token queries (post-RoPE)
 * k_full/v_full [L][B][Hkv][cap_full][d] prompt cache: visual rows [0, nvis[b]),
 *                                        text rows [nvis[b], nvis[b] + T)
 * nvis        device int32 [B]           visual tokens per sequence
 * nvis_max    host bound >= every nvis[b]; sizes the launch and the workspace
 * K           1 <= K <= nvis[b] (checked on the device), K <= nvis_max and
 *             K + T <= cap_sparse (checked on the host)
 * idx_out     device int32 [L][B][Hkv][K]  selected visual positions, ascending
 * k_sparse/v_sparse [L][B][Hkv][cap_sparse][d]  rows [0, K + T) written
 * len_sparse  device int32 [B]           set to K + T
 * scores_out  device float [L][B][Hkv][nvis_max] or NULL; entries n >= nvis[b]
 *             are not written
 * ws          device workspace of at least std_select_workspace_size() bytes
 */
int std_select_topk(const std_dims* dims, const void* q_text, int T, const void* k_full,
                    const void* v_full, const int32_t* nvis, int nvis_max, int K,
                    int32_t* idx_out, void* k_sparse, void* v_sparse, int32_t* len_sparse,
                    float* scores_out, void* ws, size_t ws_bytes, std_stream_t stream);

/* Flags of std_select_topk_ex. */
enum std_select_flags {
  /* Causal full-row score: the softmax of text row (g, t) runs over the visual keys
   * and the text keys [nvis[b], nvis[b] + t] -- the keys that query sees in the
   * prompt's causal attention -- instead of the visual keys only.  The score of
   * visual key n is still the mean over the G * T rows of that row's probability
   * at n, so the scores sum to 1 minus the rows' mean mass on text keys.  The
   * summary's "average attention from text to visual tokens" ("Methodik" item 4)
   * does not say which keys the softmax covers; this is the other plain reading. */
  STD_SELECT_CAUSAL_TEXT = 1
};

/* std_select_topk for prompts with a prefix and with flags (n_prefix = 0 and
 * flags = 0 give std_select_topk; same workspace).
 * n_prefix  prompt rows before the video (a system prompt), the same for every
 *           sequence: the full cache holds [n_prefix rows | nvis[b] visual rows |
 *           T text rows].  idx_out and scores_out stay positions within the visual
 *           block; the sparse cache becomes [n_prefix rows | K selected visual rows |
 *           T text rows] and len_sparse n_prefix + K + T.  Requires
 *           n_prefix + nvis_max + T <= cap_full and n_prefix + K + T <= cap_sparse.
 *           The default score ignores the prefix rows (the softmax runs over the
 *           visual keys); with STD_SELECT_CAUSAL_TEXT they join every text row's
 *           softmax, as they precede it.
 * flags     a bitwise OR of std_select_flags; unknown bits are rejected with
 *           STD_ERR_INVALID_ARG. */
int std_select_topk_ex(const std_dims* dims, const void* q_text, int T, const void* k_full,
                       const void* v_full, const int32_t* nvis, int nvis_max, int K, int n_prefix,
                       int flags, int32_t* idx_out, void* k_sparse, void* v_sparse, int32_t* len_sparse,
                       float* scores_out, void* ws, size_t ws_bytes, std_stream_t stream);

/* The selection's top-K step alone, on caller-supplied float32 scores:
 * `rows` independent rows of `n` scores each (row stride n), K <= n.
 * idx_out [rows][K] receives the K highest positions of each row, ties to the
 * lower position, ascending.  -0.0 ranks equal to +0.0; NaN is not allowed. */
int std_topk_from_scores(const float* scores, int rows, int n, int K, int32_t* idx_out,
                         std_stream_t stream);

/* ---------------------------------------------------------------- selection over a cache split by position
 *
 * When one sequence's prompt cache is split by position over several GPUs (one part
 * each), the selection above runs in four steps with two exchanges between them, and
 * gives the indices the single-GPU call gives (up to ties at the K-th score).  Per text
 * row r of a problem the softmax over all visual keys is exp(x_rn - m_r) / l_r; split
 * over parts, every part computes its own rows' (m, l) over its keys, the parts' values
 * merge into the whole row's, every part scores its keys against the merged (m, l) --
 * the same scores -- and keeps its own top-K, and the global top-K is the top-K of the
 * parts' candidates (every one of its keys is among its own part's top-K):
 *   1. std_select_rowstats on every part;          all-gather (row_m, row_l)
 *   2. std_merge_rowstats on every part;
 *      std_select_candidates on every part;        all-gather (cand_idx, cand_score)
 *   3. std_merge_candidates on every part          (the global idx, ascending)
 *   4. std_gather_sparse_part on every part;       all-reduce (sum) of the sparse caches
 * The row statistics are in the exp2 domain: for the scaled logit x = q . k / sqrt(d),
 * m = log2(e) * max_n x_n and l = sum_n 2^(log2(e) x_n - m).  Only the default score
 * (flags 0: the softmax over the visual keys) splits this way.  A part's buffers hold
 * the same per-(layer, sequence, KV head) layout as the full cache, restricted to the
 * part's positions; every part must hold at least K visual keys of every sequence.
 */

/* Step 1: the row statistics of this part's visual keys: keys n < nvis[b] at rows
 * n_prefix + n of k_full (this part's buffer; n_prefix here is the part's first visual
 * row, nvis[b] its visual keys, 1 <= nvis[b] <= nvis_max, n_prefix + nvis_max <= cap_full).
 * row_m, row_l  device float [L][B][Hkv][G * T], G = Hq / Hkv, row g * T + t. */
int std_select_rowstats(const std_dims* dims, const void* q_text, int T, const void* k_full, const int32_t* nvis,
                        int nvis_max, int n_prefix, float* row_m, float* row_l, std_stream_t stream);

/* Step 2a: merge n_parts parts' row statistics, m_parts / l_parts device float
 * [n_parts][n] (part-major, n = L * B * Hkv * G * T), into row_m / row_l [n]:
 * m = max_i m_i, l = sum_i l_i 2^(m_i - m) (a part with l_i = 0 contributes nothing). */
int std_merge_rowstats(int64_t n, int n_parts, const float* m_parts, const float* l_parts, float* row_m, float* row_l,
                       std_stream_t stream);

/* Device workspace bytes std_select_candidates needs (the part's scores). */
size_t std_select_candidates_workspace_size(const std_dims* dims, int nvis_max);

/* Step 2b: this part's scores against the merged row statistics (row_m, row_l from
 * std_merge_rowstats) and its K highest: cand_idx device int32 [L][B][Hkv][K] (positions
 * within the part's visual keys, ascending, ties to the lower position), cand_score device
 * float [L][B][Hkv][K] their scores.  K <= nvis[b] is checked on the device
 * (STD_DEVERR_K_RANGE).  scores_out: device float [L][B][Hkv][nvis_max] or NULL. */
int std_select_candidates(const std_dims* dims, const void* q_text, int T, const void* k_full, const int32_t* nvis,
                          int nvis_max, int n_prefix, const float* row_m, const float* row_l, int K,
                          int32_t* cand_idx, float* cand_score, float* scores_out, void* ws, size_t ws_bytes,
                          std_stream_t stream);

/* Device workspace bytes std_merge_candidates needs. */
size_t std_merge_candidates_workspace_size(const std_dims* dims, int n_parts, int K);

/* Step 3: the global top-K from n_parts parts' candidates, cand_idx / cand_score device
 * [n_parts][L][B][Hkv][K] (part-major; parts in increasing position order), and
 * part_offset device int32 [n_parts][B]: the global visual index of each part's first
 * visual key per sequence.  idx_out [L][B][Hkv][K] receives global visual indices of the
 * K highest candidates, ties to the lower index, ascending -- what std_select_topk_ex
 * gives on the whole cache (its ties to the lower position agree with the candidates'
 * order because the parts come in position order). */
int std_merge_candidates(const std_dims* dims, int n_parts, int K, const int32_t* cand_idx, const float* cand_score,
                         const int32_t* part_offset, int32_t* idx_out, void* ws, size_t ws_bytes,
                         std_stream_t stream);

/* Step 4: std_gather_sparse on one part.  k_full / v_full hold the global cache positions
 * [part_pos0, part_pos0 + part_rows) of the prompt [n_prefix rows | nvis[b] visual rows |
 * T text rows] (dims->cap_full = the part buffer's capacity >= part_rows); idx and nvis
 * are global (std_merge_candidates' output, the whole sequence's visual count).  Sparse
 * rows whose source lies in this part are copied, the others written as zeros, so the
 * parts' sparse caches sum (an all-reduce) to the one std_gather_sparse builds. */
int std_gather_sparse_part(const std_dims* dims, const void* k_full, const void* v_full, const int32_t* nvis,
                           const int32_t* idx, int K, int T, int n_prefix, int64_t part_pos0, int64_t part_rows,
                           void* k_sparse, void* v_sparse, int32_t* len_sparse, std_stream_t stream);

/* ---------------------------------------------------------------- streaming draft baseline
 *
 * Not the method's selection.  The gist.science summary ("Experimentelle
 * Ergebnisse", item "Vergleich") compares Sparse-to-Dense with a baseline named
 * Streaming that drafts with streaming attention, without details.  Read plainly,
 * it keeps fixed positions instead of the top-K by attention: the first n_sink
 * visual positions (attention sinks) and the most recent K - n_sink.  These two
 * calls build such a sparse cache so that the draft / verify / commit calls run
 * on it unchanged; std_gather_sparse also serves any caller-chosen index set.
 */

/* idx_out [L][B][Hkv][K] (device int32) <- for sequence b: j for j < n_sink, then
 * nvis[b] - K + j (ascending).  Requires 0 <= n_sink <= K; K <= nvis[b] is checked
 * on the device (STD_DEVERR_K_RANGE, that sequence skipped). */
int std_streaming_indices(const std_dims* dims, const int32_t* nvis, int K, int n_sink, int32_t* idx_out,
                          std_stream_t stream);

/* The gather step of std_select_topk_ex on caller-given indices, for a full
 * cache of [P = n_prefix rows | nvis[b] visual rows | T text rows]: sparse rows
 * [0, P) <- the prefix rows, rows [P, P + K) <- visual rows idx[l][b][h][j] (any
 * order, each a position in [0, nvis[b]); one outside it flags
 * STD_DEVERR_K_RANGE and leaves that row), rows [P + K, P + K + T) <- the text
 * rows, len_sparse[b] <- P + K + T.  P + K + T <= cap_sparse. */
int std_gather_sparse(const std_dims* dims, const void* k_full, const void* v_full, const int32_t* nvis,
                      const int32_t* idx, int K, int T, int n_prefix, void* k_sparse, void* v_sparse,
                      int32_t* len_sparse, std_stream_t stream);

/* ---------------------------------------------------------------- decode attention
 *
 * All query rows that read one KV head -- the G grouped query heads times the
 * query positions -- are processed together, so each K/V byte is read once.
 * bf16 operands (head dim 64 or 128, G x query rows <= 128, B <= 64) run on a
 * persistent tensor-core kernel: the 128-key tiles of all (layer, sequence, KV
 * head) problems form one sequence that the CTAs split into equal slices;
 * `splits` = 0 launches one CTA per SM -- or one CTA per problem when there are
 * between half and all as many problems as SMs and `cap` is short (at most 2048
 * keys for up to 16 query rows, 8192 otherwise), or, when all problems together
 * have fewer than 5 tiles per SM (at `cap` keys), a few CTAs per problem: for head
 * dim 128 and at most 16 query rows per problem (the draft) each problem is cut
 * into equal parts of about 3 tiles, one CTA each (at most 16 parts, and at
 * most half as many CTAs as SMs in all), otherwise about one CTA per 5 tiles of the whole sequence -- and
 * splits = s > 0 launches s x L x B x Hkv CTAs (for the draft's kernel: s equal
 * parts of every problem; with 2 to 16 parts, the parts of a problem form one
 * thread-block cluster and merge in distributed shared memory where such a
 * cluster fits the device).  With an early start (STD_ATTN_EARLY_*) and at most 16
 * query rows, one CTA per problem applies up to 8192 keys; such a call never
 * needs more workspace than the same call without the flags.  fp32 operands (and
 * bf16 with B > 64) use split-K kernels with `splits` key ranges per problem (0 =
 * automatic).  Either way
 * the partial results go to the workspace.  The tensor-core kernel merges them
 * itself: the last CTA to finish a slice of a problem (an arrival counter per
 * problem, no waiting) combines that problem's partials; the split-K kernels
 * leave the merge to a second kernel.
 */

/* Device workspace bytes for a decode-attention call with `q_rows` query rows
 * per query head (1 for the sparse draft, gamma + 1 for the verify) over a
 * cache of `cap` rows (dims->cap_sparse for the draft, dims->cap_full for the
 * verify), and `splits` as above (0 resolves on the current device).  Returns
 * 0 when the arguments are invalid. */
size_t std_attn_workspace_size(const std_dims* dims, int q_rows, int64_t cap, int splits);

/* The number of CTAs (tensor-core kernel) or key splits per problem (split-K
 * kernels) a decode-attention call with these arguments uses, or a negative
 * STD_ERR_* code. */
int std_attn_splits(const std_dims* dims, int q_rows, int64_t cap, int splits);

/* The same for a call with early-start flags (bits of STD_ATTN_EARLY_*, defined
 * below; unknown bits, or STD_ATTN_EARLY_Q without STD_ATTN_EARLY_KV, are
 * STD_ERR_INVALID_ARG): an early-started call may use fewer CTAs, never more
 * workspace. */
int std_attn_splits_ex(const std_dims* dims, int q_rows, int64_t cap, int splits, int flags);

/*
 * Sparse draft attention ("Methodik" item 2: the draft model M_s uses top-K
 * attention over the selected KV).  For every query head:
 *     o = softmax_j(q . k_j / sqrt(d)) v_j   over sparse rows j < len_sparse[b] + len_offset
 * q          [L][B][Hq][1][d]
 * k_sparse/v_sparse [L][B][Hkv][cap_sparse][d]
 * len_sparse device int32 [B]: committed sparse rows; len_offset (>= 0) counts
 *            rows appended since (std_kv_append with the same offset base)
 * o          float [L][B][Hq][1][d]
 */
int std_sparse_decode_attn(const std_dims* dims, const void* q, const void* k_sparse,
                           const void* v_sparse, const int32_t* len_sparse, int len_offset,
                           float* o, int splits, void* ws, size_t ws_bytes, std_stream_t stream);

/*
 * Dense verify attention ("Methodik" item 3: the dense model verifies the gamma
 * drafted tokens in parallel with one pass over the full KV cache).  Query row
 * i = 0..gamma of each query head attends causally:
 *     o_i = softmax_j(q_i . k_j / sqrt(d)) v_j   over full rows j < len_full[b] + i + 1
 * q         [L][B][Hq][gamma + 1][d]
 * k_full/v_full [L][B][Hkv][cap_full][d]; the gamma + 1 new rows must already sit at
 *           [len_full[b], len_full[b] + gamma + 1) (std_kv_append)
 * len_full  device int32 [B]: committed context length, before the new rows
 * o         float [L][B][Hq][gamma + 1][d]
 * Requires 0 <= gamma <= 31 and G * (gamma + 1) <= 128.
 */
int std_dense_verify_attn(const std_dims* dims, const void* q, int gamma, const void* k_full,
                          const void* v_full, const int32_t* len_full, float* o, int splits,
                          void* ws, size_t ws_bytes, std_stream_t stream);

/* ---------------------------------------------------------------- append + attention in one launch
 *
 * The decode loop appends the K/V rows of its new inputs and then attends over
 * them ("Methodik" item 3: each draft step, and the verify pass, see the inputs
 * appended so far).  These calls do both in one launch: the tensor-core kernel
 * writes the new rows into the cache (each by the CTA that loads its tile) before
 * reading them; other paths launch std_kv_append's kernel first.  Results equal
 * std_kv_append followed by the attention call.  Capacity beyond cap shows as
 * STD_DEVERR_LENGTH (that sequence skipped).
 */

/* Draft step: k_new/v_new [L][B][Hkv][1][d] go to sparse row len_sparse[b] +
 * len_offset - 1, then std_sparse_decode_attn with len_offset (>= 1, it counts the
 * new row). */
int std_sparse_decode_attn_append(const std_dims* dims, const void* q, void* k_sparse, void* v_sparse,
                                  const int32_t* len_sparse, int len_offset, const void* k_new, const void* v_new,
                                  float* o, int splits, void* ws, size_t ws_bytes, std_stream_t stream);

/* std_sparse_decode_attn_append with `flags`, bits that let the launch start reading
 * before the kernel just before it in the stream has finished (programmatic dependent
 * launch; the call still orders every write after that kernel):
 *   STD_ATTN_EARLY_KV  the previous kernel is one of this library's, launched after every
 *                      earlier write to this call's buffers, and writes neither len_sparse
 *                      nor any K/V row below len_sparse[b] + len_offset - 2 (true when it is
 *                      the previous draft step on the same cache, or attention on other
 *                      caches); the K/V tiles below that row are fetched early.
 *   STD_ATTN_EARLY_Q   with STD_ATTN_EARLY_KV: it does not write q either (q is fetched early).
 * A wrong promise gives wrong results.  The bf16 tensor-core kernel uses the flags; other
 * paths ignore them.  std_decode_round passes both for its draft steps after the first. */
#define STD_ATTN_EARLY_KV 1
#define STD_ATTN_EARLY_Q 2
int std_sparse_decode_attn_append_ex(const std_dims* dims, const void* q, void* k_sparse, void* v_sparse,
                                     const int32_t* len_sparse, int len_offset, const void* k_new,
                                     const void* v_new, float* o, int splits, int flags, void* ws, size_t ws_bytes,
                                     std_stream_t stream);

/* Verify: k_new/v_new [L][B][Hkv][gamma + 1][d] go to full rows [len_full[b],
 * len_full[b] + gamma + 1), then std_dense_verify_attn. */
int std_dense_verify_attn_append(const std_dims* dims, const void* q, int gamma, void* k_full, void* v_full,
                                 const int32_t* len_full, const void* k_new, const void* v_new, float* o, int splits,
                                 void* ws, size_t ws_bytes, std_stream_t stream);

/* ---------------------------------------------------------------- attention over a key range
 *
 * The summary keeps every KV cache in one GPU's HBM ("Bedeutung"); when a cache
 * is split by position over several GPUs, each attends its own rows and one
 * exchange of per-row partials combines them.  These calls are the decode
 * attention calls above restricted to the cache rows [row_begin, row_end) of
 * the given buffers, whose row r holds sequence position pos0 + r (pos0 = 0: the
 * buffers are the whole cache).  Query row i of a sequence attends the positions
 * j it attends in the full call (j < len_full[b] + 1 + i for the verify,
 * j < len_sparse[b] + len_offset for the draft) that lie in that row range.
 * Instead of the normalised output they write, per query row,
 *     o_part = sum_j exp(s_j - m) v_j       (s_j = q . k_j / sqrt(d))
 *     ml_part = (m, l),  l = sum_j exp(s_j - m)
 * where m is a reference value the kernel chose near the row's largest logit
 * (not necessarily equal to it): o_part / l and m + ln l are the determined
 * quantities.  A row that attends no key gets o_part = 0, m = -inf, l = 0.
 * std_merge_partials combines the partials of disjoint ranges into the full
 * result.  bf16 tensor-core shapes only (STD_ERR_UNSUPPORTED otherwise); the
 * workspace is that of the full call (std_attn_workspace_size with the same
 * cap and splits).  Lengths outside the range are not errors here (a range may
 * hold no attended row).
 * o_part  float [L][B][Hq][q_rows][d];  ml_part float [L][B][Hq][q_rows][2]
 * Requires 0 <= row_begin <= row_end <= cap and 0 <= pos0 <= 2^30.
 */
int std_dense_verify_attn_partial(const std_dims* dims, const void* q, int gamma, const void* k_full,
                                  const void* v_full, const int32_t* len_full, int64_t pos0, int64_t row_begin,
                                  int64_t row_end, float* o_part, float* ml_part, int splits, void* ws,
                                  size_t ws_bytes, std_stream_t stream);

int std_sparse_decode_attn_partial(const std_dims* dims, const void* q, const void* k_sparse, const void* v_sparse,
                                   const int32_t* len_sparse, int len_offset, int64_t pos0, int64_t row_begin,
                                   int64_t row_end, float* o_part, float* ml_part, int splits, void* ws,
                                   size_t ws_bytes, std_stream_t stream);

/* Merge n_parts partials of the same query rows over disjoint key ranges:
 *     M = max_k m_k,  w_k = exp(m_k - M),  o = sum_k w_k o_part_k / sum_k w_k l_k
 * (o = 0 for a row no range attends).  o_parts [n_parts][rows][d] and ml_parts
 * [n_parts][rows][2] (the layout an all-gather of the per-GPU partials gives),
 * o [rows][d], all device float; d a multiple of 4.  rows = 0 does nothing. */
int std_merge_partials(int64_t rows, int d, int n_parts, const float* o_parts, const float* ml_parts, float* o,
                       std_stream_t stream);

/* ---------------------------------------------------------------- verify attention, no workspace
 *
 * No counterpart in the paper: this entry point exists for callers, not for the method.
 *
 * std_dense_verify_attn without the workspace argument, for code that cannot
 * hand the library device memory while it decodes: a plugin inside another
 * engine that owns every device allocation, or a latency-bound service that
 * bans cudaMalloc/cudaFree after start-up because they can synchronise the
 * device and stall unrelated streams.  The split-K partials go to a scratch
 * array compiled into the library: STD_NOALLOC_SCRATCH_BYTES on every GPU on
 * which the library is loaded, held until the process exits.  Arguments,
 * layouts, requirements and results are those of std_dense_verify_attn.
 *  - A call whose partials need more than STD_NOALLOC_SCRATCH_BYTES is
 *    rejected with STD_ERR_WORKSPACE before anything is launched.  It never
 *    allocates.  std_attn_workspace_size(dims, gamma + 1, cap_full, splits)
 *    gives the bytes a call uses; a call touches the shared array exactly when
 *    that is non-zero.  On the bf16 tensor-core kernel that is every call,
 *    splits = 1 included (a persistent CTA may cover parts of two problems
 *    and the merge counters live there too); only the split-K kernels (fp32
 *    operands, more than 64 sequences) need none at splits = 1.
 *  - The first call on a device looks up the array's device address with that
 *    device current; make that first call before capturing any stream.
 *  - All calls on a device share the one array and it keeps what the last call
 *    wrote.  Nothing in it has to start at zero (each call writes every partial
 *    it reads), but two calls whose kernels may overlap on the GPU -- different
 *    streams with no ordering between them -- race on it and corrupt each
 *    other's results.
 */
#define STD_NOALLOC_SCRATCH_BYTES (16u << 20)

int std_dense_verify_attn_noalloc(const std_dims* dims, const void* q, int gamma, const void* k_full,
                                  const void* v_full, const int32_t* len_full, float* o, int splits,
                                  std_stream_t stream);

/* ---------------------------------------------------------------- acceptance
 *
 * "Methodik" item 3: keep the longest prefix of draft tokens that matches the
 * dense model's predictions (n tokens) plus one bonus token.
 * draft        device int32 [B][gamma]      drafted tokens d_0..d_{gamma-1}
 * dense_argmax device int32 [B][gamma + 1]  dense prediction after each input
 * n_plus_1     device int32 [B]             n + 1, in [1, gamma + 1]
 * accepted     device int32 [B][gamma + 1]  dense_argmax[b][0..n], then -1
 * The bonus token is dense_argmax[b][n].  Requires 0 <= gamma <= 31.
 */
int std_accept_prefix(int B, int gamma, const int32_t* draft, const int32_t* dense_argmax,
                      int32_t* n_plus_1, int32_t* accepted, std_stream_t stream);

/* ---------------------------------------------------------------- cache bookkeeping */

/* Write `n_new` rows per (layer, sequence, KV head) into a cache at positions
 * len[b] + pos_offset + r, r < n_new.  k_new/v_new [L][B][Hkv][n_new][d];
 * cache [L][B][Hkv][cap][d].  Lengths are not changed.  A sequence whose rows
 * would pass `cap` is skipped and flags STD_DEVERR_CAPACITY. */
int std_kv_append(const std_dims* dims, void* k_cache, void* v_cache, int64_t cap,
                  const int32_t* len, int pos_offset, const void* k_new, const void* v_new,
                  int n_new, std_stream_t stream);

/* "Methodik" item 3, last step: append the accepted inputs to the context.
 * For every sequence, the n_plus_1[b] verified rows at full positions
 * [len_full[b], len_full[b] + n_plus_1[b]) are copied (K and V) to sparse
 * positions [len_sparse[b], ...), then both lengths grow by n_plus_1[b].
 * max_n bounds every n_plus_1[b] (gamma + 1) and sizes the launch. */
int std_kv_commit(const std_dims* dims, void* k_full, void* v_full, void* k_sparse,
                  void* v_sparse, int32_t* len_full, int32_t* len_sparse,
                  const int32_t* n_plus_1, int max_n, std_stream_t stream);

/* ---------------------------------------------------------------- one decode round */

typedef struct std_cache {
  void* k_full;         /* [L][B][Hkv][cap_full][d] */
  void* v_full;
  void* k_sparse;       /* [L][B][Hkv][cap_sparse][d] */
  void* v_sparse;
  int32_t* len_full;    /* device [B], committed context length */
  int32_t* len_sparse;  /* device [B], committed sparse length */
} std_cache;

typedef struct std_round_io {
  const void* q_draft;          /* [gamma][L][B][Hq][1][d]   query of draft step j */
  const void* k_draft;          /* [gamma][L][B][Hkv][1][d]  K/V row of draft step j's input */
  const void* v_draft;
  const void* q_verify;         /* [L][B][Hq][gamma + 1][d] */
  const void* k_verify;         /* [L][B][Hkv][gamma + 1][d] K/V rows of the gamma + 1 inputs */
  const void* v_verify;
  const int32_t* draft_tokens;  /* [B][gamma] */
  const int32_t* dense_tokens;  /* [B][gamma + 1] */
  float* o_draft;               /* [gamma][L][B][Hq][1][d] */
  float* o_verify;              /* [L][B][Hq][gamma + 1][d] */
  int32_t* n_plus_1;            /* [B] */
  int32_t* accepted;            /* [B][gamma + 1] */
} std_round_io;

/* Workspace bytes for std_decode_round (the larger of its attention calls). */
size_t std_round_workspace_size(const std_dims* dims, int gamma, int splits_draft,
                                int splits_verify);

/*
 * One draft + verify round ("Methodik" item 3), all on `stream`:
 *   for j < gamma: append draft row j to the sparse cache at len_sparse + j and
 *                  attend over len_sparse + j + 1 rows (one launch, as
 *                  std_sparse_decode_attn_append);
 *   append the gamma + 1 verify rows to the full cache at len_full;
 *   dense verify attention; acceptance; commit (lengths advance by n + 1).
 * The token ids of the LM head are inputs here (the language-model layers
 * around attention are not part of this library).
 */
int std_decode_round(const std_dims* dims, int gamma, const std_cache* cache,
                     const std_round_io* io, int splits_draft, int splits_verify, void* ws,
                     size_t ws_bytes, std_stream_t stream);

/* ---------------------------------------------------------------- test hook
 *
 * The selection kernels evaluate part of their exponentials with a polynomial
 * on the FP32 pipe instead of the special-function unit.  This hook runs both
 * on n device floats x (x <= 0): y_fma[i] = the polynomial 2^x[i], y_sfu[i] =
 * the special-function unit's 2^x[i], so tests can bound the polynomial's
 * error.  Not a step of the method. */
int std_probe_exp2(const float* x, float* y_fma, float* y_sfu, int n, std_stream_t stream);

/* Test hook for the failure path of the bounded waits.  Launches one CTA whose
 * thread 0 waits, through the same bounded mbarrier wait the tensor-core kernels
 * use, on a barrier that no thread ever arrives on.  The wait gives up after its
 * limit (0.5 s), sets STD_DEVERR_TIMEOUT in the device error word and the kernel
 * returns, so the context stays usable.  completed: one device int32, set to 0
 * when the wait gave up (1 would mean it completed).  Asynchronous on `stream`;
 * STD_ERR_INVALID_ARG for a NULL or unaligned `completed`.  Not a step of the
 * method. */
int std_probe_wait_timeout(int32_t* completed, std_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* STD_B200_H */
