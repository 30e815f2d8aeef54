// C ABI of the Sparse-to-Dense decoding library: argument checks, workspace
// sizing, launch configuration.  Declarations and the contract of every entry
// point are in include/std_b200.h.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <atomic>
#include <mutex>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "../../include/std_b200.h"
#include "internal.h"

namespace {

// An NVTX range around each entry point that launches work, named after it, so that a
// profiler timeline shows the library's calls (free when no tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
#define STD_NVTX_RANGE() NvtxRange nvtx_range_(__func__)

thread_local std::string g_last_error;
std::atomic<uint32_t> g_epoch{0};  // tags the in-kernel merge counters of each attention call

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int ok() {
  g_last_error.clear();
  return STD_OK;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(STD_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ---------------------------------------------------------------- per-device state
__device__ int g_device_error;  // OR of STD_DEVERR_* bits, one word per device

constexpr int kMaxDevices = 64;
std::mutex g_dev_mu;
int* g_err_ptr[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};

int current_device(int* dev) {
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (*dev < 0 || *dev >= kMaxDevices) return fail(STD_ERR_UNSUPPORTED, "device ordinal %d", *dev);
  return STD_OK;
}

int device_state(int** err_ptr, int* sm_count) {
  int dev;
  int rc = current_device(&dev);
  if (rc) return rc;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_device_error);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(device error word)");
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(SM count)");
    g_err_ptr[dev] = static_cast<int*>(p);
    g_sm_count[dev] = sms;
  }
  if (err_ptr) *err_ptr = g_err_ptr[dev];
  if (sm_count) *sm_count = g_sm_count[dev];
  return STD_OK;
}

// ---------------------------------------------------------------- checks
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int elem_bytes(int dtype) { return dtype == STD_F32 ? 4 : 2; }

int check_dims(const std_dims* d) {
  if (!d) return fail(STD_ERR_INVALID_ARG, "dims is NULL");
  if (d->L < 1 || d->B < 1 || d->Hq < 1 || d->Hkv < 1)
    return fail(STD_ERR_INVALID_ARG, "L, B, Hq, Hkv must be >= 1 (got %d, %d, %d, %d)", d->L, d->B, d->Hq, d->Hkv);
  if (d->Hq % d->Hkv) return fail(STD_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", d->Hq, d->Hkv);
  if (d->dtype == STD_BF16) {
    if (d->d != 64 && d->d != 128) return fail(STD_ERR_UNSUPPORTED, "bf16 head dim %d (supported: 64, 128)", d->d);
  } else if (d->dtype == STD_F32) {
    if (d->d != 32 && d->d != 64 && d->d != 96 && d->d != 128)
      return fail(STD_ERR_UNSUPPORTED, "fp32 head dim %d (supported: 32, 64, 96, 128)", d->d);
  } else {
    return fail(STD_ERR_UNSUPPORTED, "dtype %d", d->dtype);
  }
  if (d->cap_full < 1 || d->cap_sparse < 1) return fail(STD_ERR_INVALID_ARG, "capacities must be >= 1");
  if (d->cap_full > INT32_MAX || d->cap_sparse > INT32_MAX) return fail(STD_ERR_INVALID_ARG, "capacity above 2^31-1");
  return STD_OK;
}

int check_ptr(const void* p, size_t align, const char* name) {
  if (!p) return fail(STD_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned(p, align)) return fail(STD_ERR_INVALID_ARG, "%s is not %zu-byte aligned", name, align);
  return STD_OK;
}

#define STD_TRY(x)            \
  do {                        \
    int rc_ = (x);            \
    if (rc_ != STD_OK) return rc_; \
  } while (0)

int probs_of(const std_dims* d) { return d->L * d->B * d->Hkv; }

int auto_splits(int probs, int64_t cap, int sm_count) {
  // split-K kernels: about 8 CTAs per SM over the whole grid, at least 256 keys per split
  int s = (sm_count * 8 + probs - 1) / probs;
  const int64_t by_len = cap / 256;
  if (s > by_len) s = (int)by_len;
  if (s < 1) s = 1;
  if (s > 256) s = 256;
  return s;
}

// Launch plan of one decode-attention call: which kernel, how many splits / CTAs,
// how much workspace.  The same function sizes the workspace and runs the call.
struct AttnPlan {
  stdb::AttnArgs a;
  bool tc;
  size_t ws_bytes;
};

int plan_attn(const std_dims* dims, int nq, int64_t cap, int splits, AttnPlan* p, int early = 0) {
  if (splits < 0 || splits > 1024) return fail(STD_ERR_INVALID_ARG, "splits %d out of range [0, 1024]", splits);
  const int G = dims->Hq / dims->Hkv;
  stdb::AttnArgs& a = p->a;
  a = stdb::AttnArgs{};
  a.L = dims->L; a.B = dims->B; a.Hq = dims->Hq; a.Hkv = dims->Hkv; a.G = G; a.nq = nq; a.rows = G * nq;
  a.d = dims->d; a.dtype = dims->dtype; a.cap = cap;
  a.row_begin = 0; a.row_end = (int)cap;
  if (dims->dtype == STD_BF16 && a.rows > 128)
    return fail(STD_ERR_UNSUPPORTED, "G * query rows = %d exceeds 128", a.rows);
  const int probs = probs_of(dims);
  p->tc = stdb::attn_tc_supported(a);
  if (p->tc) {
    // keys-on-lanes kernel: CTAs cut problems into equal parts instead of stream-K ranges
    // wherever there are at most about as many CTAs as SMs (parts = 0: stream-K)
    const bool aligned = stdb::attn_tc_keys_on_lanes(a);
    int ctas = splits, parts = 0;
    if (splits > 0) {
      const int64_t want = (int64_t)splits * probs;
      ctas = (int)(want > 65535 ? 65535 : want);
      if (aligned && want <= 65535) parts = splits;
    } else {
      // One persistent CTA per SM (stream-K), unless the problems are short and nearly
      // fill the SMs: then one CTA per problem saves the segment partials and their merge,
      // which cost more than the SMs left idle.  Measured on a B200 (28 layers x 4 KV
      // heads, kernels timed alone): 7 query rows, 1024 keys 19.6 -> 14.7 us, 4352 keys
      // 48.6 -> 47.9 us but slower inside a decode step; 63 rows, 4352 keys 62.2 -> 50.4
      // us, 8192 keys 95.4 -> 85.9 us, 32768 keys 297 -> 328 us.  cap bounds the keys.
      // With an early start the SMs left idle are where the next kernel's CTAs start
      // early, so short-query calls take one CTA per problem up to 8192 keys too (the
      // long-video draft, 112 problems of 4353 keys: a chain of early-started steps 46.2 ->
      // 43.9 us per launch, 55.4 -> 53.7 us inside the decode step).  The workspace query,
      // which knows no flags, sizes for the larger grid.
      //
      // With few tiles in all (a single layer's draft: 4 problems of ~35 tiles), one CTA per
      // SM would cut every problem into dozens of one-tile segments whose partials the last
      // CTA merges; instead each problem gets a few CTAs.  The keys-on-lanes kernel cuts a
      // problem into equal parts of about kTilesPerPart tiles (a part fits the three K/V
      // stages, so with an early start all of it is fetched before the previous kernel
      // ends) and, up to 16 parts, merged inside a thread-block cluster.  28 launches of
      // one layer's draft, 4 x 4352 keys, in a CUDA graph, us per step without (with) an
      // early K/V start: 312 (276) with 12 parts in clusters, 328 (286) with 13, 324
      // (283) with 14, 330 (286) with 16, 377 (313) with 8; merged through global memory: 341 (276)
      // with 18 parts, 362 (287) with 16, 361 with 35 early; the other kernel
      // takes stream-K ranges of about kMinTilesPerCta tiles (the same launches, us per
      // launch: 25.8 with 148 CTAs, 17.9 with 48, 15.1 with 32, 18.0 with 24).
      int sms;
      STD_TRY(device_state(nullptr, &sms));
      const int64_t short_cap = a.rows <= 16 && !early ? 2048 : 8192;
      const int64_t nt_cap = (cap + 127) / 128;
      const int64_t tiles_max = (int64_t)probs * nt_cap;
      constexpr int64_t kMinTilesPerCta = 5;
      constexpr int64_t kTilesPerPart = 3;
      constexpr int64_t kMaxParts = 16;
      if (probs <= sms && 2 * probs >= sms && cap <= short_cap) {
        ctas = probs;
        parts = aligned ? 1 : 0;
      } else if (tiles_max < (int64_t)sms * kMinTilesPerCta) {
        if (aligned) {
          // at most half the SMs: the next launch's CTAs fit beside this one's and can
          // start early (the same launches with 19 parts, 76 CTAs: 322 us per step); at
          // most 16, so that a problem's parts form one thread-block cluster
          int64_t k = nt_cap / kTilesPerPart;  // parts of at least kTilesPerPart tiles at cap
          const int64_t k_fit = sms / (2 * (int64_t)probs);
          if (k > k_fit) k = k_fit;
          if (k > kMaxParts) k = kMaxParts;
          if (k < 1) k = 1;
          parts = (int)k;
          ctas = (int)(k * probs);
        } else {
          const int64_t c = (tiles_max + kMinTilesPerCta - 1) / kMinTilesPerCta;
          ctas = (int)(c < probs ? probs : c);
        }
      } else {
        ctas = sms;
      }
    }
    a.parts = parts;
    a.splits = ctas;
    p->ws_bytes = stdb::attn_tc_ws_floats(probs, ctas, a.rows, a.d) * sizeof(float);
  } else {
    int sp = splits;
    if (sp == 0) {
      int sms;
      STD_TRY(device_state(nullptr, &sms));
      sp = auto_splits(probs, cap, sms);
    }
    a.splits = sp;
    p->ws_bytes = stdb::attn_ws_floats(probs, sp, a.rows, a.d, a.dtype) * sizeof(float);
  }
  return STD_OK;
}

// Partials over a key range instead of the normalised output (tensor-core kernel only).
struct RangeOpt {
  int row_begin, row_end;
  float* ml;
};

// k_new / v_new (optional): rows to append to the cache at len[b] + new_off + r (r < new_rows)
// before attending -- inside the tensor-core kernel, else as a separate append launch.
int run_attn(const std_dims* dims, const void* q, const void* k, const void* v, int64_t cap,
             const int32_t* len, int len_off, int nq, float* o, int splits, void* ws, size_t ws_bytes,
             cudaStream_t stream, const void* k_new = nullptr, const void* v_new = nullptr, int new_rows = 0,
             int new_off = 0, int early = 0, const RangeOpt* range = nullptr) {
  AttnPlan p;
  STD_TRY(plan_attn(dims, nq, cap, splits, &p, early));
  if (range && !p.tc)
    return fail(STD_ERR_UNSUPPORTED, "key-range partials need the bf16 tensor-core kernel (d 64 or 128, "
                "G * query rows <= 128, at most 64 sequences)");
  if (p.ws_bytes > 0 && (!ws || ws_bytes < p.ws_bytes))
    return fail(STD_ERR_WORKSPACE, "attention workspace: need %zu bytes, got %zu", p.ws_bytes, ws ? ws_bytes : 0);
  if (p.ws_bytes > 0) STD_TRY(check_ptr(ws, 16, "ws"));
  int* err;
  STD_TRY(device_state(&err, nullptr));
  stdb::AttnArgs& a = p.a;
  a.q = q; a.k = k; a.v = v; a.o = o; a.len = len; a.len_off = len_off;
  a.ws = static_cast<float*>(ws); a.err = err;
  a.epoch = g_epoch.fetch_add(1, std::memory_order_relaxed) + 1;
  a.early = p.tc ? early : 0;
  if (range) {
    a.row_begin = range->row_begin;
    a.row_end = range->row_end;
    a.partial = 1;
    a.ml = range->ml;
  }
  if (k_new && new_rows > 0) {
    if (p.tc) {
      a.k_new = k_new; a.v_new = v_new; a.new_rows = new_rows; a.new_off = new_off;
    } else {
      cudaError_t e = stdb::launch_append(const_cast<void*>(k), const_cast<void*>(v), cap, len, new_off, k_new,
                                          v_new, new_rows, dims->L, dims->B, dims->Hkv,
                                          dims->d * elem_bytes(dims->dtype), err, stream);
      if (e != cudaSuccess) return cuda_fail(e, "append launch");
    }
  }
  cudaError_t e = p.tc ? stdb::launch_decode_attn_tc(a, stream) : stdb::launch_decode_attn(a, stream);
  if (e != cudaSuccess) return cuda_fail(e, "decode attention launch");
  return ok();
}

}  // namespace

namespace stdb {
std::atomic<unsigned long long> g_launch_count{0};
cudaError_t launch_probe_wait(int* err, int* completed, cudaStream_t s);  // probe.cu
}  // namespace stdb

extern "C" {

unsigned long long std_launch_count(void) { return stdb::g_launch_count.load(std::memory_order_relaxed); }

int std_version(void) { return 10000; }

const char* std_last_error(void) { return g_last_error.c_str(); }

int std_probe_wait_timeout(int32_t* completed, std_stream_t stream) {
  STD_NVTX_RANGE();
  STD_TRY(check_ptr(completed, 4, "completed"));
  int* err;
  STD_TRY(device_state(&err, nullptr));
  cudaError_t e = stdb::launch_probe_wait(err, completed, stream);
  if (e != cudaSuccess) return cuda_fail(e, "wait probe launch");
  return ok();
}

int std_get_device_error(int32_t* flags, int clear, std_stream_t stream) {
  STD_NVTX_RANGE();
  int* err;
  STD_TRY(device_state(&err, nullptr));
  int32_t host = 0;
  cudaError_t e = cudaMemcpyAsync(&host, err, sizeof(int32_t), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess && clear) e = cudaMemsetAsync(err, 0, sizeof(int32_t), stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  if (flags) *flags = host;
  if (host) return fail(STD_ERR_DEVICE, "device error flags 0x%x", host);
  return ok();
}

size_t std_select_workspace_size(const std_dims* dims, int T, int nvis_max) {
  if (check_dims(dims) || T < 1 || nvis_max < 1) return 0;
  const size_t probs = probs_of(dims);
  const size_t M = (size_t)(dims->Hq / dims->Hkv) * T;
  // row max and sum [probs][M] each, scores [probs][nvis_max], top-digit histograms [probs][256]
  return (probs * M * 2 + probs * (size_t)nvis_max + probs * 256) * sizeof(float) + 256;
}

int std_select_topk(const std_dims* dims, const void* q_text, int T, const void* k_full,
                    const void* v_full, const int32_t* nvis, int nvis_max, int K, int32_t* idx_out,
                    void* k_sparse, void* v_sparse, int32_t* len_sparse, float* scores_out, void* ws,
                    size_t ws_bytes, std_stream_t stream) {
  return std_select_topk_ex(dims, q_text, T, k_full, v_full, nvis, nvis_max, K, 0, 0, idx_out, k_sparse,
                            v_sparse, len_sparse, scores_out, ws, ws_bytes, stream);
}

int std_select_topk_ex(const std_dims* dims, const void* q_text, int T, const void* k_full,
                       const void* v_full, const int32_t* nvis, int nvis_max, int K, int n_prefix,
                       int flags, int32_t* idx_out, void* k_sparse, void* v_sparse, int32_t* len_sparse,
                       float* scores_out, void* ws, size_t ws_bytes, std_stream_t stream) {
  STD_NVTX_RANGE();
  STD_TRY(check_dims(dims));
  if (flags & ~STD_SELECT_CAUSAL_TEXT) return fail(STD_ERR_INVALID_ARG, "unknown selection flags %#x", flags);
  if (n_prefix < 0) return fail(STD_ERR_INVALID_ARG, "n_prefix = %d must be >= 0", n_prefix);
  STD_TRY(check_ptr(q_text, 16, "q_text"));
  STD_TRY(check_ptr(k_full, 16, "k_full"));
  STD_TRY(check_ptr(v_full, 16, "v_full"));
  STD_TRY(check_ptr(nvis, 4, "nvis"));
  STD_TRY(check_ptr(idx_out, 4, "idx_out"));
  STD_TRY(check_ptr(k_sparse, 16, "k_sparse"));
  STD_TRY(check_ptr(v_sparse, 16, "v_sparse"));
  STD_TRY(check_ptr(len_sparse, 4, "len_sparse"));
  if (scores_out) STD_TRY(check_ptr(scores_out, 4, "scores_out"));
  if (T < 1) return fail(STD_ERR_INVALID_ARG, "T = %d must be >= 1", T);
  if (nvis_max < 1) return fail(STD_ERR_INVALID_ARG, "nvis_max = %d must be >= 1", nvis_max);
  if (K < 1 || K > nvis_max) return fail(STD_ERR_INVALID_ARG, "K = %d must be in [1, nvis_max = %d]", K, nvis_max);
  if ((int64_t)n_prefix + K + T > dims->cap_sparse)
    return fail(STD_ERR_CAPACITY, "n_prefix + K + T = %lld exceeds cap_sparse = %lld", (long long)n_prefix + K + T,
                (long long)dims->cap_sparse);
  if ((int64_t)n_prefix + nvis_max + T > dims->cap_full)
    return fail(STD_ERR_CAPACITY, "n_prefix + nvis_max + T = %lld exceeds cap_full = %lld",
                (long long)n_prefix + nvis_max + T, (long long)dims->cap_full);
  const size_t need = std_select_workspace_size(dims, T, nvis_max);
  if (!ws || ws_bytes < need) return fail(STD_ERR_WORKSPACE, "select workspace: need %zu bytes, got %zu", need, ws ? ws_bytes : 0);
  STD_TRY(check_ptr(ws, 16, "ws"));
  int* err;
  STD_TRY(device_state(&err, nullptr));

  const int probs = probs_of(dims);
  const int G = dims->Hq / dims->Hkv;
  const size_t M = (size_t)G * T;
  float* row_m = static_cast<float*>(ws);
  float* row_l = row_m + probs * M;
  float* scores = scores_out ? scores_out : row_l + probs * M;
  uint32_t* hist = reinterpret_cast<uint32_t*>(row_l + probs * M + (size_t)probs * nvis_max);

  stdb::ScoreArgs s{};
  s.q_text = q_text; s.k_full = k_full; s.nvis = nvis; s.nvis_max = nvis_max;
  s.L = dims->L; s.B = dims->B; s.Hq = dims->Hq; s.Hkv = dims->Hkv; s.G = G; s.T = T; s.d = dims->d;
  s.dtype = dims->dtype; s.cap = dims->cap_full; s.row_m = row_m; s.row_l = row_l; s.scores = scores; s.err = err;
  s.causal_text = (flags & STD_SELECT_CAUSAL_TEXT) ? 1 : 0;
  s.prefix = n_prefix;
  s.hist = hist;
  bool hist_done = false;
  cudaError_t e = stdb::launch_select_scores(s, stream, &hist_done);
  if (e != cudaSuccess) return cuda_fail(e, "selection score launch");
  e = stdb::launch_topk(scores, nvis_max, probs, nvis, 0, dims->Hkv, dims->B, K, idx_out, hist_done ? hist : nullptr,
                        err, stream);
  if (e != cudaSuccess) return cuda_fail(e, "top-K launch");
  stdb::GatherArgs g{};
  g.k_full = k_full; g.v_full = v_full; g.k_sp = k_sparse; g.v_sp = v_sparse; g.idx = idx_out; g.nvis = nvis;
  g.len_sparse = len_sparse; g.L = dims->L; g.B = dims->B; g.Hkv = dims->Hkv; g.T = T; g.K = K;
  g.row_bytes = dims->d * elem_bytes(dims->dtype); g.cap_full = dims->cap_full; g.cap_sparse = dims->cap_sparse;
  g.prefix = n_prefix; g.err = err;
  e = stdb::launch_gather(g, stream);
  if (e != cudaSuccess) return cuda_fail(e, "gather launch");
  return ok();
}

// ---------------------------------------------------------------- selection over parts

namespace {

// Checks shared by the two score steps of a part; fills the score arguments.
int part_score_args(const std_dims* dims, const void* q_text, int T, const void* k_full, const int32_t* nvis,
                    int nvis_max, int n_prefix, stdb::ScoreArgs* s) {
  STD_TRY(check_dims(dims));
  STD_TRY(check_ptr(q_text, 16, "q_text"));
  STD_TRY(check_ptr(k_full, 16, "k_full"));
  STD_TRY(check_ptr(nvis, 4, "nvis"));
  if (T < 1) return fail(STD_ERR_INVALID_ARG, "T = %d must be >= 1", T);
  if (nvis_max < 1) return fail(STD_ERR_INVALID_ARG, "nvis_max = %d must be >= 1", nvis_max);
  if (n_prefix < 0) return fail(STD_ERR_INVALID_ARG, "n_prefix = %d must be >= 0", n_prefix);
  if ((int64_t)n_prefix + nvis_max > dims->cap_full)
    return fail(STD_ERR_CAPACITY, "n_prefix + nvis_max = %lld exceeds cap_full = %lld", (long long)n_prefix + nvis_max,
                (long long)dims->cap_full);
  *s = stdb::ScoreArgs{};
  s->q_text = q_text; s->k_full = k_full; s->nvis = nvis; s->nvis_max = nvis_max;
  s->L = dims->L; s->B = dims->B; s->Hq = dims->Hq; s->Hkv = dims->Hkv; s->G = dims->Hq / dims->Hkv; s->T = T;
  s->d = dims->d; s->dtype = dims->dtype; s->cap = dims->cap_full; s->prefix = n_prefix;
  s->keys_only = 1;
  return STD_OK;  // s->err is set by the caller once every host check has passed
}

}  // namespace

int std_select_rowstats(const std_dims* dims, const void* q_text, int T, const void* k_full, const int32_t* nvis,
                        int nvis_max, int n_prefix, float* row_m, float* row_l, std_stream_t stream) {
  STD_NVTX_RANGE();
  stdb::ScoreArgs s;
  STD_TRY(part_score_args(dims, q_text, T, k_full, nvis, nvis_max, n_prefix, &s));
  STD_TRY(check_ptr(row_m, 4, "row_m"));
  STD_TRY(check_ptr(row_l, 4, "row_l"));
  STD_TRY(device_state(&s.err, nullptr));
  s.row_m = row_m; s.row_l = row_l; s.passes = 1;
  bool hist_done = false;
  cudaError_t e = stdb::launch_select_scores(s, stream, &hist_done);
  if (e != cudaSuccess) return cuda_fail(e, "selection row-statistics launch");
  return ok();
}

int std_merge_rowstats(int64_t n, int n_parts, const float* m_parts, const float* l_parts, float* row_m, float* row_l,
                       std_stream_t stream) {
  STD_NVTX_RANGE();
  if (n < 1) return fail(STD_ERR_INVALID_ARG, "n = %lld must be >= 1", (long long)n);
  if (n_parts < 1) return fail(STD_ERR_INVALID_ARG, "n_parts = %d must be >= 1", n_parts);
  STD_TRY(check_ptr(m_parts, 4, "m_parts"));
  STD_TRY(check_ptr(l_parts, 4, "l_parts"));
  STD_TRY(check_ptr(row_m, 4, "row_m"));
  STD_TRY(check_ptr(row_l, 4, "row_l"));
  STD_TRY(device_state(nullptr, nullptr));
  cudaError_t e = stdb::launch_merge_rowstats(m_parts, l_parts, n_parts, n, row_m, row_l, stream);
  if (e != cudaSuccess) return cuda_fail(e, "row-statistics merge launch");
  return ok();
}

size_t std_select_candidates_workspace_size(const std_dims* dims, int nvis_max) {
  if (check_dims(dims) || nvis_max < 1) return 0;
  return (size_t)probs_of(dims) * nvis_max * sizeof(float) + 256;
}

int std_select_candidates(const std_dims* dims, const void* q_text, int T, const void* k_full, const int32_t* nvis,
                          int nvis_max, int n_prefix, const float* row_m, const float* row_l, int K,
                          int32_t* cand_idx, float* cand_score, float* scores_out, void* ws, size_t ws_bytes,
                          std_stream_t stream) {
  STD_NVTX_RANGE();
  stdb::ScoreArgs s;
  STD_TRY(part_score_args(dims, q_text, T, k_full, nvis, nvis_max, n_prefix, &s));
  STD_TRY(check_ptr(row_m, 4, "row_m"));
  STD_TRY(check_ptr(row_l, 4, "row_l"));
  STD_TRY(check_ptr(cand_idx, 4, "cand_idx"));
  STD_TRY(check_ptr(cand_score, 4, "cand_score"));
  if (scores_out) STD_TRY(check_ptr(scores_out, 4, "scores_out"));
  if (K < 1 || K > nvis_max) return fail(STD_ERR_INVALID_ARG, "K = %d must be in [1, nvis_max = %d]", K, nvis_max);
  const size_t need = std_select_candidates_workspace_size(dims, nvis_max);
  if (!scores_out && (!ws || ws_bytes < need))
    return fail(STD_ERR_WORKSPACE, "candidate workspace: need %zu bytes, got %zu", need, ws ? ws_bytes : 0);
  if (!scores_out) STD_TRY(check_ptr(ws, 16, "ws"));
  STD_TRY(device_state(&s.err, nullptr));
  float* scores = scores_out ? scores_out : static_cast<float*>(ws);
  s.row_m = const_cast<float*>(row_m); s.row_l = const_cast<float*>(row_l); s.scores = scores; s.passes = 2;
  bool hist_done = false;
  cudaError_t e = stdb::launch_select_scores(s, stream, &hist_done);
  if (e != cudaSuccess) return cuda_fail(e, "selection score launch");
  const int probs = probs_of(dims);
  e = stdb::launch_topk(scores, nvis_max, probs, nvis, 0, dims->Hkv, dims->B, K, cand_idx, nullptr, s.err, stream);
  if (e != cudaSuccess) return cuda_fail(e, "top-K launch");
  e = stdb::launch_candidate_scores(scores, nvis_max, cand_idx, probs, K, cand_score, stream);
  if (e != cudaSuccess) return cuda_fail(e, "candidate score launch");
  return ok();
}

size_t std_merge_candidates_workspace_size(const std_dims* dims, int n_parts, int K) {
  if (check_dims(dims) || n_parts < 1 || K < 1) return 0;
  // the candidates' scores per problem in part order, then the chosen positions
  return (size_t)probs_of(dims) * ((size_t)n_parts * K * sizeof(float) + (size_t)K * sizeof(int32_t)) + 512;
}

int std_merge_candidates(const std_dims* dims, int n_parts, int K, const int32_t* cand_idx, const float* cand_score,
                         const int32_t* part_offset, int32_t* idx_out, void* ws, size_t ws_bytes,
                         std_stream_t stream) {
  STD_NVTX_RANGE();
  STD_TRY(check_dims(dims));
  if (n_parts < 1) return fail(STD_ERR_INVALID_ARG, "n_parts = %d must be >= 1", n_parts);
  if (K < 1) return fail(STD_ERR_INVALID_ARG, "K = %d must be >= 1", K);
  if ((int64_t)n_parts * K > (1 << 30)) return fail(STD_ERR_INVALID_ARG, "n_parts * K too large");
  STD_TRY(check_ptr(cand_idx, 4, "cand_idx"));
  STD_TRY(check_ptr(cand_score, 4, "cand_score"));
  STD_TRY(check_ptr(part_offset, 4, "part_offset"));
  STD_TRY(check_ptr(idx_out, 4, "idx_out"));
  const size_t need = std_merge_candidates_workspace_size(dims, n_parts, K);
  if (!ws || ws_bytes < need)
    return fail(STD_ERR_WORKSPACE, "candidate merge workspace: need %zu bytes, got %zu", need, ws ? ws_bytes : 0);
  STD_TRY(check_ptr(ws, 16, "ws"));
  int* err;
  STD_TRY(device_state(&err, nullptr));
  const int probs = probs_of(dims);
  float* cat = static_cast<float*>(ws);
  int32_t* pos = reinterpret_cast<int32_t*>(cat + (size_t)probs * n_parts * K);
  cudaError_t e = stdb::launch_concat_candidates(cand_score, n_parts, probs, K, cat, stream);
  if (e != cudaSuccess) return cuda_fail(e, "candidate layout launch");
  e = stdb::launch_topk(cat, (int64_t)n_parts * K, probs, nullptr, n_parts * K, 1, 1, K, pos, nullptr, err, stream);
  if (e != cudaSuccess) return cuda_fail(e, "top-K launch");
  e = stdb::launch_map_candidates(pos, cand_idx, part_offset, n_parts, probs, K, dims->B, dims->Hkv, idx_out, err,
                                  stream);
  if (e != cudaSuccess) return cuda_fail(e, "candidate index launch");
  return ok();
}

int std_gather_sparse_part(const std_dims* dims, const void* k_full, const void* v_full, const int32_t* nvis,
                           const int32_t* idx, int K, int T, int n_prefix, int64_t part_pos0, int64_t part_rows,
                           void* k_sparse, void* v_sparse, int32_t* len_sparse, std_stream_t stream) {
  STD_NVTX_RANGE();
  STD_TRY(check_dims(dims));
  STD_TRY(check_ptr(k_full, 16, "k_full"));
  STD_TRY(check_ptr(v_full, 16, "v_full"));
  STD_TRY(check_ptr(nvis, 4, "nvis"));
  STD_TRY(check_ptr(idx, 4, "idx"));
  STD_TRY(check_ptr(k_sparse, 16, "k_sparse"));
  STD_TRY(check_ptr(v_sparse, 16, "v_sparse"));
  STD_TRY(check_ptr(len_sparse, 4, "len_sparse"));
  if (K < 1 || T < 0 || n_prefix < 0) return fail(STD_ERR_INVALID_ARG, "need K >= 1, T >= 0, n_prefix >= 0");
  if (part_pos0 < 0 || part_rows < 1 || part_rows > dims->cap_full)
    return fail(STD_ERR_INVALID_ARG, "part [%lld, +%lld) must be non-empty and fit cap_full = %lld",
                (long long)part_pos0, (long long)part_rows, (long long)dims->cap_full);
  if ((int64_t)n_prefix + K + T > dims->cap_sparse)
    return fail(STD_ERR_CAPACITY, "n_prefix + K + T = %lld exceeds cap_sparse = %lld", (long long)n_prefix + K + T,
                (long long)dims->cap_sparse);
  int* err;
  STD_TRY(device_state(&err, nullptr));
  stdb::GatherArgs g{};
  g.k_full = k_full; g.v_full = v_full; g.k_sp = k_sparse; g.v_sp = v_sparse; g.idx = idx; g.nvis = nvis;
  g.len_sparse = len_sparse; g.L = dims->L; g.B = dims->B; g.Hkv = dims->Hkv; g.T = T; g.K = K;
  g.row_bytes = dims->d * elem_bytes(dims->dtype); g.cap_full = dims->cap_full; g.cap_sparse = dims->cap_sparse;
  g.prefix = n_prefix; g.err = err; g.part_pos0 = part_pos0; g.part_rows = part_rows;
  cudaError_t e = stdb::launch_gather(g, stream);
  if (e != cudaSuccess) return cuda_fail(e, "gather launch");
  return ok();
}

int std_streaming_indices(const std_dims* dims, const int32_t* nvis, int K, int n_sink, int32_t* idx_out,
                          std_stream_t stream) {
  STD_NVTX_RANGE();
  STD_TRY(check_dims(dims));
  STD_TRY(check_ptr(nvis, 4, "nvis"));
  STD_TRY(check_ptr(idx_out, 4, "idx_out"));
  if (K < 1) return fail(STD_ERR_INVALID_ARG, "K = %d must be >= 1", K);
  if (n_sink < 0 || n_sink > K) return fail(STD_ERR_INVALID_ARG, "n_sink = %d must be in [0, K = %d]", n_sink, K);
  int* err;
  STD_TRY(device_state(&err, nullptr));
  cudaError_t e = stdb::launch_streaming_indices(nvis, dims->L, dims->B, dims->Hkv, K, n_sink, idx_out, err, stream);
  if (e != cudaSuccess) return cuda_fail(e, "streaming index launch");
  return ok();
}

int std_gather_sparse(const std_dims* dims, const void* k_full, const void* v_full, const int32_t* nvis,
                      const int32_t* idx, int K, int T, int n_prefix, void* k_sparse, void* v_sparse,
                      int32_t* len_sparse, std_stream_t stream) {
  STD_NVTX_RANGE();
  STD_TRY(check_dims(dims));
  STD_TRY(check_ptr(k_full, 16, "k_full"));
  STD_TRY(check_ptr(v_full, 16, "v_full"));
  STD_TRY(check_ptr(nvis, 4, "nvis"));
  STD_TRY(check_ptr(idx, 4, "idx"));
  STD_TRY(check_ptr(k_sparse, 16, "k_sparse"));
  STD_TRY(check_ptr(v_sparse, 16, "v_sparse"));
  STD_TRY(check_ptr(len_sparse, 4, "len_sparse"));
  if (K < 1 || T < 0 || n_prefix < 0) return fail(STD_ERR_INVALID_ARG, "K = %d, T = %d, n_prefix = %d", K, T, n_prefix);
  if ((int64_t)n_prefix + K + T > dims->cap_sparse)
    return fail(STD_ERR_CAPACITY, "n_prefix + K + T = %lld exceeds cap_sparse = %lld", (long long)n_prefix + K + T,
                (long long)dims->cap_sparse);
  int* err;
  STD_TRY(device_state(&err, nullptr));
  stdb::GatherArgs g{};
  g.k_full = k_full; g.v_full = v_full; g.k_sp = k_sparse; g.v_sp = v_sparse; g.idx = idx; g.nvis = nvis;
  g.len_sparse = len_sparse; g.L = dims->L; g.B = dims->B; g.Hkv = dims->Hkv; g.T = T; g.K = K;
  g.row_bytes = dims->d * elem_bytes(dims->dtype); g.cap_full = dims->cap_full; g.cap_sparse = dims->cap_sparse;
  g.prefix = n_prefix; g.err = err;
  cudaError_t e = stdb::launch_gather(g, stream);
  if (e != cudaSuccess) return cuda_fail(e, "gather launch");
  return ok();
}

int std_topk_from_scores(const float* scores, int rows, int n, int K, int32_t* idx_out, std_stream_t stream) {
  STD_NVTX_RANGE();
  STD_TRY(check_ptr(scores, 4, "scores"));
  STD_TRY(check_ptr(idx_out, 4, "idx_out"));
  if (rows < 0 || n < 1) return fail(STD_ERR_INVALID_ARG, "rows = %d, n = %d", rows, n);
  if (K < 1 || K > n) return fail(STD_ERR_INVALID_ARG, "K = %d must be in [1, n = %d]", K, n);
  int* err;
  STD_TRY(device_state(&err, nullptr));
  cudaError_t e = stdb::launch_topk(scores, n, rows, nullptr, n, 1, 1, K, idx_out, nullptr, err, stream);
  if (e != cudaSuccess) return cuda_fail(e, "top-K launch");
  return ok();
}

size_t std_attn_workspace_size(const std_dims* dims, int q_rows, int64_t cap, int splits) {
  if (check_dims(dims) || q_rows < 1 || cap < 1) return 0;
  AttnPlan p;
  if (plan_attn(dims, q_rows, cap, splits, &p)) return 0;
  return p.ws_bytes;
}

int std_attn_splits_ex(const std_dims* dims, int q_rows, int64_t cap, int splits, int flags) {
  STD_TRY(check_dims(dims));
  if (cap < 1 || q_rows < 1) return fail(STD_ERR_INVALID_ARG, "cap = %lld, q_rows = %d", (long long)cap, q_rows);
  if (flags & ~(STD_ATTN_EARLY_KV | STD_ATTN_EARLY_Q))
    return fail(STD_ERR_INVALID_ARG, "unknown attention flags %#x", flags);
  if ((flags & STD_ATTN_EARLY_Q) && !(flags & STD_ATTN_EARLY_KV))
    return fail(STD_ERR_INVALID_ARG, "STD_ATTN_EARLY_Q needs STD_ATTN_EARLY_KV");
  AttnPlan p;
  STD_TRY(plan_attn(dims, q_rows, cap, splits, &p, flags));
  ok();
  return p.a.splits;
}

int std_attn_splits(const std_dims* dims, int q_rows, int64_t cap, int splits) {
  return std_attn_splits_ex(dims, q_rows, cap, splits, 0);
}

int std_sparse_decode_attn(const std_dims* dims, const void* q, const void* k_sparse, const void* v_sparse,
                           const int32_t* len_sparse, int len_offset, float* o, int splits, void* ws,
                           size_t ws_bytes, std_stream_t stream) {
  STD_NVTX_RANGE();
  STD_TRY(check_dims(dims));
  STD_TRY(check_ptr(q, 16, "q"));
  STD_TRY(check_ptr(k_sparse, 16, "k_sparse"));
  STD_TRY(check_ptr(v_sparse, 16, "v_sparse"));
  STD_TRY(check_ptr(len_sparse, 4, "len_sparse"));
  STD_TRY(check_ptr(o, 16, "o"));
  if (len_offset < 0) return fail(STD_ERR_INVALID_ARG, "len_offset = %d must be >= 0", len_offset);
  return run_attn(dims, q, k_sparse, v_sparse, dims->cap_sparse, len_sparse, len_offset, 1, o, splits, ws,
                  ws_bytes, stream);
}

int std_dense_verify_attn(const std_dims* dims, const void* q, int gamma, const void* k_full, const void* v_full,
                          const int32_t* len_full, float* o, int splits, void* ws, size_t ws_bytes,
                          std_stream_t stream) {
  STD_NVTX_RANGE();
  STD_TRY(check_dims(dims));
  STD_TRY(check_ptr(q, 16, "q"));
  STD_TRY(check_ptr(k_full, 16, "k_full"));
  STD_TRY(check_ptr(v_full, 16, "v_full"));
  STD_TRY(check_ptr(len_full, 4, "len_full"));
  STD_TRY(check_ptr(o, 16, "o"));
  if (gamma < 0 || gamma > 31) return fail(STD_ERR_INVALID_ARG, "gamma = %d must be in [0, 31]", gamma);
  // row i sees keys j < len_full + 1 + i
  return run_attn(dims, q, k_full, v_full, dims->cap_full, len_full, 1, gamma + 1, o, splits, ws, ws_bytes,
                  stream);
}

// Shared checks of the key-range calls: the range lies in the buffer, and the shift of the
// causal limit by pos0 fits the kernel's int arithmetic.
static int check_range(int64_t pos0, int64_t row_begin, int64_t row_end, int64_t cap, const float* o_part,
                       const float* ml_part) {
  STD_TRY(check_ptr(o_part, 16, "o_part"));
  STD_TRY(check_ptr(ml_part, 8, "ml_part"));
  if (pos0 < 0 || pos0 > (1 << 30))
    return fail(STD_ERR_INVALID_ARG, "pos0 = %lld must be in [0, 2^30]", (long long)pos0);
  if (row_begin < 0 || row_begin > row_end || row_end > cap)
    return fail(STD_ERR_INVALID_ARG, "rows [%lld, %lld) must satisfy 0 <= row_begin <= row_end <= cap = %lld",
                (long long)row_begin, (long long)row_end, (long long)cap);
  return STD_OK;
}

int std_dense_verify_attn_partial(const std_dims* dims, const void* q, int gamma, const void* k_full,
                                  const void* v_full, const int32_t* len_full, int64_t pos0, int64_t row_begin,
                                  int64_t row_end, float* o_part, float* ml_part, int splits, void* ws,
                                  size_t ws_bytes, std_stream_t stream) {
  STD_NVTX_RANGE();
  STD_TRY(check_dims(dims));
  STD_TRY(check_ptr(q, 16, "q"));
  STD_TRY(check_ptr(k_full, 16, "k_full"));
  STD_TRY(check_ptr(v_full, 16, "v_full"));
  STD_TRY(check_ptr(len_full, 4, "len_full"));
  if (gamma < 0 || gamma > 31) return fail(STD_ERR_INVALID_ARG, "gamma = %d must be in [0, 31]", gamma);
  STD_TRY(check_range(pos0, row_begin, row_end, dims->cap_full, o_part, ml_part));
  const RangeOpt rg{(int)row_begin, (int)row_end, ml_part};
  // row i sees positions j < len_full + 1 + i, i.e. buffer rows r < len_full + 1 - pos0 + i
  return run_attn(dims, q, k_full, v_full, dims->cap_full, len_full, 1 - (int)pos0, gamma + 1, o_part, splits, ws,
                  ws_bytes, stream, nullptr, nullptr, 0, 0, 0, &rg);
}

int std_sparse_decode_attn_partial(const std_dims* dims, const void* q, const void* k_sparse, const void* v_sparse,
                                   const int32_t* len_sparse, int len_offset, int64_t pos0, int64_t row_begin,
                                   int64_t row_end, float* o_part, float* ml_part, int splits, void* ws,
                                   size_t ws_bytes, std_stream_t stream) {
  STD_NVTX_RANGE();
  STD_TRY(check_dims(dims));
  STD_TRY(check_ptr(q, 16, "q"));
  STD_TRY(check_ptr(k_sparse, 16, "k_sparse"));
  STD_TRY(check_ptr(v_sparse, 16, "v_sparse"));
  STD_TRY(check_ptr(len_sparse, 4, "len_sparse"));
  if (len_offset < 0 || len_offset > (1 << 30))
    return fail(STD_ERR_INVALID_ARG, "len_offset = %d must be in [0, 2^30]", len_offset);
  STD_TRY(check_range(pos0, row_begin, row_end, dims->cap_sparse, o_part, ml_part));
  const RangeOpt rg{(int)row_begin, (int)row_end, ml_part};
  return run_attn(dims, q, k_sparse, v_sparse, dims->cap_sparse, len_sparse, len_offset - (int)pos0, 1, o_part,
                  splits, ws, ws_bytes, stream, nullptr, nullptr, 0, 0, 0, &rg);
}

int std_merge_partials(int64_t rows, int d, int n_parts, const float* o_parts, const float* ml_parts, float* o,
                       std_stream_t stream) {
  STD_NVTX_RANGE();
  if (rows < 0) return fail(STD_ERR_INVALID_ARG, "rows = %lld must be >= 0", (long long)rows);
  if (d < 4 || d % 4) return fail(STD_ERR_INVALID_ARG, "d = %d must be a positive multiple of 4", d);
  if (n_parts < 1) return fail(STD_ERR_INVALID_ARG, "n_parts = %d must be >= 1", n_parts);
  if (rows == 0) return ok();
  STD_TRY(check_ptr(o_parts, 16, "o_parts"));
  STD_TRY(check_ptr(ml_parts, 8, "ml_parts"));
  STD_TRY(check_ptr(o, 16, "o"));
  int sms;
  STD_TRY(device_state(nullptr, &sms));
  cudaError_t e = stdb::launch_merge_partials(rows, d, n_parts, o_parts, ml_parts, o, sms, stream);
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  return ok();
}

int std_accept_prefix(int B, int gamma, const int32_t* draft, const int32_t* dense_argmax, int32_t* n_plus_1,
                      int32_t* accepted, std_stream_t stream) {
  STD_NVTX_RANGE();
  if (B < 1) return fail(STD_ERR_INVALID_ARG, "B = %d must be >= 1", B);
  if (gamma < 0 || gamma > 31) return fail(STD_ERR_INVALID_ARG, "gamma = %d must be in [0, 31]", gamma);
  if (gamma > 0) STD_TRY(check_ptr(draft, 4, "draft"));
  STD_TRY(check_ptr(dense_argmax, 4, "dense_argmax"));
  STD_TRY(check_ptr(n_plus_1, 4, "n_plus_1"));
  STD_TRY(check_ptr(accepted, 4, "accepted"));
  cudaError_t e = stdb::launch_accept(B, gamma, draft, dense_argmax, n_plus_1, accepted, stream);
  if (e != cudaSuccess) return cuda_fail(e, "accept launch");
  return ok();
}

int std_sparse_decode_attn_append(const std_dims* dims, const void* q, void* k_sparse, void* v_sparse,
                                  const int32_t* len_sparse, int len_offset, const void* k_new, const void* v_new,
                                  float* o, int splits, void* ws, size_t ws_bytes, std_stream_t stream) {
  return std_sparse_decode_attn_append_ex(dims, q, k_sparse, v_sparse, len_sparse, len_offset, k_new, v_new, o, splits,
                                          0, ws, ws_bytes, stream);
}

int std_sparse_decode_attn_append_ex(const std_dims* dims, const void* q, void* k_sparse, void* v_sparse,
                                     const int32_t* len_sparse, int len_offset, const void* k_new,
                                     const void* v_new, float* o, int splits, int flags, void* ws, size_t ws_bytes,
                                     std_stream_t stream) {
  STD_NVTX_RANGE();
  if (flags & ~(STD_ATTN_EARLY_KV | STD_ATTN_EARLY_Q))
    return fail(STD_ERR_INVALID_ARG, "unknown attention flags %#x", flags);
  if ((flags & STD_ATTN_EARLY_Q) && !(flags & STD_ATTN_EARLY_KV))
    return fail(STD_ERR_INVALID_ARG, "STD_ATTN_EARLY_Q needs STD_ATTN_EARLY_KV");
  STD_TRY(check_dims(dims));
  STD_TRY(check_ptr(q, 16, "q"));
  STD_TRY(check_ptr(k_sparse, 16, "k_sparse"));
  STD_TRY(check_ptr(v_sparse, 16, "v_sparse"));
  STD_TRY(check_ptr(len_sparse, 4, "len_sparse"));
  STD_TRY(check_ptr(k_new, 16, "k_new"));
  STD_TRY(check_ptr(v_new, 16, "v_new"));
  STD_TRY(check_ptr(o, 16, "o"));
  if (len_offset < 1) return fail(STD_ERR_INVALID_ARG, "len_offset = %d must be >= 1 (it counts the new row)", len_offset);
  if ((int64_t)len_offset > dims->cap_sparse) return fail(STD_ERR_CAPACITY, "len_offset exceeds cap_sparse");
  return run_attn(dims, q, k_sparse, v_sparse, dims->cap_sparse, len_sparse, len_offset, 1, o, splits, ws,
                  ws_bytes, stream, k_new, v_new, 1, len_offset - 1, flags);
}

int std_dense_verify_attn_append(const std_dims* dims, const void* q, int gamma, void* k_full, void* v_full,
                                 const int32_t* len_full, const void* k_new, const void* v_new, float* o, int splits,
                                 void* ws, size_t ws_bytes, std_stream_t stream) {
  STD_NVTX_RANGE();
  STD_TRY(check_dims(dims));
  STD_TRY(check_ptr(q, 16, "q"));
  STD_TRY(check_ptr(k_full, 16, "k_full"));
  STD_TRY(check_ptr(v_full, 16, "v_full"));
  STD_TRY(check_ptr(len_full, 4, "len_full"));
  STD_TRY(check_ptr(k_new, 16, "k_new"));
  STD_TRY(check_ptr(v_new, 16, "v_new"));
  STD_TRY(check_ptr(o, 16, "o"));
  if (gamma < 0 || gamma > 31) return fail(STD_ERR_INVALID_ARG, "gamma = %d must be in [0, 31]", gamma);
  if ((int64_t)gamma + 1 > dims->cap_full) return fail(STD_ERR_CAPACITY, "gamma + 1 exceeds cap_full");
  return run_attn(dims, q, k_full, v_full, dims->cap_full, len_full, 1, gamma + 1, o, splits, ws, ws_bytes, stream,
                  k_new, v_new, gamma + 1, 0);
}

int std_kv_append(const std_dims* dims, void* k_cache, void* v_cache, int64_t cap, const int32_t* len,
                  int pos_offset, const void* k_new, const void* v_new, int n_new, std_stream_t stream) {
  STD_NVTX_RANGE();
  STD_TRY(check_dims(dims));
  STD_TRY(check_ptr(k_cache, 16, "k_cache"));
  STD_TRY(check_ptr(v_cache, 16, "v_cache"));
  STD_TRY(check_ptr(len, 4, "len"));
  STD_TRY(check_ptr(k_new, 16, "k_new"));
  STD_TRY(check_ptr(v_new, 16, "v_new"));
  if (cap < 1 || cap > INT32_MAX) return fail(STD_ERR_INVALID_ARG, "cap = %lld", (long long)cap);
  if (n_new < 0 || pos_offset < 0) return fail(STD_ERR_INVALID_ARG, "n_new = %d, pos_offset = %d", n_new, pos_offset);
  if ((int64_t)n_new + pos_offset > cap) return fail(STD_ERR_CAPACITY, "offset + rows exceed cap");
  int* err;
  STD_TRY(device_state(&err, nullptr));
  cudaError_t e = stdb::launch_append(k_cache, v_cache, cap, len, pos_offset, k_new, v_new, n_new, dims->L,
                                      dims->B, dims->Hkv, dims->d * elem_bytes(dims->dtype), err, stream);
  if (e != cudaSuccess) return cuda_fail(e, "append launch");
  return ok();
}

int std_kv_commit(const std_dims* dims, void* k_full, void* v_full, void* k_sparse, void* v_sparse,
                  int32_t* len_full, int32_t* len_sparse, const int32_t* n_plus_1, int max_n,
                  std_stream_t stream) {
  STD_NVTX_RANGE();
  STD_TRY(check_dims(dims));
  STD_TRY(check_ptr(k_full, 16, "k_full"));
  STD_TRY(check_ptr(v_full, 16, "v_full"));
  STD_TRY(check_ptr(k_sparse, 16, "k_sparse"));
  STD_TRY(check_ptr(v_sparse, 16, "v_sparse"));
  STD_TRY(check_ptr(len_full, 4, "len_full"));
  STD_TRY(check_ptr(len_sparse, 4, "len_sparse"));
  STD_TRY(check_ptr(n_plus_1, 4, "n_plus_1"));
  if (max_n < 1 || max_n > 32) return fail(STD_ERR_INVALID_ARG, "max_n = %d must be in [1, 32]", max_n);
  int* err;
  STD_TRY(device_state(&err, nullptr));
  cudaError_t e = stdb::launch_commit(k_full, v_full, k_sparse, v_sparse, len_full, len_sparse, n_plus_1, max_n,
                                      dims->L, dims->B, dims->Hkv, dims->d * elem_bytes(dims->dtype),
                                      dims->cap_full, dims->cap_sparse, err, stream);
  if (e != cudaSuccess) return cuda_fail(e, "commit launch");
  return ok();
}

size_t std_round_workspace_size(const std_dims* dims, int gamma, int splits_draft, int splits_verify) {
  if (check_dims(dims) || gamma < 0 || gamma > 31) return 0;
  const size_t a = gamma > 0 ? std_attn_workspace_size(dims, 1, dims->cap_sparse, splits_draft) : 0;
  const size_t b = std_attn_workspace_size(dims, gamma + 1, dims->cap_full, splits_verify);
  return a > b ? a : b;
}

int std_decode_round(const std_dims* dims, int gamma, const std_cache* c, const std_round_io* io,
                     int splits_draft, int splits_verify, void* ws, size_t ws_bytes, std_stream_t stream) {
  STD_NVTX_RANGE();
  STD_TRY(check_dims(dims));
  if (!c || !io) return fail(STD_ERR_INVALID_ARG, "cache or io is NULL");
  if (gamma < 0 || gamma > 31) return fail(STD_ERR_INVALID_ARG, "gamma = %d must be in [0, 31]", gamma);
  const size_t eb = elem_bytes(dims->dtype);
  const size_t q_step = (size_t)dims->L * dims->B * dims->Hq * dims->d;   // elements per draft query step
  const size_t kv_step = (size_t)dims->L * dims->B * dims->Hkv * dims->d;  // elements per draft K/V step
  const void* ptrs[] = {c->k_full, c->v_full, c->k_sparse, c->v_sparse, io->q_draft, io->k_draft, io->v_draft,
                        io->q_verify, io->k_verify, io->v_verify, io->o_draft, io->o_verify};
  for (const void* ptr : ptrs)
    if (gamma > 0 || (ptr != io->q_draft && ptr != io->k_draft && ptr != io->v_draft && ptr != io->o_draft))
      STD_TRY(check_ptr(ptr, 16, "round buffer"));
  STD_TRY(check_ptr(c->len_full, 4, "len_full"));
  STD_TRY(check_ptr(c->len_sparse, 4, "len_sparse"));
  if (gamma > dims->cap_sparse || gamma + 1 > dims->cap_full) return fail(STD_ERR_CAPACITY, "gamma exceeds a cache");
  {  // both attention plans and the workspace are checked before anything is launched
    AttnPlan pd, pv;
    size_t need = 0;
    if (gamma > 0) {
      STD_TRY(plan_attn(dims, 1, dims->cap_sparse, splits_draft, &pd));
      need = pd.ws_bytes;
    }
    STD_TRY(plan_attn(dims, gamma + 1, dims->cap_full, splits_verify, &pv));
    if (pv.ws_bytes > need) need = pv.ws_bytes;
    if (need > 0 && (!ws || ws_bytes < need))
      return fail(STD_ERR_WORKSPACE, "round workspace: need %zu bytes, got %zu", need, ws ? ws_bytes : 0);
  }
  // draft step j: append its input's K/V row at len_sparse + j, attend over len_sparse + j + 1 rows.
  // Steps j > 0 follow step j - 1, which writes only its output, its partials and sparse row
  // len_sparse + j - 1, and reads inputs all queued before this call: they start early.
  for (int j = 0; j < gamma; ++j) {
    STD_TRY(run_attn(dims, static_cast<const uint8_t*>(io->q_draft) + j * q_step * eb, c->k_sparse, c->v_sparse,
                     dims->cap_sparse, c->len_sparse, j + 1, 1, io->o_draft + j * q_step, splits_draft, ws, ws_bytes,
                     stream, static_cast<const uint8_t*>(io->k_draft) + j * kv_step * eb,
                     static_cast<const uint8_t*>(io->v_draft) + j * kv_step * eb, 1, j,
                     j > 0 ? STD_ATTN_EARLY_KV | STD_ATTN_EARLY_Q : 0));
  }
  // verify: append the gamma + 1 rows at len_full (a separate launch: fused into the verify
  // kernel it measured ~1% slower on the long-video step, fused into the draft faster), then
  // row i attends over len_full + i + 1 rows
  STD_TRY(std_kv_append(dims, c->k_full, c->v_full, dims->cap_full, c->len_full, 0, io->k_verify, io->v_verify,
                        gamma + 1, stream));
  STD_TRY(run_attn(dims, io->q_verify, c->k_full, c->v_full, dims->cap_full, c->len_full, 1, gamma + 1, io->o_verify,
                   splits_verify, ws, ws_bytes, stream));
  STD_TRY(std_accept_prefix(dims->B, gamma, io->draft_tokens, io->dense_tokens, io->n_plus_1, io->accepted,
                            stream));
  STD_TRY(std_kv_commit(dims, c->k_full, c->v_full, c->k_sparse, c->v_sparse, c->len_full, c->len_sparse,
                        io->n_plus_1, gamma + 1, stream));
  return ok();
}

}  // extern "C"

// ---------------------------------------------------------------- verify attention without a workspace
// Scratch for std_dense_verify_attn_noalloc: split-K partials live here instead
// of in a caller-provided workspace.  One copy per device, for the process lifetime.
static __device__ __align__(256) float g_noalloc_scratch[STD_NOALLOC_SCRATCH_BYTES / sizeof(float)];

namespace {

std::mutex g_noalloc_mu;
float* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code
// the array's name only stands in for the symbol, so the address is looked up
// once per device (with that device current) and cached.
int noalloc_scratch(float** out) {
  int dev;
  STD_TRY(current_device(&dev));
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
    g_noalloc_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return STD_OK;
}

}  // namespace

extern "C" int std_dense_verify_attn_noalloc(const std_dims* dims, const void* q, int gamma, const void* k_full,
                                             const void* v_full, const int32_t* len_full, float* o, int splits,
                                             std_stream_t stream) {
  STD_NVTX_RANGE();
  STD_TRY(check_dims(dims));
  STD_TRY(check_ptr(q, 16, "q"));
  STD_TRY(check_ptr(k_full, 16, "k_full"));
  STD_TRY(check_ptr(v_full, 16, "v_full"));
  STD_TRY(check_ptr(len_full, 4, "len_full"));
  STD_TRY(check_ptr(o, 16, "o"));
  if (gamma < 0 || gamma > 31) return fail(STD_ERR_INVALID_ARG, "gamma = %d must be in [0, 31]", gamma);
  AttnPlan plan;
  STD_TRY(plan_attn(dims, gamma + 1, dims->cap_full, splits, &plan));
  const size_t need = plan.ws_bytes;
  if (need > STD_NOALLOC_SCRATCH_BYTES)
    return fail(STD_ERR_WORKSPACE, "verify partials need %zu bytes of scratch; the built-in array holds %u "
                "(use fewer splits or std_dense_verify_attn with a workspace)", need, STD_NOALLOC_SCRATCH_BYTES);
  float* scratch = nullptr;
  if (need > 0) STD_TRY(noalloc_scratch(&scratch));
  return run_attn(dims, q, k_full, v_full, dims->cap_full, len_full, 1, gamma + 1, o, splits, scratch,
                  need > 0 ? STD_NOALLOC_SCRATCH_BYTES : 0, stream);
}
