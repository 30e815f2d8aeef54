// Decode attention on the 5th-generation tensor cores for the sparse draft and
// the dense verify of Sparse-to-Dense decoding ("Methodik" items 2 and 3 of
// the gist.science summary: the draft attends to the selected top-K KV, the
// verifier attends to the whole cache with gamma + 1 query positions in one
// pass).  bf16 operands, fp32 accumulation, fp32 softmax.
//
// Layout of the work.  A problem is one (layer, sequence, KV head); all query
// rows that read it -- the G grouped query heads times the nq query positions,
// at most 128 -- form the M = 128 side of every MMA, so each K/V byte crosses
// HBM once.  The keys of all problems, cut into 128-key tiles, form one flat
// sequence; a persistent grid of CTAs (one per SM by default) takes equal
// contiguous slices of it (stream-K), so the load is balanced whatever the
// lengths.  A CTA that covers a whole problem writes its output directly;
// otherwise it writes one partial (m, l, o) per run of tiles of the same
// problem ("segment") into slot problem + cta, and the last CTA to finish a
// problem (an epoch-tagged arrival counter per problem, no waiting) merges the
// partials of that problem.  The keys-on-lanes kernel for the draft (further down)
// can instead cut each problem into equal parts, one CTA each, whose CTAs form one
// thread-block cluster and merge through distributed shared memory.
//
// Per tile, inside a CTA (warp 0: TMA producers, lane 0 for K/V and lane 1 for
// Q; warp 1: TMEM owner and MMA issuer; warps 2-5: softmax -- one thread per
// query row when a problem has more than 64 rows (M = 128 MMAs); with at most
// 64 rows (the draft, and the verify up to gamma + 1 = 64 / G) the MMAs use
// M = 64, which spreads the rows over all four TMEM lane quarters, so all four
// SM sub-partitions share the softmax, two threads per row):
//   TMA        K tile and V tile (128 keys x d, 128-byte swizzle) -> stage ring
//   MMA        S = Q K^T  -> TMEM S buffer (a ring of three, 128 fp32 columns each)
//   softmax    row max, lazy rescale of O (only when the max grows by more than
//              2^8), P = 2^(x - m) as bf16 written back over S in TMEM
//   MMA        O += P V   (A = P from TMEM, B = V from shared memory, MN-major)
// At the end of a segment the row threads read O from TMEM and write the partial.
// Every wait is bounded; a timeout flags the device error word and unwinds.
#include <cuda.h>
#include <math.h>

#include <atomic>

#include "common.cuh"
#include "internal.h"
#include "tc100.cuh"

namespace stdb {
namespace {

constexpr int TK = 128;           // keys per tile
constexpr int kThreads = 192;
constexpr int STAGES = 3;
constexpr int kMaxB = 64;         // sequences per call handled by this kernel
constexpr int kTmemCols = 512;
constexpr uint32_t kColS = 128;   // TMEM column of S/P buffer 0 (buffer b at 128 + 128 b); O at column 0
constexpr int NSB = 3;            // S/P buffers: S of tile u + 1 is computed while tile u - 1's P V runs
static_assert(kColS + NSB * 128 <= kTmemCols, "O and the S/P ring must fit the TMEM allocation");
constexpr float kTau = 8.f;       // log2 growth of a row max that forces an O rescale
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kMergeSegs = 4;     // segments a merge loads per L2 round trip

struct Ctl {
  uint64_t kv_full[STAGES], kv_empty[STAGES];
  uint64_t q_full, q_empty, done;
  uint64_t s_full[NSB], p_full[NSB], s_free[NSB];
  uint64_t o_ready, o_free;
  uint64_t pub, flag;  // partial published by all 128 row threads / merge decision made
  uint64_t nr_ready;   // fused append: the CTA's new cache rows are written (30 copy lanes)
  uint64_t xb1, xb2, xb3;  // SPLIT layout: a segment's quarter (m, l) published / O halves summed / summed
  float xml[4][16][2];  // SPLIT layout: per quarter and query row, (m in log2 units, l)
  float xrow[16][2];    // SPLIT layout: per query row, the combined (M, L)
  uint32_t tmem;
  int abort_flag;
  int consumed;
  int tl;      // tiles per layer
  int tb;      // first tile of every problem (row_begin / TK)
  int total;   // tiles of the whole call
  int per;     // tiles per CTA
  int last_flag;
  int tiles_b[kMaxB];
  int pre_b[kMaxB];  // Hkv * (tiles of sequences before b)
  int len_b[kMaxB];  // len[b], read once at setup
};

// Arrival on the merge counter of one problem: the counter holds (epoch << 32) |
// arrivals; a stale epoch (an earlier call, or uninitialised memory) restarts the
// count.  Returns true for the arrival that completes `need`.  The merging CTA leaves
// the counter at ((epoch + 1) << 32) | 0, and the host numbers calls in issue order, so
// in a run of calls on one workspace the next call finds its own epoch and each arrival
// is one atomic add, however many CTAs arrive together.  An add that lands on a stale
// epoch is wiped when the count restarts, so that arrival counts itself again with a
// CAS loop.  Lock-free: never a wait on another CTA.
__device__ __forceinline__ bool arrive_last(unsigned long long* ctr, uint32_t epoch, int need) {
  const unsigned long long old = atomicAdd(ctr, 1ull);
  if ((uint32_t)(old >> 32) == epoch) return (int)(old & 0xffffffffull) + 1 == need;
  unsigned long long cur = old + 1ull;
  for (;;) {
    const unsigned long long want =
        (uint32_t)(cur >> 32) == epoch ? cur + 1 : (((unsigned long long)epoch << 32) | 1ull);
    const unsigned long long prev = atomicCAS(ctr, cur, want);
    if (prev == cur) return (int)(want & 0xffffffffull) == need;
    cur = prev;
  }
}

// The counter value the merging CTA leaves for the next call on the workspace.
__device__ __forceinline__ unsigned long long next_call_counter(uint32_t epoch) {
  return (unsigned long long)(uint32_t)(epoch + 1u) << 32;
}


// Tiles of sequence b from tile row_begin / TK on (0 for an invalid length, which is
// flagged, and, for partials, for a sequence with no key in the range).
__device__ __forceinline__ int seq_tiles(const AttnArgs& a, int b, bool flag) {
  const int base = a.len[b] + a.len_off;
  const int lim_max = base + a.nq - 1;
  if (!a.partial && (base <= 0 || (int64_t)lim_max > a.cap)) {
    if (flag) flag_error(a.err, STD_DEVERR_LENGTH);
    return 0;
  }
  const int end = min(lim_max, a.row_end);
  return end > a.row_begin ? (end + TK - 1) / TK - a.row_begin / TK : 0;
}

// Walk over this CTA's slice of the flat (problem, tile) sequence.
struct Iter {
  int g, g_end;
  int l, b, h, t, nt;
  bool first;  // first tile of a segment
};

__device__ __forceinline__ void iter_seek(Iter& it, const Ctl* c, const AttnArgs& a, int g0, int g1) {
  it.g = g0;
  it.g_end = g1;
  it.first = true;
  it.l = it.b = it.h = it.t = 0;
  it.nt = 1;
  if (g0 >= g1) return;
  it.l = g0 / c->tl;
  int r = g0 % c->tl;
  int b = 0;
  while (r >= a.Hkv * c->tiles_b[b]) {
    r -= a.Hkv * c->tiles_b[b];
    ++b;
  }
  it.b = b;
  it.nt = c->tiles_b[b];
  it.h = r / it.nt;
  it.t = r % it.nt;
}

__device__ __forceinline__ bool iter_last(const Iter& it) { return it.g + 1 == it.g_end || it.t + 1 == it.nt; }

__device__ __forceinline__ void iter_next(Iter& it, const Ctl* c, const AttnArgs& a) {
  if (++it.g >= it.g_end) return;
  if (++it.t < it.nt) {
    it.first = false;
    return;
  }
  it.first = true;
  it.t = 0;
  if (++it.h < a.Hkv) return;
  it.h = 0;
  do {
    if (++it.b == a.B) {
      it.b = 0;
      ++it.l;
    }
    it.nt = c->tiles_b[it.b];
  } while (it.nt == 0);
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t adr = smem_u32(bar);
  const uint64_t t0 = tc::globaltimer();
  while (!tc::mbar_try_wait(adr, parity)) {
    if (tc::globaltimer() - t0 > tc::kWaitTimeoutNs) return;
  }
}

// Merge of a problem's segment partials (m, l, o) into its output, by the NTHREADS softmax
// threads of the last CTA to finish the problem.  One item = 4 columns of one query row.
// BATCHED: the segments are taken kMergeSegs at a time, every load of a batch issued
// before any is used (one L2 round trip per batch instead of one per segment), and the
// batches are combined with an online rescale (running max M, sum L, accumulator), so a
// problem split over many CTAs costs ceil(nseg / kMergeSegs) round trips.  The M = 128
// kernel, already near the register limit, keeps the two-pass form (max over all
// segments, then the weighted sums).  Partial k of row r sits at slot0 + k * rows + r;
// output row r at orow0 + r.
template <int D, bool BATCHED, int NTHREADS = 128>
__device__ __forceinline__ void merge_problem(float* out, float* ml_out, const float* ws, const float* ml, int rows,
                                           size_t slot0, int nseg, size_t orow0, int tid) {
  const int nitems = rows * (D / 4);
  // ml_out == nullptr: normalised output; else the merged partial, unnormalised, and its
  // (m, l) with m converted from log2 to natural-log units
  auto write = [&](int r, int col, float M, float L, float4 acc) {
    const float inv = ml_out ? 1.f : (L > 0.f ? 1.f / L : 0.f);
    *reinterpret_cast<float4*>(out + (orow0 + r) * D + col) =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    if (ml_out && col == 0) {
      ml_out[(orow0 + r) * 2] = M * kLn2;
      ml_out[(orow0 + r) * 2 + 1] = L;
    }
  };
  auto two_pass = [&](int item) {
    const int r = item / (D / 4), col = (item % (D / 4)) * 4;
    float M = -INFINITY;
    for (int c = 0; c < nseg; ++c) M = fmaxf(M, __ldcg(ml + (slot0 + (size_t)c * rows + r) * 2));
    const float ref = M == -INFINITY ? 0.f : M;
    float L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = 0; c < nseg; ++c) {
      const size_t k = slot0 + (size_t)c * rows + r;
      const float2 mlk = __ldcg(reinterpret_cast<const float2*>(ml + k * 2));
      const float w = ex2(mlk.x - ref);
      L += w * mlk.y;
      const float4 x = __ldcg(reinterpret_cast<const float4*>(ws + k * D + col));
      acc.x += w * x.x;
      acc.y += w * x.y;
      acc.z += w * x.z;
      acc.w += w * x.w;
    }
    write(r, col, M, L, acc);
  };
  for (int item = tid; item < nitems; item += NTHREADS) {
    if (!BATCHED) {
      two_pass(item);
      continue;
    }
    const int r = item / (D / 4), col = (item % (D / 4)) * 4;
    float M = -INFINITY, L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c0 = 0; c0 < nseg; c0 += kMergeSegs) {
      float2 mlv[kMergeSegs];
      float4 xv[kMergeSegs];
#pragma unroll
      for (int c = 0; c < kMergeSegs; ++c) {
        if (c0 + c < nseg) {
          const size_t k = slot0 + (size_t)(c0 + c) * rows + r;
          mlv[c] = __ldcg(reinterpret_cast<const float2*>(ml + k * 2));
          xv[c] = __ldcg(reinterpret_cast<const float4*>(ws + k * D + col));
        }
      }
      float Mn = M;
#pragma unroll
      for (int c = 0; c < kMergeSegs; ++c)
        if (c0 + c < nseg) Mn = fmaxf(Mn, mlv[c].x);
      const float ref = Mn == -INFINITY ? 0.f : Mn;
      const float f = ex2(M - ref);  // rescale of the batches so far (0 while M is -inf)
      L *= f;
      acc.x *= f;
      acc.y *= f;
      acc.z *= f;
      acc.w *= f;
#pragma unroll
      for (int c = 0; c < kMergeSegs; ++c) {
        if (c0 + c >= nseg) break;
        const float w = ex2(mlv[c].x - ref);
        L += w * mlv[c].y;
        acc.x += w * xv[c].x;
        acc.y += w * xv[c].y;
        acc.z += w * xv[c].z;
        acc.w += w * xv[c].w;
      }
      M = Mn;
    }
    write(r, col, M, L, acc);
  }
}

// Fused append: the 30 idle lanes (index c = 0..29) of the producer warp copy the new
// cache rows whose tiles lie in the CTA's slice [g0, g1) of the flat tile sequence.  Row r
// of problem (l, b, h) goes to position len[b] + new_off + r; the rows are 16-byte chunks,
// K then V, spread over the lanes.
template <int D>
__device__ __forceinline__ void copy_new_rows(const AttnArgs& a, const Ctl* ctl, int g0, int g1, int c) {
  constexpr int kChunks = D * 2 / 16;  // 16-byte chunks per bf16 row
  const size_t row_bytes = (size_t)D * 2;
  Iter it;
  iter_seek(it, ctl, a, g0, g1);
  int l = it.l, b = it.b, h = it.h, nt = it.nt;
  int gp = g0 - it.t;  // flat index of tile 0 of the current problem
  while (gp < g1 && l < a.L) {
    const int prob = (l * a.B + b) * a.Hkv + h;
    const int p0 = ctl->len_b[b] + a.new_off;
    for (int r = 0; r < a.new_rows; ++r) {
      const int pos = p0 + r;
      const int flat = gp + pos / TK - ctl->tb;
      if (flat < g0 || flat >= g1 || pos < 0 || (int64_t)pos >= a.cap) continue;
      for (int i = c; i < 2 * kChunks; i += 30) {
        const bool isv = i >= kChunks;
        const size_t off = (size_t)(i % kChunks) * 16;
        const uint8_t* src = static_cast<const uint8_t*>(isv ? a.v_new : a.k_new) +
                             ((size_t)prob * a.new_rows + r) * row_bytes + off;
        uint8_t* dst = static_cast<uint8_t*>(const_cast<void*>(isv ? a.v : a.k)) +
                       ((size_t)prob * a.cap + pos) * row_bytes + off;
        *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
      }
    }
    gp += nt;
    if (++h == a.Hkv) {  // next sequence (or layer) with tiles
      h = 0;
      do {
        if (++b == a.B) {
          b = 0;
          ++l;
        }
        nt = ctl->tiles_b[b];
      } while (nt == 0 && l < a.L);
    }
  }
}

template <int D>
struct Cfg {
  static constexpr int KB = D / 64;                   // 128-byte column blocks of a row
  static constexpr uint32_t Q_BYTES = KB * 128 * 128;  // 128 query rows
  static constexpr uint32_t T_BYTES = KB * TK * 128;   // one K or V tile
  static constexpr uint32_t ST_BYTES = 2 * T_BYTES;    // K + V
  static constexpr uint32_t SMEM = 1024 + Q_BYTES + STAGES * ST_BYTES + sizeof(Ctl);
  static_assert(SMEM <= 232448, "dynamic shared memory above the 227 KB a CTA may use");
};

// HALF: at most 64 query rows per problem.  The MMAs then use M = 64, whose
// accumulator row i sits in TMEM lane 32 * (i / 16) + i % 16, so the rows are
// spread over all four lane quarters (and SM sub-partitions) and two softmax
// threads share a row, each taking 64 of its 128 columns.
// SPLIT (with HALF; at most 16 query rows, the draft's case): the 16 query rows are
// loaded four times, to MMA rows q * 16 + i for q = 0..3, so every lane quarter holds
// a copy of every row and every softmax warp has work.  Quarter q takes 32 of each
// tile's 128 keys (keys 16q..16q+15 and 64+16q..64+16q+15; the thread pair of a row
// 16 each) and keeps its own running max, sum and O row -- zeros in P elsewhere keep
// the other quarters' keys out of its O; at the end of a segment the four (m, l, O)
// are combined in shared memory in a fixed order ((q0 + q2) + (q1 + q3)), so results
// do not depend on scheduling.  Each softmax thread then handles 16 keys of a tile
// instead of 64: the per-tile latency that bounds a CTA with few query rows drops.
template <int D, bool HALF, bool SPLIT>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_k16,
               const __grid_constant__ CUtensorMap tm_v16, const AttnArgs a) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sKV = sQ + C::Q_BYTES;
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + C::Q_BYTES + STAGES * C::ST_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    // the tensor maps are kernel parameters: fetch them while the barriers are set up
    // (and, launched early, while the previous kernel finishes)
    tc::prefetch_tmap(&tm_q);
    tc::prefetch_tmap(&tm_k);
    tc::prefetch_tmap(&tm_v);
    tc::prefetch_tmap(&tm_k16);
    tc::prefetch_tmap(&tm_v16);
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(&ctl->kv_full[s], 1);
      tc::mbar_init(&ctl->kv_empty[s], 1);
    }
    tc::mbar_init(&ctl->q_full, 1);
    tc::mbar_init(&ctl->q_empty, 1);
    tc::mbar_init(&ctl->done, 1);
    for (int i = 0; i < NSB; ++i) {
      tc::mbar_init(&ctl->s_full[i], 1);
      tc::mbar_init(&ctl->p_full[i], 128);
      tc::mbar_init(&ctl->s_free[i], 1);
    }
    tc::mbar_init(&ctl->o_ready, 1);
    tc::mbar_init(&ctl->o_free, 128);
    tc::mbar_init(&ctl->pub, 128);
    tc::mbar_init(&ctl->flag, 1);
    tc::mbar_init(&ctl->nr_ready, 30);
    tc::mbar_init(&ctl->xb1, 128);
    tc::mbar_init(&ctl->xb2, 128);
    tc::mbar_init(&ctl->xb3, 128);
    ctl->abort_flag = 0;
    ctl->consumed = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    __syncwarp();
    tc::tmem_alloc(&ctl->tmem, kTmemCols);
    tc::tmem_relinquish();
  }
  // The barrier and TMEM set-up above touch no global memory and may overlap the previous
  // kernel.  Without the early start, everything below waits for it; with it (a.early),
  // the lengths are read now and each role waits just before it needs to (below).
  if (!a.early) {
    pdl_wait();
    pdl_trigger();  // only after this CTA's wait: the next kernel may start early itself
  }
  if (threadIdx.x == 0) {
    int sum = 0;
    for (int b = 0; b < a.B; ++b) {
      ctl->tiles_b[b] = seq_tiles(a, b, blockIdx.x == 0);
      ctl->len_b[b] = a.len[b];
      ctl->pre_b[b] = a.Hkv * sum;
      sum += ctl->tiles_b[b];
    }
    ctl->tl = a.Hkv * sum;
    ctl->tb = a.row_begin / TK;
    ctl->total = a.L * ctl->tl;
    ctl->per = ctl->total > 0 ? (ctl->total + gridDim.x - 1) / gridDim.x : 1;
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = ctl->tmem;
  volatile int* abort_flag = &ctl->abort_flag;
  const int g0 = min(ctl->total, (int)blockIdx.x * ctl->per);
  const int g1 = min(ctl->total, g0 + ctl->per);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producers
    if (lane == 0 && g0 < g1) {
      Iter it;
      iter_seek(it, ctl, a, g0, g1);
      int kv = 0;
      bool rows_ready = a.k_new == nullptr;
      bool waited = !a.early;
      while (it.g < it.g_end) {
        const int prob = (it.l * a.B + it.b) * a.Hkv + it.h;
        const int s = kv % STAGES;
        const int tabs = it.t + ctl->tb;  // tile index within the problem
        // early start: rows from len[b] + new_off - 1 on may still be written by the previous kernel
        if (!waited && (tabs + 1) * TK > ctl->len_b[it.b] + a.new_off - 1) {
          pdl_wait();
          waited = true;
        }
        if (!rows_ready) {  // fused append: a tile holding new rows waits until they are written
          const int p0 = ctl->len_b[it.b] + a.new_off;
          if (tabs * TK < p0 + a.new_rows && p0 < (tabs + 1) * TK) {
            if (!tc::mbar_wait(&ctl->nr_ready, 0, abort_flag, a.err)) break;
            rows_ready = true;
          }
        }
        if (!tc::mbar_wait(&ctl->kv_empty[s], ((kv / STAGES) & 1) ^ 1, abort_flag, a.err)) break;
        if (!STD_DCHECK(tabs * TK < a.cap && prob < a.L * a.B * a.Hkv, a.err)) break;
        const int row = prob * (int)a.cap + tabs * TK;
        const uint32_t st = sKV + s * C::ST_BYTES;
        // keys any query row of the problem attends to in this tile; a short last tile is
        // fetched in 16-row boxes (the rows past them are masked and their V zeroed)
        const int nvalid = min(ctl->len_b[it.b] + a.len_off + a.nq - 1, a.row_end) - tabs * TK;
        if (nvalid >= TK) {
          tc::mbar_expect_tx(&ctl->kv_full[s], C::ST_BYTES);
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb) {
            tc::tma_load_2d(st + kb * TK * 128, &tm_k, kb * 64, row, &ctl->kv_full[s]);
            tc::tma_load_2d(st + C::T_BYTES + kb * TK * 128, &tm_v, kb * 64, row, &ctl->kv_full[s]);
          }
        } else {
          const int nb = (nvalid + 15) >> 4;  // 1..8 boxes of 16 rows
          tc::mbar_expect_tx(&ctl->kv_full[s], (uint32_t)nb * 16 * 128 * C::KB * 2);
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb) {
            for (int i = 0; i < nb; ++i) {
              tc::tma_load_2d(st + kb * TK * 128 + i * 16 * 128, &tm_k16, kb * 64, row + i * 16, &ctl->kv_full[s]);
              tc::tma_load_2d(st + C::T_BYTES + kb * TK * 128 + i * 16 * 128, &tm_v16, kb * 64, row + i * 16,
                              &ctl->kv_full[s]);
            }
          }
        }
        ++kv;
        iter_next(it, ctl, a);
      }
      if (*abort_flag) {  // let the copies in flight land
        for (int k = *(volatile int*)&ctl->consumed; k < kv; ++k) drain_wait(&ctl->kv_full[k % STAGES], (k / STAGES) & 1);
      }
    } else if (lane == 1 && g0 < g1) {
      Iter it;
      iter_seek(it, ctl, a, g0, g1);
      int seg = 0;
      bool waited = !a.early;
      while (it.g < it.g_end) {
        if (it.first) {
          if (!waited && !(a.early & STD_ATTN_EARLY_Q)) {  // Q may still be written by the previous kernel
            pdl_wait();
            pdl_trigger();
            waited = true;
          }
          if (!tc::mbar_wait(&ctl->q_empty, (seg & 1) ^ 1, abort_flag, a.err)) break;
          tc::mbar_expect_tx(&ctl->q_full, HALF ? C::Q_BYTES / 2 : C::Q_BYTES);  // HALF: 64-row boxes
          const int qrow = ((it.l * a.B + it.b) * a.Hq + it.h * a.G) * a.nq;
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb) {
            if constexpr (SPLIT) {  // the same 16 rows at MMA rows 0, 16, 32, 48 (tm_q: 16-row boxes)
#pragma unroll
              for (int q = 0; q < 4; ++q)
                tc::tma_load_2d(sQ + kb * 128 * 128 + q * 16 * 128, &tm_q, kb * 64, qrow, &ctl->q_full);
            } else {
              tc::tma_load_2d(sQ + kb * 128 * 128, &tm_q, kb * 64, qrow, &ctl->q_full);
            }
          }
          ++seg;
          if (!waited) {  // this CTA's wait, off every other role's path
            pdl_wait();
            pdl_trigger();
            waited = true;
          }
        }
        iter_next(it, ctl, a);
      }
      if (*abort_flag && seg > 0) drain_wait(&ctl->q_full, (seg - 1) & 1);
    } else if (lane >= 2 && g0 < g1 && a.k_new != nullptr) {
      // fused append: write the new rows whose tiles fall in this CTA's slice (only this
      // CTA reads those tiles), then order the writes before the TMA loads of them
      if (a.early) pdl_wait();  // the previous kernel may still read the tile these rows land in
      copy_new_rows<D>(a, ctl, g0, g1, lane - 2);
      asm volatile("fence.proxy.async.global;" ::: "memory");
      tc::mbar_arrive(&ctl->nr_ready);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && g0 < g1) {
      constexpr int MM = HALF ? 64 : 128;  // MMA M: query rows covered
      constexpr uint32_t idS = tc::idesc_bf16(MM, TK);
      constexpr uint32_t idPV = tc::idesc_bf16(MM, D) | (1u << 16);  // B = V, MN-major
      Iter it;
      iter_seek(it, ctl, a, g0, g1);
      int seg = -1, kv = 0, u = 0;
      int pu = -1, ps = 0, pseg = 0;
      bool pfirst = false, any = false, ok = true;
      auto issue_pv = [&](int vu, int vs, bool vfirst, bool vlast, int vseg) -> bool {
        const int vb = vu % NSB;
        if (!tc::mbar_wait(&ctl->p_full[vb], (vu / NSB) & 1, abort_flag, a.err)) return false;
        if (vfirst && !tc::mbar_wait(&ctl->o_free, (vseg & 1) ^ 1, abort_flag, a.err)) return false;
        tc::fence_after_sync();
        const uint32_t p_tm = tmem + kColS + vb * 128;
        const uint32_t sv = sKV + vs * C::ST_BYTES + C::T_BYTES;
#pragma unroll
        for (int k = 0; k < TK / 16; ++k)
          tc::umma_bf16_ts(tmem, p_tm + 8 * k, tc::sdesc_sw128_mn(sv + k * 16 * 128, TK * 128), idPV,
                           (vfirst && k == 0) ? 0u : 1u);
        tc::umma_commit(&ctl->kv_empty[vs]);
        tc::umma_commit(&ctl->s_free[vb]);
        if (vlast) tc::umma_commit(&ctl->o_ready);
        return true;
      };
      while (it.g < it.g_end) {
        const bool first = it.first, last = iter_last(it);
        if (first) {
          ++seg;
          if (!tc::mbar_wait(&ctl->q_full, seg & 1, abort_flag, a.err)) { ok = false; break; }
        }
        const int s = kv % STAGES;
        if (!tc::mbar_wait(&ctl->kv_full[s], (kv / STAGES) & 1, abort_flag, a.err)) { ok = false; break; }
        *(volatile int*)&ctl->consumed = kv + 1;
        const int bu = u % NSB;
        if (!tc::mbar_wait(&ctl->s_free[bu], ((u / NSB) & 1) ^ 1, abort_flag, a.err)) { ok = false; break; }
        tc::fence_after_sync();
        const uint32_t s_tm = tmem + kColS + bu * 128;
        const uint32_t sk = sKV + s * C::ST_BYTES;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k & 3) * 32;
          tc::umma_bf16(s_tm, tc::sdesc_sw128(sQ + (k >> 2) * 128 * 128 + off),
                        tc::sdesc_sw128(sk + (k >> 2) * TK * 128 + off), idS, k > 0 ? 1u : 0u);
        }
        any = true;
        tc::umma_commit(&ctl->s_full[bu]);
        if (last) tc::umma_commit(&ctl->q_empty);
        if (pu >= 0) {
          if (!issue_pv(pu, ps, pfirst, false, pseg)) { ok = false; break; }
          pu = -1;
        }
        if (last) {
          if (!issue_pv(u, s, first, true, seg)) { ok = false; break; }
        } else {
          pu = u;
          ps = s;
          pfirst = first;
          pseg = seg;
        }
        ++u;
        ++kv;
        iter_next(it, ctl, a);
      }
      if (!ok && any) {  // MMAs still in flight must finish before TMEM is freed
        tc::umma_commit(&ctl->done);
        drain_wait(&ctl->done, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax threads
    // Full layout: one thread per query row = TMEM lane (warp % 4) * 32 + lane, all 128
    // columns of S.  HALF layout: query row (warp % 4) * 16 + lane % 16 in TMEM lane
    // (warp % 4) * 32 + lane % 16; lane < 16 takes columns [0, 64), lane >= 16 [64, 128).
    // SPLIT layout: query row lane % 16, copy of quarter (warp % 4); the thread takes keys
    // 16 (warp % 4) + 64 (lane / 16) + [0, 16) of each tile.
    constexpr int NC = SPLIT ? 16 : (HALF ? TK / 2 : TK);  // S columns (keys) per thread
    constexpr int OC = HALF ? D / 2 : D;    // O columns per thread
    const int qd = warp & 3;                // TMEM lane quarter of this warp
    const int row = SPLIT ? (lane & 15) : HALF ? qd * 16 + (lane & 15) : qd * 32 + lane;  // query row
    const int hh = HALF ? lane >> 4 : 0;    // which column half (HALF layout)
    const bool wactive = SPLIT || (HALF ? qd * 16 : qd * 32) < a.rows;  // warp holds a real query row
    // SPLIT: two [16][D] fp32 sums of the quarters' O rows (quarters 0 + 2 and 1 + 3), in the
    // parts of the Q area that the 64-row query tile leaves unused (8 KB at 8 KB, and 8 KB at
    // 24 KB for D = 128 or 4 KB at 12 KB for D = 64)
    float* redA = reinterpret_cast<float*>(smem + 8192);
    float* redB = reinterpret_cast<float*>(smem + (D == 128 ? 24576 : 12288));
    const uint32_t lane_base = tmem + ((uint32_t)(qd * 32) << 16);
    const float sc = kLog2e * rsqrtf((float)D);
    const int tid = threadIdx.x - 64;
    Iter it;
    iter_seek(it, ctl, a, g0, g1);
    int seg = -1, kv = 0, u = 0, npub = 0, nx = 0;
    float m = -INFINITY, l = 0.f;
    int lim = 0, lim_max = 0;
    while (it.g < it.g_end) {
      const bool first = it.first, last = iter_last(it);
      const int lb = it.l * a.B + it.b;
      const int prob = lb * a.Hkv + it.h;
      if (first) {
        ++seg;
        m = -INFINITY;
        l = 0.f;
        const int base = a.len[it.b] + a.len_off;
        lim = min(base + (row < a.rows ? row % a.nq : 0), a.row_end);
        lim_max = min(base + a.nq - 1, a.row_end);
      }
      const int bu = u % NSB;
      const int s = kv % STAGES;
      const int key0 = (it.t + ctl->tb) * TK;
      if (!tc::mbar_wait_warp(&ctl->s_full[bu], (u / NSB) & 1, abort_flag, a.err)) break;
      tc::fence_after_sync();
      if (key0 + TK > lim_max || key0 < a.row_begin) {
        // last tile of the problem (or first tile of a key range): zero the V rows past
        // the last query's limit and before the range, so that whatever bytes sit there
        // cannot turn 0 * V into NaN
        if (!tc::mbar_wait_warp(&ctl->kv_full[s], (kv / STAGES) & 1, abort_flag, a.err)) break;
        const int z0 = max(0, lim_max - key0);
        const int zb = a.row_begin - key0;
        uint8_t* vb = smem + C::Q_BYTES + s * C::ST_BYTES + C::T_BYTES;
        for (int i = tid; i < C::KB * TK * 8; i += 128) {
          const int r = (i >> 3) % TK;
          if (r >= z0 || r < zb)
            *reinterpret_cast<uint4*>(vb + (i / (TK * 8)) * TK * 128 + r * 128 + (i & 7) * 16) = make_uint4(0, 0, 0, 0);
        }
        tc::fence_proxy_async();
      }
      if (wactive) {
        // this thread's logits of the tile: v[j] is key kc0 + j
        float v[NC];
        const int kc0 = key0 + hh * (TK / 2) + (SPLIT ? 16 * qd : 0);
        {
          const uint32_t sa = lane_base + kColS + bu * 128;
          if constexpr (SPLIT) {
            uint32_t r0[16];
            __syncwarp();
            tc::tmem_ld16_x16<TK / 2>(sa + 16 * qd, r0);
            tc::tmem_ld_wait16(r0);
  #pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r0[j]);
          } else if constexpr (HALF) {
            uint32_t r0[32], r1[32];
            __syncwarp();
            tc::tmem_ld16_x32<TK / 2>(sa, r0);
            tc::tmem_ld16_x32<TK / 2>(sa + 32, r1);
            tc::tmem_ld_wait(r0);
            tc::tmem_ld_wait(r1);
  #pragma unroll
            for (int j = 0; j < 32; ++j) {
              v[j] = __uint_as_float(r0[j]);
              v[32 + j] = __uint_as_float(r1[j]);
            }
          } else {
            uint32_t r0[32], r1[32], r2[32], r3[32];
            __syncwarp();
            tc::tmem_ld_x32(sa, r0);
            tc::tmem_ld_x32(sa + 32, r1);
            tc::tmem_ld_x32(sa + 64, r2);
            tc::tmem_ld_x32(sa + 96, r3);
            tc::tmem_ld_wait(r0);
            tc::tmem_ld_wait(r1);
            tc::tmem_ld_wait(r2);
            tc::tmem_ld_wait(r3);
  #pragma unroll
            for (int j = 0; j < 32; ++j) {
              v[j] = __uint_as_float(r0[j]);
              v[32 + j] = __uint_as_float(r1[j]);
              v[64 + j] = __uint_as_float(r2[j]);
              v[96 + j] = __uint_as_float(r3[j]);
            }
          }
        }
        if (kc0 + NC > lim) {
  #pragma unroll
          for (int j = 0; j < NC; ++j)
            if (kc0 + j >= lim) v[j] = -INFINITY;
        }
        if (kc0 < a.row_begin) {  // key range: keys before it are not attended
  #pragma unroll
          for (int j = 0; j < NC; ++j)
            if (kc0 + j < a.row_begin) v[j] = -INFINITY;
        }
        float mx = v[0];
  #pragma unroll
        for (int j = 1; j + 1 < NC; j += 2) mx = max3f(mx, v[j], v[j + 1]);
        mx = fmaxf(mx, v[NC - 1]);
        if constexpr (HALF) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));  // both halves of the row
        // lazy rescale: only when the max grows by more than 2^kTau (whole warp, O is warp-collective)
        const bool resc = (m != -INFINITY) && (mx - m) * sc > kTau;
        if (__any_sync(0xffffffffu, resc)) {
          // the previous tile's P V must have landed in O before O is rescaled
          // (u >= 1 here: a rescale needs an earlier tile of the same segment)
          if (!tc::mbar_wait_warp(&ctl->s_free[(u - 1) % NSB], ((u - 1) / NSB) & 1, abort_flag, a.err)) break;
          tc::fence_after_sync();
          const float f = resc ? ex2((m - mx) * sc) : 1.f;
  #pragma unroll
          for (int c = 0; c < OC / 32; ++c) {  // this thread's O columns
            uint32_t o[32];
            __syncwarp();
            if constexpr (HALF) tc::tmem_ld16_x32<D / 2>(lane_base + c * 32, o);
            else tc::tmem_ld_x32(lane_base + c * 32, o);
            tc::tmem_ld_wait(o);
  #pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
            if constexpr (HALF) tc::tmem_st16_x32<D / 2>(lane_base + c * 32, o);
            else tc::tmem_st_x32(lane_base + c * 32, o);
          }
          tc::tmem_st_wait();
          l *= f;
          if (resc) m = mx;
        }
        if (m == -INFINITY) m = mx;  // first key this row may see (stays -inf if none yet)
        const float msc = m * sc;
        const bool live = m != -INFINITY;
        // P = 2^(x - m) as bf16 pairs, written over the S columns already read
        // (packed column j of the tile holds keys 2j and 2j + 1)
        uint32_t pk[NC / 2];
        const f32x2 scc = f2_make(sc, sc), nm = f2_make(-msc, -msc);
        if constexpr (SPLIT) {
          f32x2 sacc = f2_make(0.f, 0.f);
  #pragma unroll
          for (int j = 0; j < 8; ++j) {
            float x0, x1;
            f2_split(f2_fma(f2_make(v[2 * j], v[2 * j + 1]), scc, nm), x0, x1);
            const float p0 = live ? ex2(x0) : 0.f;
            const float p1 = live ? ex2(x1) : 0.f;
            sacc = f2_add(sacc, f2_make(p0, p1));
            pk[j] = pack_bf16(p0, p1);
          }
          float sl, sh;
          f2_split(sacc, sl, sh);
          l += sl + sh;
          // this thread's half of the P row: its 8 packed columns, zeros for the other quarters' keys
          uint32_t prow[32];
  #pragma unroll
          for (int c = 0; c < 32; ++c) prow[c] = (c >> 3) == qd ? pk[c & 7] : 0u;
          __syncwarp();
          tc::tmem_st16_x32<TK / 4>(lane_base + kColS + bu * 128, prow);
        }
  #pragma unroll
        for (int c = 0; c < NC / 32; ++c) {
          f32x2 sacc = f2_make(0.f, 0.f);
  #pragma unroll
          for (int j = 0; j < 16; ++j) {
            float x0, x1;
            f2_split(f2_fma(f2_make(v[c * 32 + 2 * j], v[c * 32 + 2 * j + 1]), scc, nm), x0, x1);
            const float p0 = live ? ex2(x0) : 0.f;
            const float p1 = live ? ex2(x1) : 0.f;
            sacc = f2_add(sacc, f2_make(p0, p1));
            pk[c * 16 + j] = pack_bf16(p0, p1);
          }
          float sl, sh;
          f2_split(sacc, sl, sh);
          l += sl + sh;  // HALF: this thread's half of the row sum
          if constexpr (!HALF) {
            __syncwarp();
            tc::tmem_st_x16(lane_base + kColS + bu * 128 + c * 16, reinterpret_cast<const uint32_t(&)[16]>(pk[c * 16]));
          }
        }
        if constexpr (HALF && !SPLIT) {
          __syncwarp();
          tc::tmem_st16_x32<TK / 4>(lane_base + kColS + bu * 128, pk);
        }
        tc::tmem_st_wait();
      }
      tc::fence_before_sync();
      tc::mbar_arrive(&ctl->p_full[bu]);
      if (last) {
        if (!tc::mbar_wait_warp(&ctl->o_ready, seg & 1, abort_flag, a.err)) break;
        tc::fence_after_sync();
        if (a.early) pdl_wait();  // outputs, partials and merge counters: after the previous kernel
        const float lrow = HALF ? l + __shfl_xor_sync(0xffffffffu, l, 16) : l;  // the row's (quarter's) sum
        // CTAs whose slices touch this problem
        const int start = it.l * ctl->tl + ctl->pre_b[it.b] + it.h * it.nt;
        const int c0 = start / ctl->per, c1 = (start + it.nt - 1) / ctl->per;
        const size_t orow0 = (size_t)(lb * a.Hq + it.h * a.G) * a.nq;  // output row of query row 0
        const size_t orow = orow0 + row;
        // segment partials: slot prob + blockIdx.x of [slots][rows][D], then (m, l), then counters
        const size_t nslots = (size_t)a.L * a.B * a.Hkv + gridDim.x;
        float* wml = a.ws + nslots * a.rows * D;
        unsigned long long* ctr = reinterpret_cast<unsigned long long*>(wml + nslots * a.rows * 2);
        const int slot = prob + blockIdx.x;
        if constexpr (SPLIT) {
          // combine the four quarters' (m, l, O) of every query row: publish (m, l), weigh each
          // quarter's O row by 2^(m_q - M) into the shared sum, then write from the sum
          if (hh == 0) {
            ctl->xml[qd][row][0] = m * sc;
            ctl->xml[qd][row][1] = lrow;
          }
          tc::mbar_arrive(&ctl->xb1);
          if (!tc::mbar_wait_warp(&ctl->xb1, nx & 1, abort_flag, a.err)) break;
          float M = -INFINITY;
#pragma unroll
          for (int q = 0; q < 4; ++q) M = fmaxf(M, ctl->xml[q][row][0]);
          const float ref = M == -INFINITY ? 0.f : M;
          if (qd == 0 && hh == 0) {
            float L = 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) L += ex2(ctl->xml[q][row][0] - ref) * ctl->xml[q][row][1];
            ctl->xrow[row][0] = M;
            ctl->xrow[row][1] = L;
          }
          const float w = ex2(m * sc - ref);  // 0 for a quarter that saw no key
          // quarters 0 and 1 store w O into redA / redB, then quarters 2 and 3 add theirs: every
          // element is written by one thread at a time, in a fixed order
          // (16-byte chunk k of a row is stored at chunk k ^ (row & 7): the eight rows a
          // quarter-warp stores at once then fall in eight different bank groups)
          float* red = (qd & 1) ? redB : redA;
          if (qd < 2) {
#pragma unroll
            for (int c = 0; c < OC / 32; ++c) {
              uint32_t o[32];
              __syncwarp();
              tc::tmem_ld16_x32<D / 2>(lane_base + c * 32, o);
              tc::tmem_ld_wait(o);
              if (row < a.rows) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  const int k = ((hh * OC + c * 32) / 4 + j) ^ (row & 7);
                  *reinterpret_cast<float4*>(red + row * D + 4 * k) =
                      make_float4(w * __uint_as_float(o[4 * j]), w * __uint_as_float(o[4 * j + 1]),
                                  w * __uint_as_float(o[4 * j + 2]), w * __uint_as_float(o[4 * j + 3]));
                }
              }
            }
          }
          tc::mbar_arrive(&ctl->xb2);
          if (!tc::mbar_wait_warp(&ctl->xb2, nx & 1, abort_flag, a.err)) break;
          if (qd >= 2) {
#pragma unroll
            for (int c = 0; c < OC / 32; ++c) {
              uint32_t o[32];
              __syncwarp();
              tc::tmem_ld16_x32<D / 2>(lane_base + c * 32, o);
              tc::tmem_ld_wait(o);
              if (row < a.rows) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  float4* dst = reinterpret_cast<float4*>(red + row * D + 4 * (((hh * OC + c * 32) / 4 + j) ^ (row & 7)));
                  const float4 x = *dst;
                  *dst = make_float4(x.x + w * __uint_as_float(o[4 * j]), x.y + w * __uint_as_float(o[4 * j + 1]),
                                     x.z + w * __uint_as_float(o[4 * j + 2]), x.w + w * __uint_as_float(o[4 * j + 3]));
                }
              }
            }
          }
          tc::fence_before_sync();
          tc::mbar_arrive(&ctl->o_free);  // O may be reused
          tc::mbar_arrive(&ctl->xb3);
          if (!tc::mbar_wait_warp(&ctl->xb3, nx & 1, abort_flag, a.err)) break;
          ++nx;
          for (int e = tid; e < a.rows * (D / 4); e += 128) {
            const int r = e / (D / 4), col = (e % (D / 4)) * 4;
            const int sw = 4 * ((e % (D / 4)) ^ (r & 7));  // where the chunk of col sits
            const float4 xa = *reinterpret_cast<const float4*>(redA + r * D + sw);
            const float4 xb = *reinterpret_cast<const float4*>(redB + r * D + sw);
            const float4 x = make_float4(xa.x + xb.x, xa.y + xb.y, xa.z + xb.z, xa.w + xb.w);
            const float Mr = ctl->xrow[r][0], Lr = ctl->xrow[r][1];
            if (c0 == c1) {
              const float inv = a.partial ? 1.f : (Lr > 0.f ? 1.f / Lr : 0.f);
              *reinterpret_cast<float4*>(a.o + (orow0 + r) * D + col) =
                  make_float4(x.x * inv, x.y * inv, x.z * inv, x.w * inv);
              if (a.partial && col == 0) {
                a.ml[(orow0 + r) * 2] = Mr * kLn2;
                a.ml[(orow0 + r) * 2 + 1] = Lr;
              }
            } else {
              *reinterpret_cast<float4*>(a.ws + ((size_t)slot * a.rows + r) * D + col) = x;
              if (col == 0) {
                wml[((size_t)slot * a.rows + r) * 2] = Mr;
                wml[((size_t)slot * a.rows + r) * 2 + 1] = Lr;
              }
            }
          }
        } else if (c0 == c1) {
          // this CTA saw the whole problem: normalised output straight from TMEM (partials:
          // unnormalised, with (m, l) beside it)
          const float inv = a.partial ? 1.f : (lrow > 0.f ? 1.f / lrow : 0.f);
          if (a.partial && row < a.rows && hh == 0) {
            a.ml[orow * 2] = m * rsqrtf((float)D);
            a.ml[orow * 2 + 1] = lrow;
          }
#pragma unroll
          for (int c = 0; c < OC / 32; ++c) {
            uint32_t o[32];
            __syncwarp();
            if constexpr (HALF) tc::tmem_ld16_x32<D / 2>(lane_base + c * 32, o);
            else tc::tmem_ld_x32(lane_base + c * 32, o);
            tc::tmem_ld_wait(o);
            if (row < a.rows) {
              float* dst = a.o + orow * D + hh * OC + c * 32;
#pragma unroll
              for (int j = 0; j < 32; j += 4)
                *reinterpret_cast<float4*>(dst + j) =
                    make_float4(__uint_as_float(o[j]) * inv, __uint_as_float(o[j + 1]) * inv,
                                __uint_as_float(o[j + 2]) * inv, __uint_as_float(o[j + 3]) * inv);
            }
          }
          tc::fence_before_sync();
          tc::mbar_arrive(&ctl->o_free);
        } else {
          float* po = a.ws + ((size_t)slot * a.rows + row) * D + hh * OC;
#pragma unroll
          for (int c = 0; c < OC / 32; ++c) {
            uint32_t o[32];
            __syncwarp();
            if constexpr (HALF) tc::tmem_ld16_x32<D / 2>(lane_base + c * 32, o);
            else tc::tmem_ld_x32(lane_base + c * 32, o);
            tc::tmem_ld_wait(o);
            if (row < a.rows) {
#pragma unroll
              for (int j = 0; j < 32; j += 4)
                *reinterpret_cast<float4*>(po + c * 32 + j) =
                    make_float4(__uint_as_float(o[j]), __uint_as_float(o[j + 1]), __uint_as_float(o[j + 2]),
                                __uint_as_float(o[j + 3]));
            }
          }
          if (row < a.rows && hh == 0) {
            wml[((size_t)slot * a.rows + row) * 2] = m * sc;
            wml[((size_t)slot * a.rows + row) * 2 + 1] = lrow;
          }
          tc::fence_before_sync();
          tc::mbar_arrive(&ctl->o_free);  // O may be reused: the rest reads global memory only
        }
        if (c0 != c1) {
          // publish the partial, count the arrival; the last CTA merges every slot of the problem.
          // The CTA's partial writes reach thread 0 through the mbarrier (release / acquire in
          // the CTA); thread 0's device-scope fence before the counter publishes them all, and
          // its fence after the counter makes the other CTAs' partials visible to the merge,
          // which the other threads order after through the second mbarrier.
          tc::mbar_arrive(&ctl->pub);
          if (tid == 0) {
            if (!tc::mbar_wait(&ctl->pub, npub & 1, abort_flag, a.err)) break;
            __threadfence();
            ctl->last_flag = arrive_last(ctr + prob, a.epoch, c1 - c0 + 1) ? 1 : 0;
            if (ctl->last_flag) __threadfence();
            tc::mbar_arrive(&ctl->flag);
          }
          if (!tc::mbar_wait(&ctl->flag, npub & 1, abort_flag, a.err)) break;
          ++npub;
          if (ctl->last_flag && STD_DCHECK((size_t)prob + c1 < nslots && c0 <= c1, a.err)) {
            // all 128 softmax threads share the merge
            merge_problem<D, HALF>(a.o, a.partial ? a.ml : nullptr, a.ws, wml, a.rows, (size_t)(prob + c0) * a.rows,
                                   c1 - c0 + 1, orow0, tid);
            if (tid == 0) atomicExch(ctr + prob, next_call_counter(a.epoch));
          }
        }
      }
      ++u;
      ++kv;
      iter_next(it, ctl, a);
    }
    if (a.partial && blockIdx.x == 0) {
      // partials of a sequence with no key in the range: o = 0, m = -inf, l = 0
      const int per_b = a.Hq * a.nq;  // output rows of one (layer, sequence)
      for (int b = 0; b < a.B; ++b) {
        if (ctl->tiles_b[b] != 0) continue;
        for (int i = tid; i < a.L * per_b * (D / 4); i += 128) {
          const int l_ = i / (per_b * (D / 4)), rem = i % (per_b * (D / 4));
          const size_t orow = (size_t)(l_ * a.B + b) * per_b + rem / (D / 4);
          *reinterpret_cast<float4*>(a.o + orow * D + (rem % (D / 4)) * 4) = make_float4(0.f, 0.f, 0.f, 0.f);
          if (rem % (D / 4) == 0) {
            a.ml[orow * 2] = -INFINITY;
            a.ml[orow * 2 + 1] = 0.f;
          }
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Keys-on-lanes layout (at most 16 query rows, d = 128: the draft step).  With a
// handful of query rows the M = 64 MMAs above are mostly padding, so here every
// MMA is transposed and the tile's 128 keys fill its M = 128 side:
//   MMA      S^T = K Q^T     A = K tile, B = the 16-row query tile (both K-major)
//                            -> TMEM S buffer: lane = key, column = query row
//   softmax  thread t of the four softmax warps owns key t of the tile and reads
//            its 16 logits; the warps combine their per-row maxima once per tile
//            through shared memory (lazy rescale of O as above) and thread t writes
//            P^T[row][t] as bf16 into a shared buffer [16 rows][128 keys]
//   MMA      O^T += V^T P^T  A = V tile read MN-major, B = the P buffer (K-major)
//                            -> TMEM O: lane = element of d, column = query row
// One tile costs 16 MMAs of 128 x 16 x 16 instead of 16 of 64 x 128 x 16, each
// softmax thread evaluates one exponential per real query row, and the segment end
// needs no combine of lane quarters: thread t holds element t of every output row.
struct CtlT : Ctl {
  uint64_t prev_done;    // early start: the previous kernel has completed (its writes are visible)
  uint64_t xmax[2][2];   // [row group][tile parity]: the group's four warps' row maxima are in wmax
  uint64_t xsum[2];      // [row group] segment end: the group's four warps' row sums are in wsum
  alignas(16) float wmax[2][16][4];  // [tile parity][query row][softmax warp], read as float4
  alignas(16) float wsum[16][4];
};
static_assert(alignof(CtlT) >= 16, "the float4 reads of wmax / wsum need 16-byte alignment");

struct CfgT {
  static constexpr int D = 128;
  static constexpr int KB = D / 64;
  static constexpr uint32_t Q_BYTES = KB * 16 * 128;   // 16 query rows
  static constexpr uint32_t P_BYTES = 2 * 16 * 128;    // one P buffer: 16 rows x 128 keys, bf16
  static constexpr uint32_t T_BYTES = KB * TK * 128;   // one K or V tile
  static constexpr uint32_t ST_BYTES = 2 * T_BYTES;
  static constexpr uint32_t KV_OFF = Q_BYTES + NSB * P_BYTES;
  static constexpr uint32_t SMEM = 1024 + KV_OFF + STAGES * ST_BYTES + sizeof(CtlT);
  static_assert(KV_OFF % 1024 == 0, "stages must start on a 1024-byte swizzle atom");
  static_assert(SMEM <= 232448, "dynamic shared memory above the 227 KB a CTA may use");
};
constexpr int kTmemColsT = 64;     // O^T at columns 0..15, S^T buffer b at 16 + 16 b
constexpr uint32_t kColST = 16;
// Largest thread-block cluster the keys-on-lanes kernel merges a problem's parts in.
constexpr int kMaxClusterT = 16;
// Early start: the roles wait for prev_done, which the waiting warp signals once its
// griddepcontrol.wait returns; the previous kernel may run for long, hence a long bound.
constexpr uint64_t kPrevWaitNs = 20ull * 1000 * 1000 * 1000;

// Per-row sums of a warp's N values per lane (N = 8 or 16) over its 32 lanes.  Each
// halving step keeps half of a lane's values (lane bit 4 picks the upper half, then bit
// 3, ...) and adds its partner's; the lanes then sum the rest of the warp.  Afterwards
// lane i * (32 / N) + j, j < 32 / N, holds the sum of value i.  Fixed order: the sums
// are deterministic.
template <int N>
__device__ __forceinline__ float warp_row_sums(const float (&v)[N], int lane) {
  float a[N];
#pragma unroll
  for (int i = 0; i < N; ++i) a[i] = v[i];
  int bit = 16;
#pragma unroll
  for (int n = N; n > 1; n >>= 1, bit >>= 1) {
    const bool hi = lane & bit;
#pragma unroll
    for (int i = 0; i < n / 2; ++i)
      a[i] = (hi ? a[i + n / 2] : a[i]) + __shfl_xor_sync(0xffffffffu, hi ? a[i] : a[i + n / 2], bit);
  }
#pragma unroll
  for (int b = (32 / N) / 2; b >= 1; b >>= 1) a[0] += __shfl_xor_sync(0xffffffffu, a[0], b);
  return a[0];
}

// RT: query rows handled (8 or 16; rows up to RT of the 16-row tile).  NG: softmax row
// groups -- 1: four softmax warps, each thread all RT rows of its key; 2: eight warps, two
// per TMEM lane quarter, group g taking rows g RT/2 .. (g + 1) RT/2 - 1 of the same keys.
// Warps: 0 the K/V producer (lane 0) and the Q loader (lane 1), 1 the MMA issuer, 2 ..
// 1 + 4 NG the softmax, 2 + 4 NG the waiting warp.  griddepcontrol.wait stalls every lane
// of the warp that runs it, so with an early start only the waiting warp runs it (then
// copies the appended rows); the other roles wait for its prev_done signal, each only
// where it needs the previous kernel's writes, and keep streaming K/V until then.
template <int RT, int NG>
__global__ void __launch_bounds__(96 + 128 * NG, 1)
attn_tq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_k16,
               const __grid_constant__ CUtensorMap tm_v16, const AttnArgs a) {
  constexpr int D = 128;
  constexpr int RTT = RT / NG;        // query rows per softmax thread
  constexpr int NSM = 128 * NG;       // softmax threads
  using C = CfgT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sP = sQ + C::Q_BYTES;
  const uint32_t sKV = sQ + C::KV_OFF;
  CtlT* ctl = reinterpret_cast<CtlT*>(smem + C::KV_OFF + STAGES * C::ST_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    // the tensor maps are kernel parameters: fetch them while the barriers are set up
    // (and, launched early, while the previous kernel finishes)
    tc::prefetch_tmap(&tm_q);
    tc::prefetch_tmap(&tm_k);
    tc::prefetch_tmap(&tm_v);
    tc::prefetch_tmap(&tm_k16);
    tc::prefetch_tmap(&tm_v16);
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(&ctl->kv_full[s], 1);
      tc::mbar_init(&ctl->kv_empty[s], 1);
    }
    tc::mbar_init(&ctl->q_full, 1);
    tc::mbar_init(&ctl->q_empty, 1);
    tc::mbar_init(&ctl->done, 1);
    for (int i = 0; i < NSB; ++i) {
      tc::mbar_init(&ctl->s_full[i], 1);
      tc::mbar_init(&ctl->p_full[i], NSM);
      tc::mbar_init(&ctl->s_free[i], 1);
    }
    tc::mbar_init(&ctl->o_ready, 1);
    tc::mbar_init(&ctl->o_free, NSM);
    tc::mbar_init(&ctl->pub, NSM);
    tc::mbar_init(&ctl->flag, 1);
    tc::mbar_init(&ctl->nr_ready, 30);
    tc::mbar_init(&ctl->prev_done, 1);
    for (int g = 0; g < NG; ++g) {
      tc::mbar_init(&ctl->xmax[g][0], 128);
      tc::mbar_init(&ctl->xmax[g][1], 128);
      tc::mbar_init(&ctl->xsum[g], 128);
    }
    ctl->abort_flag = 0;
    ctl->consumed = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    __syncwarp();
    tc::tmem_alloc(&ctl->tmem, kTmemColsT);
    tc::tmem_relinquish();
  }
  if (!a.early) {
    pdl_wait();
    pdl_trigger();
  }
  if (threadIdx.x == 0) {
    int sum = 0;
    for (int b = 0; b < a.B; ++b) {
      ctl->tiles_b[b] = seq_tiles(a, b, blockIdx.x == 0);
      ctl->len_b[b] = a.len[b];
      ctl->pre_b[b] = a.Hkv * sum;
      sum += ctl->tiles_b[b];
    }
    ctl->tl = a.Hkv * sum;
    ctl->tb = a.row_begin / TK;
    ctl->total = a.L * ctl->tl;
    ctl->per = ctl->total > 0 ? (ctl->total + gridDim.x - 1) / gridDim.x : 1;
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = ctl->tmem;
  volatile int* abort_flag = &ctl->abort_flag;
  // this CTA's slice [g0, g1) of the flat (problem, tile) sequence
  int g0, g1;
  if (a.parts > 0) {  // part r of problem p: tiles [r nt / k, (r + 1) nt / k), k = min(parts, nt)
    const int p = blockIdx.x / a.parts, r = blockIdx.x % a.parts;
    const int h = p % a.Hkv, b = (p / a.Hkv) % a.B, l = p / (a.Hkv * a.B);
    const int nt = l < a.L ? ctl->tiles_b[b] : 0;
    const int k = min(a.parts, nt);
    const int start = l < a.L ? l * ctl->tl + ctl->pre_b[b] + h * nt : ctl->total;
    g0 = start + (r < k ? r * nt / k : nt);
    g1 = start + (r < k ? (r + 1) * nt / k : nt);
  } else {
    g0 = min(ctl->total, (int)blockIdx.x * ctl->per);
    g1 = min(ctl->total, g0 + ctl->per);
  }

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producers
    if (lane == 0 && g0 < g1) {
      Iter it;
      iter_seek(it, ctl, a, g0, g1);
      int kv = 0;
      bool rows_ready = a.k_new == nullptr;
      bool waited = !a.early;
      while (it.g < it.g_end) {
        const int prob = (it.l * a.B + it.b) * a.Hkv + it.h;
        const int s = kv % STAGES;
        const int tabs = it.t + ctl->tb;
        if (!waited && (tabs + 1) * TK > ctl->len_b[it.b] + a.new_off - 1) {
          // this tile holds rows the previous kernel may write
          if (!tc::mbar_wait(&ctl->prev_done, 0, abort_flag, a.err, kPrevWaitNs)) break;
          waited = true;
        }
        if (!rows_ready) {
          const int p0 = ctl->len_b[it.b] + a.new_off;
          if (tabs * TK < p0 + a.new_rows && p0 < (tabs + 1) * TK) {
            if (!tc::mbar_wait(&ctl->nr_ready, 0, abort_flag, a.err)) break;
            rows_ready = true;
          }
        }
        if (!tc::mbar_wait(&ctl->kv_empty[s], ((kv / STAGES) & 1) ^ 1, abort_flag, a.err)) break;
        if (!STD_DCHECK(tabs * TK < a.cap && prob < a.L * a.B * a.Hkv, a.err)) break;
        const int row = prob * (int)a.cap + tabs * TK;
        const uint32_t st = sKV + s * C::ST_BYTES;
        const int nvalid = min(ctl->len_b[it.b] + a.len_off + a.nq - 1, a.row_end) - tabs * TK;
        if (nvalid >= TK) {
          tc::mbar_expect_tx(&ctl->kv_full[s], C::ST_BYTES);
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb) {
            tc::tma_load_2d(st + kb * TK * 128, &tm_k, kb * 64, row, &ctl->kv_full[s]);
            tc::tma_load_2d(st + C::T_BYTES + kb * TK * 128, &tm_v, kb * 64, row, &ctl->kv_full[s]);
          }
        } else {
          const int nb = (nvalid + 15) >> 4;
          tc::mbar_expect_tx(&ctl->kv_full[s], (uint32_t)nb * 16 * 128 * C::KB * 2);
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb) {
            for (int i = 0; i < nb; ++i) {
              tc::tma_load_2d(st + kb * TK * 128 + i * 16 * 128, &tm_k16, kb * 64, row + i * 16, &ctl->kv_full[s]);
              tc::tma_load_2d(st + C::T_BYTES + kb * TK * 128 + i * 16 * 128, &tm_v16, kb * 64, row + i * 16,
                              &ctl->kv_full[s]);
            }
          }
        }
        ++kv;
        iter_next(it, ctl, a);
      }
      if (*abort_flag) {
        for (int k = *(volatile int*)&ctl->consumed; k < kv; ++k) drain_wait(&ctl->kv_full[k % STAGES], (k / STAGES) & 1);
      }
    } else if (lane == 1 && g0 < g1) {
      // ---------------------------------------------------------- Q loader (one 16-row box
      // per segment; with an early start but no early Q, after the previous kernel)
      Iter it;
      iter_seek(it, ctl, a, g0, g1);
      int seg = 0;
      bool waited = !a.early || (a.early & STD_ATTN_EARLY_Q);
      while (it.g < it.g_end) {
        if (it.first) {
          if (!waited) {
            if (!tc::mbar_wait(&ctl->prev_done, 0, abort_flag, a.err, kPrevWaitNs)) break;
            waited = true;
          }
          if (!tc::mbar_wait(&ctl->q_empty, (seg & 1) ^ 1, abort_flag, a.err)) break;
          tc::mbar_expect_tx(&ctl->q_full, C::Q_BYTES);
          const int qrow = ((it.l * a.B + it.b) * a.Hq + it.h * a.G) * a.nq;
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb) tc::tma_load_2d(sQ + kb * 16 * 128, &tm_q, kb * 64, qrow, &ctl->q_full);
          ++seg;
        }
        iter_next(it, ctl, a);
      }
      if (*abort_flag && seg > 0) drain_wait(&ctl->q_full, (seg - 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && g0 < g1) {
      constexpr uint32_t idS = tc::idesc_bf16(128, 16);               // S^T: M = keys, N = query rows
      constexpr uint32_t idPV = tc::idesc_bf16(128, 16) | (1u << 15);  // O^T: A = V^T read MN-major
      Iter it;
      iter_seek(it, ctl, a, g0, g1);
      int seg = -1, kv = 0, u = 0;
      int pu = -1, ps = 0, pseg = 0;
      bool pfirst = false, any = false, ok = true;
      auto issue_pv = [&](int vu, int vs, bool vfirst, bool vlast, int vseg) -> bool {
        const int vb = vu % NSB;
        if (!tc::mbar_wait(&ctl->p_full[vb], (vu / NSB) & 1, abort_flag, a.err)) return false;
        if (vfirst && !tc::mbar_wait(&ctl->o_free, (vseg & 1) ^ 1, abort_flag, a.err)) return false;
        tc::fence_after_sync();
        const uint32_t sp = sP + vb * C::P_BYTES;
        const uint32_t sv = sKV + vs * C::ST_BYTES + C::T_BYTES;
#pragma unroll
        for (int k = 0; k < TK / 16; ++k)
          tc::umma_bf16(tmem, tc::sdesc_sw128_mn(sv + k * 16 * 128, TK * 128),
                        tc::sdesc_sw128(sp + (k >> 2) * 16 * 128 + (k & 3) * 32), idPV,
                        (vfirst && k == 0) ? 0u : 1u);
        tc::umma_commit(&ctl->kv_empty[vs]);
        tc::umma_commit(&ctl->s_free[vb]);
        if (vlast) tc::umma_commit(&ctl->o_ready);
        return true;
      };
      while (it.g < it.g_end) {
        const bool first = it.first, last = iter_last(it);
        if (first) {
          ++seg;
          if (!tc::mbar_wait(&ctl->q_full, seg & 1, abort_flag, a.err)) { ok = false; break; }
        }
        const int s = kv % STAGES;
        if (!tc::mbar_wait(&ctl->kv_full[s], (kv / STAGES) & 1, abort_flag, a.err)) { ok = false; break; }
        *(volatile int*)&ctl->consumed = kv + 1;
        const int bu = u % NSB;
        if (!tc::mbar_wait(&ctl->s_free[bu], ((u / NSB) & 1) ^ 1, abort_flag, a.err)) { ok = false; break; }
        tc::fence_after_sync();
        const uint32_t sk = sKV + s * C::ST_BYTES;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k & 3) * 32;
          tc::umma_bf16(tmem + kColST + bu * 16, tc::sdesc_sw128(sk + (k >> 2) * TK * 128 + off),
                        tc::sdesc_sw128(sQ + (k >> 2) * 16 * 128 + off), idS, k > 0 ? 1u : 0u);
        }
        any = true;
        tc::umma_commit(&ctl->s_full[bu]);
        if (last) tc::umma_commit(&ctl->q_empty);
        if (pu >= 0) {
          if (!issue_pv(pu, ps, pfirst, false, pseg)) { ok = false; break; }
          pu = -1;
        }
        if (last) {
          if (!issue_pv(u, s, first, true, seg)) { ok = false; break; }
        } else {
          pu = u;
          ps = s;
          pfirst = first;
          pseg = seg;
        }
        ++u;
        ++kv;
        iter_next(it, ctl, a);
      }
      if (!ok && any) {
        tc::umma_commit(&ctl->done);
        drain_wait(&ctl->done, 0);
      }
    }
  } else if (warp == 2 + 4 * NG) {
    // ------------------------------------------------------------ waiting warp
    if (a.early) {
      pdl_wait();
      pdl_trigger();  // only after this CTA's wait: the next kernel may start early itself
      if (lane == 0) tc::mbar_arrive(&ctl->prev_done);
    }
    if (lane >= 2 && g0 < g1 && a.k_new != nullptr) {
      // the previous kernel may still read the tile these rows land in: after the wait
      copy_new_rows<D>(a, ctl, g0, g1, lane - 2);
      asm volatile("fence.proxy.async.global;" ::: "memory");
      tc::mbar_arrive(&ctl->nr_ready);
    }
  } else {
    // ------------------------------------------------------------ softmax threads
    const int w = warp & 3;               // TMEM lane quarter of this warp
    const int grp = NG == 1 ? 0 : (warp - 2) >> 2;  // row group
    const int r0 = grp * RTT;                       // the group's first query row
    // value r0 + r of a 16-column load, with compile-time register indices only
    auto pick = [&](const uint32_t(&x)[16], int r) -> uint32_t { return (NG == 2 && grp) ? x[RTT + r] : x[r]; };
    const int tk = w * 32 + lane;         // this thread's key of every tile, and its element of d
    const uint32_t lane_base = tmem + ((uint32_t)(w * 32) << 16);
    const float sc = kLog2e * rsqrtf((float)D);
    const int tid = threadIdx.x - 64;
    // where this thread's P^T elements go: key tk of row r in the 128-byte-swizzled [16][64] block
    const uint32_t p_off = (uint32_t)(tk >> 6) * 16 * 128 + (uint32_t)(tk & 7) * 2;
    const int p_chunk = (tk & 63) >> 3;
    // the P buffers start as zeros: rows RT..15 are never written and must contribute nothing
    for (int i = tid; i < (int)(NSB * C::P_BYTES / 16); i += NSM)
      *reinterpret_cast<uint4*>(smem + C::Q_BYTES + i * 16) = make_uint4(0, 0, 0, 0);
    tc::fence_proxy_async();
    Iter it;
    iter_seek(it, ctl, a, g0, g1);
    int seg = -1, kv = 0, u = 0, npub = 0, nxs = 0;
    float m[RTT], l[RTT];  // this thread's rows r0 + i
    int lim[RTT];
    int lim_max = 0;
#pragma unroll
    for (int r = 0; r < RTT; ++r) {
      m[r] = -INFINITY;
      l[r] = 0.f;
      lim[r] = 0;
    }
    while (it.g < it.g_end) {
      const bool first = it.first, last = iter_last(it);
      const int lb = it.l * a.B + it.b;
      const int prob = lb * a.Hkv + it.h;
      if (first) {
        ++seg;
        const int base = a.len[it.b] + a.len_off;
#pragma unroll
        for (int r = 0; r < RTT; ++r) {
          m[r] = -INFINITY;
          l[r] = 0.f;
          lim[r] = r0 + r < a.rows ? min(base + (r0 + r) % a.nq, a.row_end) : 0;  // keys below lim[r] are attended
        }
        lim_max = min(base + a.nq - 1, a.row_end);
      }
      const int bu = u % NSB;
      const int s = kv % STAGES;
      const int key0 = (it.t + ctl->tb) * TK;
      if (!tc::mbar_wait_warp(&ctl->s_full[bu], (u / NSB) & 1, abort_flag, a.err)) break;
      tc::fence_after_sync();
      if (key0 + TK > lim_max || key0 < a.row_begin) {
        // zero the V rows past the last query's limit and before the range (0 * garbage
        // could be NaN)
        if (!tc::mbar_wait_warp(&ctl->kv_full[s], (kv / STAGES) & 1, abort_flag, a.err)) break;
        const int z0 = max(0, lim_max - key0);
        const int zb = a.row_begin - key0;
        uint8_t* vb = smem + C::KV_OFF + s * C::ST_BYTES + C::T_BYTES;
        for (int i = tid; i < C::KB * TK * 8; i += NSM) {
          const int r = (i >> 3) % TK;
          if (r >= z0 || r < zb)
            *reinterpret_cast<uint4*>(vb + (i / (TK * 8)) * TK * 128 + r * 128 + (i & 7) * 16) = make_uint4(0, 0, 0, 0);
        }
        tc::fence_proxy_async();
      }
      // this thread's key against the query rows
      float v[RTT];
      {
        uint32_t r16[16];
        __syncwarp();
        tc::tmem_ld_x16(lane_base + kColST + bu * 16, r16);
        tc::tmem_ld_wait16(r16);
        const int kc = key0 + tk;
        const bool in_range = kc >= a.row_begin;
#pragma unroll
        for (int r = 0; r < RTT; ++r) v[r] = (in_range && kc < lim[r]) ? __uint_as_float(pick(r16, r)) : -INFINITY;
      }
      // row maxima of the tile: per warp (every lane gets them), then across the four warps
      const int par = u & 1;
      {
        float mine = -INFINITY;
#pragma unroll
        for (int r = 0; r < RTT; ++r) {
          const float wm = warp_max_f32(v[r]);
          mine = lane == r ? wm : mine;
        }
        if (lane < RTT) ctl->wmax[par][r0 + lane][w] = mine;
      }
      tc::mbar_arrive(&ctl->xmax[grp][par]);
      if (!tc::mbar_wait_warp(&ctl->xmax[grp][par], (u >> 1) & 1, abort_flag, a.err)) break;
      bool need = false;
      float mt[RTT];
#pragma unroll
      for (int r = 0; r < RTT; ++r) {
        const float4 q4 = *reinterpret_cast<const float4*>(ctl->wmax[par][r0 + r]);
        mt[r] = fmaxf(fmaxf(q4.x, q4.y), fmaxf(q4.z, q4.w));
        // lazy rescale: only when the max grows by more than 2^kTau (the same decision in
        // every thread: all see the same m and mt)
        need |= m[r] != -INFINITY && (mt[r] - m[r]) * sc > kTau;
      }
      if (need) {
        float f[RTT];
#pragma unroll
        for (int r = 0; r < RTT; ++r) {
          const bool resc = m[r] != -INFINITY && (mt[r] - m[r]) * sc > kTau;
          f[r] = resc ? ex2((m[r] - mt[r]) * sc) : 1.f;
          m[r] = resc ? mt[r] : m[r];
        }
        // the previous tile's P V must have landed in O before O is rescaled (u >= 1: a
        // rescale needs an earlier tile of the same segment)
        if (!tc::mbar_wait_warp(&ctl->s_free[(u - 1) % NSB], ((u - 1) / NSB) & 1, abort_flag, a.err)) break;
        tc::fence_after_sync();
        if constexpr (NG == 1) {
          uint32_t o16[16];
          __syncwarp();
          tc::tmem_ld_x16(lane_base, o16);
          tc::tmem_ld_wait16(o16);
#pragma unroll
          for (int r = 0; r < RTT; ++r) o16[r] = __float_as_uint(__uint_as_float(o16[r]) * f[r]);
          __syncwarp();
          tc::tmem_st_x16(lane_base, o16);
        } else {  // only this group's columns: the other group rescales its own
          static_assert(RTT == 4, "two row groups of four rows");
          uint32_t o4[4];
          __syncwarp();
          tc::tmem_ld_x4(lane_base + r0, o4);
          tc::tmem_ld_wait4(o4);
#pragma unroll
          for (int r = 0; r < 4; ++r) o4[r] = __float_as_uint(__uint_as_float(o4[r]) * f[r]);
          __syncwarp();
          tc::tmem_st_x4(lane_base + r0, o4);
        }
        tc::tmem_st_wait();
#pragma unroll
        for (int r = 0; r < RTT; ++r) l[r] *= f[r];
      }
#pragma unroll
      for (int r = 0; r < RTT; ++r) m[r] = m[r] == -INFINITY ? mt[r] : m[r];  // first keys the row sees
      // P^T[r][tk] = 2^(x - m) as bf16 into the tile's P buffer (a row that has seen no key
      // yet has m = -inf and only -inf logits: its P is 2^-inf = 0)
      {
        uint8_t* pb = smem + C::Q_BYTES + bu * C::P_BYTES + p_off;
#pragma unroll
        for (int r = 0; r < RTT; ++r) {
          const float msc = (m[r] == -INFINITY ? 0.f : m[r]) * sc;
          const float p = ex2(fmaf(v[r], sc, -msc));
          l[r] += p;
          const int row = r0 + r;
          *reinterpret_cast<__nv_bfloat16*>(pb + row * 128 + ((p_chunk ^ (row & 7)) << 4)) = __float2bfloat16_rn(p);
        }
      }
      tc::fence_proxy_async();
      tc::fence_before_sync();
      tc::mbar_arrive(&ctl->p_full[bu]);
      if (last) {
        if (!tc::mbar_wait_warp(&ctl->o_ready, seg & 1, abort_flag, a.err)) break;
        tc::fence_after_sync();
        // outputs, partials and merge counters: after the previous kernel
        if (a.early && !tc::mbar_wait_warp(&ctl->prev_done, 0, abort_flag, a.err, kPrevWaitNs)) break;
        // row sums over the 128 key threads
        {
          const float ws = warp_row_sums<RTT>(l, lane);
          if ((lane & (32 / RTT - 1)) == 0) ctl->wsum[r0 + lane / (32 / RTT)][w] = ws;
        }
        tc::mbar_arrive(&ctl->xsum[grp]);
        if (!tc::mbar_wait_warp(&ctl->xsum[grp], nxs & 1, abort_flag, a.err)) break;
        ++nxs;
        float L[RTT];
#pragma unroll
        for (int r = 0; r < RTT; ++r) {
          const float4 q4 = *reinterpret_cast<const float4*>(ctl->wsum[r0 + r]);
          L[r] = (q4.x + q4.y) + (q4.z + q4.w);
        }
        uint32_t o16[16];
        __syncwarp();
        tc::tmem_ld_x16(lane_base, o16);
        tc::tmem_ld_wait16(o16);
        tc::fence_before_sync();
        tc::mbar_arrive(&ctl->o_free);  // O may be reused: the rest reads registers and global memory
        // (m, L) of row tk, for the thread that writes them
        float m_tk = 0.f, L_tk = 0.f;
        const bool own_tk = tk >= r0 && tk < r0 + RTT;  // row tk is one of this group's rows
#pragma unroll
        for (int r = 0; r < RTT; ++r) {
          m_tk = tk == r0 + r ? m[r] : m_tk;
          L_tk = tk == r0 + r ? L[r] : L_tk;
        }
        // the CTAs c0 .. c1 that hold a segment of this problem
        const int start = it.l * ctl->tl + ctl->pre_b[it.b] + it.h * it.nt;
        const int c0 = a.parts > 0 ? prob * a.parts : start / ctl->per;
        const int c1 = a.parts > 0 ? c0 + min(a.parts, it.nt) - 1 : (start + it.nt - 1) / ctl->per;
        const size_t orow0 = (size_t)(lb * a.Hq + it.h * a.G) * a.nq;
        const size_t nslots = (size_t)a.L * a.B * a.Hkv + gridDim.x;
        float* wml = a.ws + nslots * a.rows * D;
        unsigned long long* ctr = reinterpret_cast<unsigned long long*>(wml + nslots * a.rows * 2);
        const int slot = prob + blockIdx.x;
        if (a.cluster > 1) {
          // the problem's parts form a cluster: this part's partial stays in shared memory
          // (K/V stage 0, idle once the segment's last P V has run) for the cluster merge
          float* po = reinterpret_cast<float*>(smem + C::KV_OFF);
#pragma unroll
          for (int r = 0; r < RTT; ++r)
            if (r0 + r < a.rows) po[(r0 + r) * D + tk] = __uint_as_float(pick(o16, r));
          if (own_tk && tk < a.rows) {
            po[RT * D + tk] = m_tk * sc;
            po[RT * D + RT + tk] = L_tk;
          }
        } else if (c0 == c1) {
          // this CTA saw the whole problem: the output (partials: unnormalised, with (m, l))
#pragma unroll
          for (int r = 0; r < RTT; ++r) {
            if (r0 + r < a.rows) {
              const float inv = a.partial ? 1.f : (L[r] > 0.f ? 1.f / L[r] : 0.f);
              a.o[(orow0 + r0 + r) * D + tk] = __uint_as_float(pick(o16, r)) * inv;
            }
          }
          if (a.partial && own_tk && tk < a.rows) {
            a.ml[(orow0 + tk) * 2] = m_tk * rsqrtf((float)D);
            a.ml[(orow0 + tk) * 2 + 1] = L_tk;
          }
        } else {
          if (!STD_DCHECK((size_t)slot < nslots, a.err)) break;
#pragma unroll
          for (int r = 0; r < RTT; ++r)
            if (r0 + r < a.rows) a.ws[((size_t)slot * a.rows + r0 + r) * D + tk] = __uint_as_float(pick(o16, r));
          if (own_tk && tk < a.rows) {
            wml[((size_t)slot * a.rows + tk) * 2] = m_tk * sc;
            wml[((size_t)slot * a.rows + tk) * 2 + 1] = L_tk;
          }
          // publish the partial, count the arrival; the last CTA merges every slot of the
          // problem (the same protocol as the kernel above)
          tc::mbar_arrive(&ctl->pub);
          if (tid == 0) {
            if (!tc::mbar_wait(&ctl->pub, npub & 1, abort_flag, a.err)) break;
            __threadfence();
            ctl->last_flag = arrive_last(ctr + prob, a.epoch, c1 - c0 + 1) ? 1 : 0;
            if (ctl->last_flag) __threadfence();
            tc::mbar_arrive(&ctl->flag);
          }
          if (!tc::mbar_wait(&ctl->flag, npub & 1, abort_flag, a.err)) break;
          ++npub;
          if (ctl->last_flag && STD_DCHECK((size_t)prob + c1 < nslots && c0 <= c1, a.err)) {
            // all NSM softmax threads share the merge
            merge_problem<D, true, NSM>(a.o, a.partial ? a.ml : nullptr, a.ws, wml, a.rows,
                                        (size_t)(prob + c0) * a.rows, c1 - c0 + 1, orow0, tid);
            if (tid == 0) atomicExch(ctr + prob, next_call_counter(a.epoch));
          }
        }
      }
      ++u;
      ++kv;
      iter_next(it, ctl, a);
    }
    if (a.cluster > 1 && seg < 0 && tid < RT) {  // no part of the problem here: an empty partial
      float* po = reinterpret_cast<float*>(smem + C::KV_OFF);
      po[RT * D + tid] = -INFINITY;
      po[RT * D + RT + tid] = 0.f;
    }
    if (a.partial && blockIdx.x == 0 && tid < 128 &&
        (!a.early || tc::mbar_wait(&ctl->prev_done, 0, abort_flag, a.err, kPrevWaitNs))) {
      // partials of a sequence with no key in the range: o = 0, m = -inf, l = 0
      const int per_b = a.Hq * a.nq;
      for (int b = 0; b < a.B; ++b) {
        if (ctl->tiles_b[b] != 0) continue;
        for (int i = tid; i < a.L * per_b * (D / 4); i += 128) {
          const int l_ = i / (per_b * (D / 4)), rem = i % (per_b * (D / 4));
          const size_t orow = (size_t)(l_ * a.B + b) * per_b + rem / (D / 4);
          *reinterpret_cast<float4*>(a.o + orow * D + (rem % (D / 4)) * 4) = make_float4(0.f, 0.f, 0.f, 0.f);
          if (rem % (D / 4) == 0) {
            a.ml[orow * 2] = -INFINITY;
            a.ml[orow * 2 + 1] = 0.f;
          }
        }
      }
    }
  }
  if (a.cluster > 1) {
    // Cluster merge: every CTA of the cluster holds one part of problem blockIdx.x / parts
    // (or an empty partial); rank k's softmax threads combine items [k, k + 1) x rows x D /
    // cluster of the outputs from all parts' shared memory, in rank order (deterministic).
    tc::cluster_sync();
    if (warp >= 2 && warp < 2 + 4 * NG) {
      const int tid = threadIdx.x - 64;
      const int cs = a.cluster;
      const int rank = (int)tc::cluster_ctarank();
      const int p = blockIdx.x / a.parts;
      const size_t orow0 = (size_t)((p / a.Hkv) * a.Hq + (p % a.Hkv) * a.G) * a.nq;
      const uint32_t pb = smem_u32(smem + C::KV_OFF);
      const int items = a.rows * D;
      const int i1 = (rank + 1) * items / cs;
      // outputs after the previous kernel (an early start)
      const bool go = !a.early || tc::mbar_wait(&ctl->prev_done, 0, abort_flag, a.err, kPrevWaitNs);
      for (int i = rank * items / cs + tid; go && i < i1; i += NSM) {
        const int r = i / D, c = i % D;
        float mk[kMaxClusterT];
        float M = -INFINITY;
#pragma unroll
        for (int k = 0; k < kMaxClusterT; ++k) {
          mk[k] = k < cs ? tc::ld_dsmem_f32(tc::dsmem_addr(pb + (RT * D + r) * 4, k)) : -INFINITY;
          M = fmaxf(M, mk[k]);
        }
        float L = 0.f, acc = 0.f;
#pragma unroll
        for (int k = 0; k < kMaxClusterT; ++k) {
          if (mk[k] != -INFINITY) {  // an empty part contributes nothing (its o is not read)
            const float w = ex2(mk[k] - M);
            L += w * tc::ld_dsmem_f32(tc::dsmem_addr(pb + (RT * D + RT + r) * 4, k));
            acc += w * tc::ld_dsmem_f32(tc::dsmem_addr(pb + (r * D + c) * 4, k));
          }
        }
        a.o[(orow0 + r) * D + c] = a.partial ? acc : (L > 0.f ? acc / L : 0.f);
        if (a.partial && c == 0) {
          a.ml[(orow0 + r) * 2] = M * kLn2;
          a.ml[(orow0 + r) * 2 + 1] = L;
        }
      }
    }
    tc::cluster_sync();  // no CTA leaves while another may still read its shared memory
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemColsT);
  }
}

template <int D>
cudaError_t launch(const AttnArgs& a, cudaStream_t s) {
  using C = Cfg<D>;
  // at most 64 query rows per problem (the draft's G rows, the verify's G * (gamma + 1)
  // up to 64): M = 64 MMAs, the spread softmax layout, and 64-row query boxes; at most 16
  // (the draft): every row copied to all four lane quarters, 16-row query boxes
  const bool half = a.rows <= 64;
  const bool split = a.rows <= 16;
  const uint64_t qrows = (uint64_t)a.L * a.B * a.Hq * a.nq;
  const uint64_t krows = (uint64_t)a.L * a.B * a.Hkv * a.cap;
  CUtensorMap tq, tk, tv, tk16, tv16;
  if (!make_tmap_bf16_2d(&tq, a.q, D, qrows, split ? 16 : half ? 64 : 128) ||
      !make_tmap_bf16_2d(&tk, a.k, D, krows, TK) || !make_tmap_bf16_2d(&tv, a.v, D, krows, TK) ||
      !make_tmap_bf16_2d(&tk16, a.k, D, krows, 16) || !make_tmap_bf16_2d(&tv16, a.v, D, krows, 16))
    return cudaErrorInvalidValue;
  // d = 128 with at most 16 rows: the keys-on-lanes kernel; d = 64 keeps the quarter split
  const bool keys_on_lanes = attn_tc_keys_on_lanes(a);
  const int variant = keys_on_lanes ? (a.rows <= 8 ? 3 : 2) : split ? 2 : half ? 1 : 0;
  auto kern = keys_on_lanes ? (a.rows <= 8 ? attn_tq_kernel<8, 2> : attn_tq_kernel<16, 1>)
              : split       ? attn_tc_kernel<D, true, true>
              : half        ? attn_tc_kernel<D, true, false>
                            : attn_tc_kernel<D, false, false>;
  const uint32_t smem_bytes = keys_on_lanes ? CfgT::SMEM : C::SMEM;
  // the shared-memory size is a per-device attribute of each kernel: set it once per device
  static std::atomic<uint64_t> attr_done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << ((dev & 15) * 4 + variant);
  if (!(attr_done.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
    if (e != cudaSuccess) return e;
    attr_done.fetch_or(bit, std::memory_order_release);
  }
  const int threads = keys_on_lanes ? 96 + 128 * (a.rows <= 8 ? 2 : 1) : kThreads;
  // keys-on-lanes kernel with 2 .. 16 parts per problem: each problem's parts form one
  // thread-block cluster (merged in distributed shared memory) if a cluster that large can
  // be resident on this device (asked once per device and kernel)
  int cl = 0;
  if (keys_on_lanes && a.parts >= 2 && a.parts <= kMaxClusterT) {
    static std::atomic<int> cl_max[16][2];  // largest resident cluster + 1; 0: not asked yet
    std::atomic<int>& slot = cl_max[dev & 15][a.rows <= 8 ? 1 : 0];
    int m = slot.load(std::memory_order_acquire);
    if (m == 0) {
      m = 1;
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
        for (int c = kMaxClusterT; c >= 2 && m == 1; c /= 2) {
          cudaLaunchConfig_t cfg = {};
          cfg.gridDim = dim3(c);
          cfg.blockDim = dim3(threads);
          cfg.dynamicSmemBytes = smem_bytes;
          cudaLaunchAttribute at[1];
          at[0].id = cudaLaunchAttributeClusterDimension;
          at[0].val.clusterDim.x = c;
          at[0].val.clusterDim.y = 1;
          at[0].val.clusterDim.z = 1;
          cfg.attrs = at;
          cfg.numAttrs = 1;
          int n = 0;
          if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
            (void)cudaGetLastError();  // a refused query leaves no error behind
          } else if (n > 0) {
            m = c + 1;
          }
        }
      } else {
        (void)cudaGetLastError();
      }
      slot.store(m, std::memory_order_release);
    }
    if (a.parts <= m - 1) cl = a.parts;
  }
  AttnArgs b = a;
  b.cluster = cl;
  if (cl > 1)
    return launch_pdl_cluster(kern, dim3(a.splits), dim3(threads), smem_bytes, s, (unsigned)cl, tq, tk, tv, tk16, tv16,
                              b);
  return launch_pdl(kern, dim3(a.splits), dim3(threads), smem_bytes, s, tq, tk, tv, tk16, tv16, b);
}

}  // namespace

bool attn_tc_keys_on_lanes(const AttnArgs& a) { return a.d == 128 && a.rows <= 16; }

bool attn_tc_supported(const AttnArgs& a) {
  return a.dtype == STD_BF16 && (a.d == 64 || a.d == 128) && a.rows <= 128 && a.B <= kMaxB &&
         (uint64_t)a.L * a.B * a.Hkv * a.cap + TK < (1ull << 31) &&
         (uint64_t)a.L * a.B * a.Hq * a.nq + 128 < (1ull << 31);
}

// partial o, partial (m, l), then one 64-bit merge counter per problem
size_t attn_tc_ws_floats(int probs, int ctas, int rows, int d) {
  const size_t slots = (size_t)probs + ctas;
  return slots * rows * d + slots * rows * 2 + (size_t)probs * 2;
}

// a.splits = number of persistent CTAs.
cudaError_t launch_decode_attn_tc(const AttnArgs& a, cudaStream_t s) {
  return a.d == 128 ? launch<128>(a, s) : launch<64>(a, s);
}

}  // namespace stdb
