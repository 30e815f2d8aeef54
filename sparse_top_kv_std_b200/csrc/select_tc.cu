// Selection scores on the 5th-generation tensor cores (tcgen05), fed by TMA.
//
// Same quantities as select_score.cu ("Methodik" item 4 of the gist.science
// summary: average text-to-visual attention per (layer, KV head)):
//   pass 1  m_r = max_n x_rn,  l_r = sum_n 2^(x_rn - m_r)        x = log2(e) q_r . k_n / sqrt(d)
//   pass 2  score_n = 1/M sum_r 2^(x_rn - m_r) / l_r  = 1/M sum_r 2^(x_rn - m_r - log2 l_r)
//
// Pass 1: CTA = 128 text rows (the MMA M axis) of one (layer, seq, KV head);
//   keys stream through a 3-stage TMA ring in 256-key tiles; S = Q K^T lands
//   in a double-buffered TMEM accumulator (2 x 256 fp32 columns); four
//   epilogue warpgroups each take 64 of every tile's columns, one row per
//   thread with its running max / sum, merged once at the end.
// Pass 2: transposed.  CTA = eight consecutive 256-key blocks of one head; each
//   block's two 128-key halves (M axis) stay in shared memory while the text
//   rows stream through as 128-row chunks (N axis) into four TMEM accumulators
//   (key half x chunk parity); each of the four epilogue warpgroups owns one,
//   so each thread sums half of one key's column in registers, and the two
//   halves meet once per key block in shared memory.
// Warp roles: warp 0 TMA producer, warp 1 TMEM allocator + MMA issuer (one
// elected lane), the rest epilogue warpgroups (TMEM lane quarter = warp % 4):
// four in each pass (576 threads, 4 epilogue warps per SM sub-partition), so
// every SM sub-partition has several epilogue warps to hide the TMEM-load and
// dependency latency; TMEM loads are pipelined one 32-column chunk ahead.  A quarter of the
// exponentials run as a polynomial on the FMA pipe (exp2_fma2) beside the
// special-function unit.
// Every wait is bounded; on a timeout the CTA raises its abort flag, records
// the error, lets in-flight copies and MMAs finish (bounded), frees TMEM and
// returns.  No multicast loads are used.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc100.cuh"

namespace stdb {
namespace {

constexpr int kThreads = 64 + 32 * 16;  // pass 2: producer, MMA, four epilogue warpgroups (576)
constexpr int BM = 128;      // MMA M
constexpr int BN = 256;      // MMA N (keys in pass 1, text rows in pass 2)
constexpr int kMaxRows = 2048;  // G * T supported by pass 2 (row statistics kept in shared memory)
constexpr int kTmemCols = 512;
constexpr int kP1Groups = 4;                      // pass-1 epilogue warpgroups
constexpr int kP1Threads = 64 + 128 * kP1Groups;  // pass 1 launches 576 threads
constexpr int kP1Cols = BN / kP1Groups;           // accumulator columns per pass-1 warpgroup
// Of every 16 pairs of exponentials, these 4 (spread through the chunk so both
// pipes have work at every point of it) run as a polynomial on the FMA pipe,
// the other 12 on the special-function unit.
__host__ __device__ constexpr bool poly_pair(int p) { return (p & 3) == 1; }

struct Ctl {
  uint64_t full[8], empty[8];
  uint64_t qfull, kfull, kempty, done;
  uint64_t accfull[4], accempty[4];
  uint64_t xfull[4], xempty[4];
  uint32_t tmem;
  int abort_flag;
  int consumed, kconsumed;
};

__device__ __forceinline__ bool visual_ok(const ScoreArgs& a, int b, int* nv_out) {
  const int nv = a.nvis[b];
  *nv_out = nv;
  return nv >= 1 && nv <= a.nvis_max && (int64_t)a.prefix + nv + (a.keys_only ? 0 : a.T) <= a.cap;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Wait that ignores the abort flag (used while unwinding), bounded in time.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = tc::globaltimer();
  while (!tc::mbar_try_wait(a, parity)) {
    if (tc::globaltimer() - t0 > tc::kWaitTimeoutNs) return;
  }
}

// Pass-1 epilogue on 32 logits of one row: online max / sum of 2^(x - m).
// Pairs of logits go through packed fp32 instructions; the pairs poly_pair()
// picks take their exponential on the FMA pipe, the rest on the SFU.
template <bool TAIL>
__device__ __forceinline__ void p1_chunk(const uint32_t (&r)[32], int key, int nv, float sc, float& m, float& l) {
  float v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    v[j] = __uint_as_float(r[j]);
    if (TAIL && key + j >= nv) v[j] = -INFINITY;
  }
  float cm = v[0];
#pragma unroll
  for (int j = 1; j < 31; j += 2) cm = max3f(cm, v[j], v[j + 1]);
  cm = fmaxf(cm, v[31]);
  if (cm == -INFINITY) return;  // every key of the chunk is past the visual tokens
  if (cm > m) {
    l *= ex2((m - cm) * sc);
    m = cm;
  }
  const float msc = m * sc;
  const f32x2 scc = f2_make(sc, sc), nm = f2_make(-msc, -msc);
  f32x2 a0 = f2_make(0.f, 0.f), a1 = a0;
#pragma unroll
  for (int p = 0; p < 16; ++p) {
    const f32x2 x = f2_fma(f2_make(v[2 * p], v[2 * p + 1]), scc, nm);
    f32x2 e;
    if (poly_pair(p)) {
      e = exp2_fma2(x);
    } else {
      float x0, x1;
      f2_split(x, x0, x1);
      e = f2_make(ex2(x0), ex2(x1));
    }
    if (p & 1) a1 = f2_add(a1, e); else a0 = f2_add(a0, e);
  }
  float s0, s1, s2, s3;
  f2_split(a0, s0, s1);
  f2_split(a1, s2, s3);
  l += (s0 + s1) + (s2 + s3);
}

// Pass-2 epilogue on 32 logits of one key: sum_r 2^(x_r - m'_r), where
// m'_r = m_r + log2 l_r folds the row normalisation 1 / l_r into the exponent
// (shared memory holds -m'_r).
__device__ __forceinline__ float p2_chunk(const uint32_t (&r)[32], const float* negm, float sc) {
  const f32x2 scc = f2_make(sc, sc);
  f32x2 a0 = f2_make(0.f, 0.f), a1 = a0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {  // 4 rows at a time
    const float4 nm4 = *reinterpret_cast<const float4*>(negm + 4 * q);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int p = 2 * q + h;
      const f32x2 nm = h ? f2_make(nm4.z, nm4.w) : f2_make(nm4.x, nm4.y);
      const f32x2 x = f2_fma(f2_make(__uint_as_float(r[2 * p]), __uint_as_float(r[2 * p + 1])), scc, nm);
      f32x2 e;
      if (poly_pair(p)) {
        e = exp2_fma2(x);
      } else {
        float x0, x1;
        f2_split(x, x0, x1);
        e = f2_make(ex2(x0), ex2(x1));
      }
      if (p & 1) a1 = f2_add(a1, e); else a0 = f2_add(a0, e);
    }
  }
  float s0, s1, s2, s3;
  f2_split(a0, s0, s1);
  f2_split(a1, s2, s3);
  return (s0 + s1) + (s2 + s3);
}

// NCH consecutive 32-column TMEM chunks at `base`, each load issued one chunk ahead of its use.
template <int NCH, typename F>
__device__ __forceinline__ void tmem_sweep(uint32_t base, F&& use) {
  static_assert(NCH % 2 == 0, "chunks go in pairs");
  uint32_t ra[32], rb[32];
  __syncwarp();
  tc::tmem_ld_x32(base, ra);
  tc::tmem_ld_wait(ra);
#pragma unroll
  for (int c = 0; c < NCH; c += 2) {
    __syncwarp();
    tc::tmem_ld_x32(base + (c + 1) * 32, rb);
    use(ra, c);
    tc::tmem_ld_wait(rb);
    if (c + 2 < NCH) {
      __syncwarp();
      tc::tmem_ld_x32(base + (c + 2) * 32, ra);
    }
    use(rb, c + 1);
    if (c + 2 < NCH) tc::tmem_ld_wait(ra);
  }
}

template <int D>
struct P1 {
  static constexpr int KB = D / 64;                  // 128-byte K-blocks per row
  static constexpr int STAGES = D == 128 ? 3 : 6;
  static constexpr uint32_t Q_BYTES = KB * BM * 128;
  static constexpr uint32_t KT_BYTES = KB * BN * 128;
  static constexpr uint32_t SMEM = 1024 + Q_BYTES + STAGES * KT_BYTES + sizeof(Ctl);
  static_assert(SMEM <= 232448, "dynamic shared memory above the 227 KB a CTA may use");
};

template <int D>
__global__ void __launch_bounds__(kP1Threads, 1)
rowstats_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const ScoreArgs a) {
  pdl_wait();  // memory of earlier kernels in the stream is visible from here on
  pdl_trigger();
  using C = P1<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sK = sQ + C::Q_BYTES;
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + C::Q_BYTES + C::STAGES * C::KT_BYTES);

  const int h = blockIdx.y, lb = blockIdx.z, b = lb % a.B;
  const int prob = lb * a.Hkv + h;
  const int M = a.G * a.T;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // pass 2 counts the top digit of every score into this problem's histogram: clear it
  if (a.hist && blockIdx.x == 0 && threadIdx.x < 256) a.hist[(size_t)prob * 256 + threadIdx.x] = 0u;
  int nv;
  if (!visual_ok(a, b, &nv)) {
    if (blockIdx.x == 0 && threadIdx.x == 0)
      flag_error(a.err, nv > a.nvis_max ? STD_DEVERR_NVIS_MAX : STD_DEVERR_K_RANGE);
    return;
  }
  const int ntiles = (nv + BN - 1) / BN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      tc::mbar_init(&ctl->full[s], 1);
      tc::mbar_init(&ctl->empty[s], 1);
    }
    tc::mbar_init(&ctl->qfull, 1);
    tc::mbar_init(&ctl->done, 1);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&ctl->accfull[i], 1);
      tc::mbar_init(&ctl->accempty[i], 128 * kP1Groups);
    }
    ctl->abort_flag = 0;
    ctl->consumed = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    __syncwarp();
    tc::tmem_alloc(&ctl->tmem, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = ctl->tmem;
  volatile int* abort_flag = &ctl->abort_flag;

  if (warp == 0) {
    if (lane == 0) {
      tc::prefetch_tmap(&tm_q);
      tc::prefetch_tmap(&tm_k);
      const int qrow = (lb * a.Hq + h * a.G) * a.T + blockIdx.x * BM;
      tc::mbar_expect_tx(&ctl->qfull, C::Q_BYTES);
#pragma unroll
      for (int kb = 0; kb < C::KB; ++kb) tc::tma_load_2d(sQ + kb * BM * 128, &tm_q, kb * 64, qrow, &ctl->qfull);
      const int krow = prob * (int)a.cap + a.prefix;  // visual key 0
      int issued = 0;
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % C::STAGES;
        const uint32_t ph = (t / C::STAGES) & 1;
        if (!tc::mbar_wait(&ctl->empty[s], ph ^ 1, abort_flag, a.err)) break;
        tc::mbar_expect_tx(&ctl->full[s], C::KT_BYTES);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb)
          tc::tma_load_2d(sK + s * C::KT_BYTES + kb * BN * 128, &tm_k, kb * 64, krow + t * BN, &ctl->full[s]);
        issued = t + 1;
      }
      if (*abort_flag) {  // let the copies still in flight land before the CTA goes away
        drain_wait(&ctl->qfull, 0);
        for (int t = *(volatile int*)&ctl->consumed; t < issued; ++t)
          drain_wait(&ctl->full[t % C::STAGES], (t / C::STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16(BM, BN);
      bool ok = tc::mbar_wait(&ctl->qfull, 0, abort_flag, a.err);
      int t = 0;
      for (; ok && t < ntiles; ++t) {
        const int s = t % C::STAGES;
        const uint32_t ph = (t / C::STAGES) & 1;
        const int buf = t & 1;
        const uint32_t aph = (t >> 1) & 1;
        if (!tc::mbar_wait(&ctl->full[s], ph, abort_flag, a.err)) break;
        *(volatile int*)&ctl->consumed = t + 1;
        if (!tc::mbar_wait(&ctl->accempty[buf], aph ^ 1, abort_flag, a.err)) break;
        tc::fence_after_sync();
        const uint32_t d = tmem + buf * BN;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k & 3) * 32;  // 16-element K step inside the 128-byte row
          const uint32_t qa = sQ + (k >> 2) * BM * 128 + off;
          const uint32_t ka = sK + s * C::KT_BYTES + (k >> 2) * BN * 128 + off;
          tc::umma_bf16(d, tc::sdesc_sw128(qa), tc::sdesc_sw128(ka), idesc, k > 0 ? 1u : 0u);
        }
        tc::umma_commit(&ctl->empty[s]);
        tc::umma_commit(&ctl->accfull[buf]);
      }
      if (*abort_flag && t > 0) {  // MMAs may still read shared memory / write TMEM
        tc::umma_commit(&ctl->done);
        drain_wait(&ctl->done, 0);
      }
    }
  } else {
    const int g = (warp - 2) >> 2;  // warpgroup: which 64 of the 256 columns
    const int q = warp & 3;         // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;
    const float sc = kLog2e * rsqrtf((float)D);
    float m = -INFINITY, l = 0.f;
    for (int t = 0; t < ntiles; ++t) {
      const int buf = t & 1;
      const uint32_t aph = (t >> 1) & 1;
      if (!tc::mbar_wait_warp(&ctl->accfull[buf], aph, abort_flag, a.err)) break;
      tc::fence_after_sync();
      const uint32_t base = tmem + ((uint32_t)(q * 32) << 16) + buf * BN + g * kP1Cols;
      const int key0 = t * BN + g * kP1Cols;
      if (t * BN + BN > nv) {
        tmem_sweep<kP1Cols / 32>(base, [&](const uint32_t(&r)[32], int c) { p1_chunk<true>(r, key0 + c * 32, nv, sc, m, l); });
      } else {
        tmem_sweep<kP1Cols / 32>(base, [&](const uint32_t(&r)[32], int c) { p1_chunk<false>(r, key0 + c * 32, nv, sc, m, l); });
      }
      tc::fence_before_sync();
      tc::mbar_arrive(&ctl->accempty[buf]);
    }
    // every MMA has completed once the last accumulator was read: the Q tile is free
    float2* part = reinterpret_cast<float2*>(smem);
    part[g * BM + row] = make_float2(m * sc, l);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  } else if (warp >= 2 && warp < 6 && !*abort_flag) {
    // merge the warpgroups' column groups of each row: (m, l) in the exp2 domain
    const int row = (warp & 3) * 32 + lane;
    const int r_glob = blockIdx.x * BM + row;
    const float2* part = reinterpret_cast<const float2*>(smem);
    float mm = -INFINITY, ll = 0.f;
#pragma unroll
    for (int gg = 0; gg < kP1Groups; ++gg) mm = fmaxf(mm, part[gg * BM + row].x);
#pragma unroll
    for (int gg = 0; gg < kP1Groups; ++gg) {
      const float2 p = part[gg * BM + row];
      if (p.y > 0.f) ll += p.y * ex2(p.x - mm);
    }
    if (r_glob < M) {
      a.row_m[(size_t)prob * M + r_glob] = mm;
      a.row_l[(size_t)prob * M + r_glob] = ll;
    }
  }
}

constexpr int BN2 = 128;       // text rows per pass-2 chunk (MMA N)
constexpr int kKeyBlocks = 8;  // 256-key blocks one pass-2 CTA walks through

template <int D>
struct P2 {
  static constexpr int KB = D / 64;
  static constexpr int QSTAGES = 4;
  static constexpr uint32_t K_BYTES = KB * 256 * 128;   // 256 keys = two 128-key MMA tiles
  static constexpr uint32_t QC_BYTES = KB * BN2 * 128;  // one chunk of 128 text rows
  static constexpr uint32_t MW_BYTES = kMaxRows * 4;
  static constexpr uint32_t XCH_BYTES = 4 * 128 * 4;  // partial column sums: [key half][slot][key]
  static constexpr uint32_t SMEM = 1024 + K_BYTES + QSTAGES * QC_BYTES + MW_BYTES + XCH_BYTES + sizeof(Ctl);
  static_assert(SMEM <= 232448, "dynamic shared memory above the 227 KB a CTA may use");
};

// Pass 2.  CTA = kKeyBlocks consecutive 256-key blocks of one (layer, seq, KV head);
// each block's two 128-key halves are the M axis of two MMAs per 128-row chunk of
// text queries.  The accumulator of (key half h, chunk parity p) sits at TMEM
// columns (2h + p) * 128, and epilogue warpgroup 2p + h owns it: each thread sums
// one key's column over the chunks of its parity in registers; per key block the
// parity-1 warpgroup leaves its sums in a double-buffered shared-memory slot and
// the parity-0 warpgroup adds them and writes the scores.  The next block's keys
// load while the last chunks are summed.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
colsum_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const ScoreArgs a) {
  pdl_wait();  // memory of earlier kernels in the stream is visible from here on
  pdl_trigger();
  using C = P2<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sK = smem_u32(smem);
  const uint32_t sQ = sK + C::K_BYTES;
  float* negm = reinterpret_cast<float*>(smem + C::K_BYTES + C::QSTAGES * C::QC_BYTES);  // -(m_r + log2 l_r)
  float* xch = reinterpret_cast<float*>(smem + C::K_BYTES + C::QSTAGES * C::QC_BYTES + C::MW_BYTES);
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + C::K_BYTES + C::QSTAGES * C::QC_BYTES + C::MW_BYTES + C::XCH_BYTES);

  // this CTA's counts of the top 8 bits of its scores' order keys (the top-K's first radix
  // pass, done here while the scores are in registers), added to the problem's histogram
  __shared__ uint32_t s_hist[256];
  const int h = blockIdx.y, lb = blockIdx.z, b = lb % a.B;
  const int prob = lb * a.Hkv + h;
  const int M = a.G * a.T;
  const int nch = (M + BN2 - 1) / BN2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int nv;
  if (!visual_ok(a, b, &nv)) return;  // pass 1 flagged it
  const int key_base = blockIdx.x * (kKeyBlocks * 256);
  if (key_base >= nv) return;
  const int nkb = min(kKeyBlocks, (nv - key_base + 255) / 256);
  for (int i = threadIdx.x; i < 256; i += kThreads) s_hist[i] = 0u;  // ordered by the set-up barrier

  // row statistics of this head as -(m_r + log2 l_r); padding rows get -inf (2^-inf = 0 on the
  // SFU, 2^-125 ~ 2e-38 on the FMA pipe: negligible)
  for (int r = threadIdx.x; r < nch * BN2; r += kThreads)
    negm[r] = r < M ? -(a.row_m[(size_t)prob * M + r] + log2f(a.row_l[(size_t)prob * M + r])) : -INFINITY;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::QSTAGES; ++s) {
      tc::mbar_init(&ctl->full[s], 1);
      tc::mbar_init(&ctl->empty[s], 1);
    }
    tc::mbar_init(&ctl->kfull, 1);
    tc::mbar_init(&ctl->kempty, 1);
    tc::mbar_init(&ctl->done, 1);
    for (int i = 0; i < 4; ++i) {
      tc::mbar_init(&ctl->accfull[i], 1);
      tc::mbar_init(&ctl->accempty[i], 128);
      tc::mbar_init(&ctl->xfull[i], 128);
      tc::mbar_init(&ctl->xempty[i], 128);
    }
    ctl->abort_flag = 0;
    ctl->consumed = 0;
    ctl->kconsumed = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    __syncwarp();
    tc::tmem_alloc(&ctl->tmem, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = ctl->tmem;
  volatile int* abort_flag = &ctl->abort_flag;

  if (warp == 0) {
    if (lane == 0) {
      tc::prefetch_tmap(&tm_q);
      tc::prefetch_tmap(&tm_k);
      const int qrow = (lb * a.Hq + h * a.G) * a.T;
      int issued = 0, kissued = 0;
      bool ok = true;
      for (int kbi = 0; ok && kbi < nkb; ++kbi) {
        // the key buffer is free once every MMA of the previous block has completed
        if (kbi > 0 && !tc::mbar_wait(&ctl->kempty, (kbi - 1) & 1, abort_flag, a.err)) break;
        tc::mbar_expect_tx(&ctl->kfull, C::K_BYTES);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb)
          tc::tma_load_2d(sK + kb * 256 * 128, &tm_k, kb * 64, prob * (int)a.cap + a.prefix + key_base + kbi * 256,
                          &ctl->kfull);
        kissued = kbi + 1;
        for (int c = 0; c < nch; ++c) {
          const int qi = kbi * nch + c;
          const int s = qi % C::QSTAGES;
          const uint32_t ph = (qi / C::QSTAGES) & 1;
          if (!tc::mbar_wait(&ctl->empty[s], ph ^ 1, abort_flag, a.err)) {
            ok = false;
            break;
          }
          tc::mbar_expect_tx(&ctl->full[s], C::QC_BYTES);
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb)
            tc::tma_load_2d(sQ + s * C::QC_BYTES + kb * BN2 * 128, &tm_q, kb * 64, qrow + c * BN2, &ctl->full[s]);
          issued = qi + 1;
        }
      }
      if (*abort_flag) {  // let the copies still in flight land before the CTA goes away
        for (int k = *(volatile int*)&ctl->kconsumed; k < kissued; ++k) drain_wait(&ctl->kfull, k & 1);
        for (int qi = *(volatile int*)&ctl->consumed; qi < issued; ++qi)
          drain_wait(&ctl->full[qi % C::QSTAGES], (qi / C::QSTAGES) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16(BM, BN2);
      bool ok = true, issued_any = false;
      for (int kbi = 0; ok && kbi < nkb; ++kbi) {
        if (!tc::mbar_wait(&ctl->kfull, kbi & 1, abort_flag, a.err)) break;
        *(volatile int*)&ctl->kconsumed = kbi + 1;
        for (int c = 0; ok && c < nch; ++c) {
          const int qi = kbi * nch + c;
          const int s = qi % C::QSTAGES;
          const uint32_t ph = (qi / C::QSTAGES) & 1;
          if (!tc::mbar_wait(&ctl->full[s], ph, abort_flag, a.err)) {
            ok = false;
            break;
          }
          *(volatile int*)&ctl->consumed = qi + 1;
#pragma unroll
          for (int blk = 0; blk < 2; ++blk) {
            const int acc = blk * 2 + (qi & 1);
            if (!tc::mbar_wait(&ctl->accempty[acc], ((qi >> 1) & 1) ^ 1, abort_flag, a.err)) {
              ok = false;
              break;
            }
            tc::fence_after_sync();
            const uint32_t d = tmem + acc * BN2;
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              const uint32_t off = (k & 3) * 32;
              const uint32_t ka = sK + (k >> 2) * 256 * 128 + blk * BM * 128 + off;
              const uint32_t qa = sQ + s * C::QC_BYTES + (k >> 2) * BN2 * 128 + off;
              tc::umma_bf16(d, tc::sdesc_sw128(ka), tc::sdesc_sw128(qa), idesc, k > 0 ? 1u : 0u);
            }
            issued_any = true;
            tc::umma_commit(&ctl->accfull[acc]);
          }
          if (!ok) break;
          tc::umma_commit(&ctl->empty[s]);
        }
        if (ok) tc::umma_commit(&ctl->kempty);
      }
      if (*abort_flag && issued_any) {  // MMAs may still read shared memory / write TMEM
        tc::umma_commit(&ctl->done);
        drain_wait(&ctl->done, 0);
      }
    }
  } else {
    const int wg = (warp - 2) >> 2;  // epilogue warpgroup 0..3
    const int blk = wg & 1;          // key half it owns
    const int par = wg >> 1;         // chunk parity it sums (its accumulator: blk * 2 + par)
    const int acc = blk * 2 + par;
    const int q = warp & 3;          // TMEM lane quarter this warp may access
    const int kl = q * 32 + lane;
    const float sc = kLog2e * rsqrtf((float)D);
    const float invM = 1.f / (float)M;
    bool ok = true;
    for (int kbi = 0; ok && kbi < nkb; ++kbi) {
      float colsum = 0.f;
      for (int c = 0; c < nch; ++c) {
        const int qi = kbi * nch + c;
        if ((qi & 1) != par) continue;
        if (!tc::mbar_wait_warp(&ctl->accfull[acc], (qi >> 1) & 1, abort_flag, a.err)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t base = tmem + ((uint32_t)(q * 32) << 16) + acc * BN2;
        float s = 0.f;
        tmem_sweep<4>(base, [&](const uint32_t(&r)[32], int cc) { s += p2_chunk(r, negm + c * BN2 + cc * 32, sc); });
        colsum += s;
        tc::fence_before_sync();
        tc::mbar_arrive(&ctl->accempty[acc]);
      }
      if (!ok) break;
      // the two parities of a key half meet in a double-buffered shared-memory slot
      const int slot = kbi & 1;
      const uint32_t use = (uint32_t)(kbi >> 1) & 1;
      float* x = xch + (blk * 2 + slot) * 128;
      if (par == 1) {
        if (!tc::mbar_wait_warp(&ctl->xempty[blk * 2 + slot], use ^ 1, abort_flag, a.err)) break;
        x[kl] = colsum;
        tc::mbar_arrive(&ctl->xfull[blk * 2 + slot]);
      } else {
        if (!tc::mbar_wait_warp(&ctl->xfull[blk * 2 + slot], use, abort_flag, a.err)) break;
        const float total = colsum + x[kl];
        tc::mbar_arrive(&ctl->xempty[blk * 2 + slot]);
        const int n = key_base + kbi * 256 + blk * BM + kl;
        const bool valid = n < nv && STD_DCHECK(n < a.nvis_max, a.err);
        const float score = total * invM;
        if (valid) a.scores[(size_t)prob * a.nvis_max + n] = score;
        if (a.hist) {  // lanes with the same digit add once, as a group
          const uint32_t digit = valid ? score_order_key(score) >> 24 : 256u;
          const uint32_t peers = __match_any_sync(0xffffffffu, digit);
          if (valid && lane == __ffs(peers) - 1) atomicAdd(&s_hist[digit], (uint32_t)__popc(peers));
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (a.hist) {
    for (int i = threadIdx.x; i < 256; i += kThreads)
      if (s_hist[i]) atomicAdd(&a.hist[(size_t)prob * 256 + i], s_hist[i]);
  }
  if (warp == 1) {
    __syncwarp();
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

}  // namespace

// 2D bf16 tensor map: `rows` rows of `inner` elements, box of 64 x box_rows,
// 128-byte swizzle (the layout the K-major shared-memory descriptors expect).
bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D>
static cudaError_t launch_tc(const ScoreArgs& a, cudaStream_t s) {
  const uint64_t krows = (uint64_t)a.L * a.B * a.Hkv * a.cap;
  const uint64_t qrows = (uint64_t)a.L * a.B * a.Hq * a.T;
  CUtensorMap tk, tq128;
  if (!make_tmap_bf16_2d(&tk, a.k_full, D, krows, BN) || !make_tmap_bf16_2d(&tq128, a.q_text, D, qrows, BM))
    return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(rowstats_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, P1<D>::SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(colsum_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, P2<D>::SMEM);
  if (e != cudaSuccess) return e;
  const int M = a.G * a.T;
  const int passes = a.passes ? a.passes : 3;
  if (passes & 1) {
    e = launch_pdl(rowstats_tc_kernel<D>, dim3((M + BM - 1) / BM, a.Hkv, a.L * a.B), dim3(kP1Threads), P1<D>::SMEM, s,
                   tq128, tk, a);
    if (e != cudaSuccess) return e;
    if (a.causal_text && (e = launch_text_rowstats(a, s)) != cudaSuccess) return e;
  }
  if (!(passes & 2)) return cudaSuccess;
  return launch_pdl(colsum_tc_kernel<D>, dim3((a.nvis_max + kKeyBlocks * 256 - 1) / (kKeyBlocks * 256), a.Hkv,
                                              a.L * a.B),
                    dim3(kThreads), P2<D>::SMEM, s, tq128, tk, a);
}

// tcgen05 path for bf16 operands; cudaErrorNotSupported for shapes it does not cover.
cudaError_t launch_select_scores_tc(const ScoreArgs& a, cudaStream_t s) {
  if (a.dtype != STD_BF16 || (a.d != 64 && a.d != 128)) return cudaErrorNotSupported;
  if (a.G * a.T > kMaxRows) return cudaErrorNotSupported;
  if ((uint64_t)a.L * a.B * a.Hkv * a.cap + 256 >= (1ull << 31)) return cudaErrorNotSupported;
  if ((uint64_t)a.L * a.B * a.Hq * a.T + 256 >= (1ull << 31)) return cudaErrorNotSupported;
  return a.d == 128 ? launch_tc<128>(a, s) : launch_tc<64>(a, s);
}

}  // namespace stdb
