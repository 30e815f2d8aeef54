// Causal full-row variant of the selection score.
//
// "Methodik" item 4 of the gist.science summary averages the attention from the
// text tokens to the visual tokens but does not say which keys that softmax runs
// over.  The default reading takes the visual keys only; this variant lets each
// text query see what it sees in the prompt's causal attention: the prompt prefix
// before the video (a system prompt, if any), every visual key and the text keys
// up to its own position.  The visual-key probabilities then carry the other
// keys' share of each row's denominator.
//
// Pass 1 of the selection leaves, per text row r, statistics of its visual logits
// in the exp2 domain: m_r = max_n x_rn and l_r = sum_n 2^(x_rn - m_r), with
// x = log2(e) q . k / sqrt(d).  This kernel adds the keys row r = (g, t) sees
// besides the visual ones -- the rows of a prompt prefix before the video (a
// system prompt), if any, and the text keys 0..t -- to (m_r, l_r); pass 2 then
// turns the merged statistics into visual-key probabilities unchanged.  These
// are a few hundred keys per row (well under 1% of the visual work at the
// long-video shapes), so plain fp32 dot products suffice.
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace stdb {
namespace {

constexpr int kWarps = 8;
constexpr int kRowsPerWarp = 4;
constexpr int kRows = kWarps * kRowsPerWarp;  // text rows per CTA
constexpr int kKeys = 32;                     // extra keys per shared-memory tile: one per lane

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <int D, typename E>
__global__ void __launch_bounds__(kWarps * 32) text_rowstats_kernel(const ScoreArgs a) {
  pdl_wait();  // pass 1's statistics are visible from here on
  pdl_trigger();
  __shared__ __align__(16) float ks[kKeys][D + 4];  // +4: conflict-free float4 reads by row
  __shared__ __align__(16) float qs[kRows][D];
  const int h = blockIdx.y, lb = blockIdx.z, b = lb % a.B;
  const int prob = lb * a.Hkv + h;
  const int M = a.G * a.T;
  const int nv = a.nvis[b];
  if (nv < 1 || nv > a.nvis_max || (int64_t)a.prefix + nv + a.T > a.cap) return;  // pass 1 flagged it
  const int r0 = blockIdx.x * kRows;
  if (r0 >= M) return;
  const int nrows = min(kRows, M - r0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // key j of the extra keys: prefix row j (j < prefix), else text key j - prefix; and
  // query row r0 of the head's G x T text rows
  const E* kpre = static_cast<const E*>(a.k_full) + (size_t)prob * a.cap * D;
  const E* ktext = kpre + ((size_t)a.prefix + nv) * D;
  const E* qbase = static_cast<const E*>(a.q_text) + ((size_t)(lb * a.Hq + h * a.G) * a.T + r0) * D;
  for (int i = threadIdx.x; i < kRows * D; i += blockDim.x) {
    const int r = i / D;
    qs[r][i % D] = r < nrows ? to_f(qbase[(size_t)r * D + i % D]) : 0.f;
  }
  int tmax = 0;  // last text position any of the CTA's rows sees
  for (int r = 0; r < nrows; ++r) tmax = max(tmax, (r0 + r) % a.T);
  const int jend = a.prefix + tmax;  // last extra key any row sees

  const float sc = kLog2e * rsqrtf((float)D);
  float m[kRowsPerWarp], l[kRowsPerWarp];
  int tpos[kRowsPerWarp];  // last extra key (prefix + t) the warp's i-th row sees, -1 past the rows
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    const int r = warp + kWarps * i;
    m[i] = -INFINITY;
    l[i] = 0.f;
    tpos[i] = r < nrows ? a.prefix + (r0 + r) % a.T : -1;
  }
  for (int k0 = 0; k0 <= jend; k0 += kKeys) {
    __syncthreads();  // the previous tile is consumed (and the query rows are written)
    for (int i = threadIdx.x; i < kKeys * D; i += blockDim.x) {
      const int j = i / D;
      const int jj = k0 + j;
      const E* row = jj < a.prefix ? kpre + (size_t)jj * D : ktext + (size_t)(jj - a.prefix) * D;
      ks[j][i % D] = jj <= jend ? to_f(row[i % D]) : 0.f;
    }
    __syncthreads();
    const int j = k0 + lane;  // this lane's extra key
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
      if (j > tpos[i]) continue;  // causal: row (g, t) sees the prefix and text keys 0..t
      const float* qr = qs[warp + kWarps * i];
      float acc = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; c += 4) {
        const float4 qv = *reinterpret_cast<const float4*>(qr + c);
        const float4 kv = *reinterpret_cast<const float4*>(&ks[lane][c]);
        acc = fmaf(qv.x, kv.x, acc);
        acc = fmaf(qv.y, kv.y, acc);
        acc = fmaf(qv.z, kv.z, acc);
        acc = fmaf(qv.w, kv.w, acc);
      }
      const float x = acc * sc;
      if (x > m[i]) {
        l[i] = l[i] * exp2f(m[i] - x) + 1.f;  // l = 0 while m = -inf
        m[i] = x;
      } else {
        l[i] += exp2f(x - m[i]);
      }
    }
  }
  // combine the lanes' (m, l) of each row, then merge them into the visual statistics
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    float mi = m[i], li = l[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, mi, o);
      const float l2 = __shfl_xor_sync(0xffffffffu, li, o);
      const float mm = fmaxf(mi, m2);
      li = (li > 0.f ? li * exp2f(mi - mm) : 0.f) + (l2 > 0.f ? l2 * exp2f(m2 - mm) : 0.f);
      mi = mm;
    }
    if (lane == 0 && tpos[i] >= 0) {
      const size_t at = (size_t)prob * M + r0 + warp + kWarps * i;
      const float mv = a.row_m[at], lv = a.row_l[at];
      const float mm = fmaxf(mv, mi);
      a.row_l[at] = lv * exp2f(mv - mm) + li * exp2f(mi - mm);
      a.row_m[at] = mm;
    }
  }
}

template <int D, typename E>
cudaError_t launch_d(const ScoreArgs& a, cudaStream_t s) {
  const int M = a.G * a.T;
  return launch_pdl(text_rowstats_kernel<D, E>, dim3((M + kRows - 1) / kRows, a.Hkv, a.L * a.B), dim3(kWarps * 32),
                    0, s, a);
}

}  // namespace

cudaError_t launch_text_rowstats(const ScoreArgs& a, cudaStream_t s) {
  if (a.dtype == STD_BF16) {
    if (a.d == 128) return launch_d<128, __nv_bfloat16>(a, s);
    if (a.d == 64) return launch_d<64, __nv_bfloat16>(a, s);
  } else {
    switch (a.d) {
      case 32: return launch_d<32, float>(a, s);
      case 64: return launch_d<64, float>(a, s);
      case 96: return launch_d<96, float>(a, s);
      case 128: return launch_d<128, float>(a, s);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace stdb
