// Prefill selection scores of Sparse-to-Dense decoding -- mma.sync / FFMA
// kernels: the fp32 path, and the bf16 fallback for shapes the tcgen05 kernels
// of select_tc.cu do not cover (more than 2048 text query rows per KV head).
//
// Prefill selection scores of Sparse-to-Dense decoding ("Methodik" item 4 of
// the gist.science summary: top-K visual KV chosen once at prefill from the
// attention from text tokens to visual tokens, averaged; per layer and head).
//
// For each (layer, sequence, KV head) with M = G * T text query rows and Nv
// visual keys:
//   pass 1  row statistics   m_r = max_n x_rn,  l_r = sum_n 2^(x_rn - m_r)
//   pass 2  column means     score_n = 1/M * sum_r 2^(x_rn - m_r) / l_r
// with x_rn = log2(e) * q_r . k_n / sqrt(d).  The M x Nv logit matrix is never
// stored: pass 2 recomputes it tile by tile.  bf16 operands run on mma.sync
// with fp32 accumulation (same instruction sequence in both passes, so both
// see bit-identical logits); fp32 operands use FFMA loops.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace stdb {
namespace {

constexpr int TKS = 64;  // keys per tile
constexpr int P1_STAGES = 3;

__device__ __forceinline__ bool visual_ok(const ScoreArgs& a, int b, int* nv_out) {
  const int nv = a.nvis[b];
  *nv_out = nv;
  return nv >= 1 && nv <= a.nvis_max && (int64_t)a.prefix + nv + (a.keys_only ? 0 : a.T) <= a.cap;
}

// Q fragments (m16n8k16 A operand) of 16 text rows starting at r_base.
template <int D>
__device__ __forceinline__ void load_qfrag(uint32_t (&qf)[D / 16][4], const __nv_bfloat16* qp,
                                           int r_base, int M, int g, int c) {
  const int r0 = r_base + g, r1 = r0 + 8;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const int col = kk * 16 + 2 * c;
    qf[kk][0] = r0 < M ? *reinterpret_cast<const uint32_t*>(qp + (size_t)r0 * D + col) : 0u;
    qf[kk][1] = r1 < M ? *reinterpret_cast<const uint32_t*>(qp + (size_t)r1 * D + col) : 0u;
    qf[kk][2] = r0 < M ? *reinterpret_cast<const uint32_t*>(qp + (size_t)r0 * D + col + 8) : 0u;
    qf[kk][3] = r1 < M ? *reinterpret_cast<const uint32_t*>(qp + (size_t)r1 * D + col + 8) : 0u;
  }
}

// S(16 x 64) = Q(16 x D) K_tile(64 x D)^T from a swizzled shared tile.
template <int D>
__device__ __forceinline__ void tile_logits(float (&s)[8][4], const uint32_t (&qf)[D / 16][4],
                                            uint32_t sk, int lane) {
#pragma unroll
  for (int nb = 0; nb < 8; ++nb) s[nb][0] = s[nb][1] = s[nb][2] = s[nb][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
    for (int nb = 0; nb < 8; nb += 2) {
      const int mi = lane >> 3, ri = lane & 7;
      const int row = (nb + (mi >> 1)) * 8 + ri;
      uint32_t x0, x1, x2, x3;
      ldsm_x4(sk + swz(row, kk * 2 + (mi & 1), D / 8), x0, x1, x2, x3);
      mma_bf16_16816(s[nb], qf[kk], x0, x1);
      mma_bf16_16816(s[nb + 1], qf[kk], x2, x3);
    }
  }
}

template <int D>
__device__ __forceinline__ void load_ktile(uint32_t sk, const __nv_bfloat16* kp, int key0, int nv,
                                           int tid, int nthreads) {
  constexpr int CH = D / 8;
  for (int i = tid; i < TKS * CH; i += nthreads) {
    const int r = i / CH, ch = i % CH;
    const int key = key0 + r;
    const bool ok = key < nv;
    cp_async16(sk + swz(r, ch, CH), kp + (size_t)(ok ? key : 0) * D + ch * 8, ok ? 16 : 0);
  }
}

// Pass 1: CTA = (64-row block, KV head, layer x sequence); 4 warps x 16 rows;
// streams every visual key of the head through a 3-stage pipeline.
template <int D>
__global__ void __launch_bounds__(128) rowstats_bf16_kernel(const ScoreArgs a) {
  pdl_wait();  // memory of earlier kernels in the stream is visible from here on
  pdl_trigger();
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int TILE = TKS * D * 2;
  const int h = blockIdx.y, lb = blockIdx.z, b = lb % a.B;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, c = lane & 3;
  const int prob = lb * a.Hkv + h;
  const int M = a.G * a.T;
  int nv;
  if (!visual_ok(a, b, &nv)) {
    if (blockIdx.x == 0 && tid == 0) flag_error(a.err, nv > a.nvis_max ? STD_DEVERR_NVIS_MAX : STD_DEVERR_K_RANGE);
    return;
  }
  const __nv_bfloat16* kp = reinterpret_cast<const __nv_bfloat16*>(a.k_full) +
                               ((size_t)prob * a.cap + a.prefix) * D;  // visual key 0
  const __nv_bfloat16* qp = reinterpret_cast<const __nv_bfloat16*>(a.q_text) + (size_t)(lb * a.Hq + h * a.G) * a.T * D;
  const int r_base = blockIdx.x * 64 + warp * 16;
  uint32_t qf[D / 16][4];
  load_qfrag<D>(qf, qp, r_base, M, g, c);
  const float sc = kLog2e * rsqrtf((float)D);
  const uint32_t sbase = smem_u32(smem);
  const int ntiles = (nv + TKS - 1) / TKS;
#pragma unroll
  for (int t = 0; t < P1_STAGES - 1; ++t) {
    if (t < ntiles) load_ktile<D>(sbase + t * TILE, kp, t * TKS, nv, tid, 128);
    cp_async_commit();
  }
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  for (int t = 0; t < ntiles; ++t) {
    cp_async_wait<P1_STAGES - 2>();
    __syncthreads();
    {
      const int tn = t + P1_STAGES - 1;
      if (tn < ntiles) load_ktile<D>(sbase + (tn % P1_STAGES) * TILE, kp, tn * TKS, nv, tid, 128);
      cp_async_commit();
    }
    float s[8][4];
    tile_logits<D>(s, qf, sbase + (t % P1_STAGES) * TILE, lane);
    const int key0 = t * TKS;
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool ok = key0 + nb * 8 + 2 * c + e < nv;
        s[nb][e] = ok ? s[nb][e] * sc : -INFINITY;
        s[nb][2 + e] = ok ? s[nb][2 + e] * sc : -INFINITY;
        mx0 = fmaxf(mx0, s[nb][e]);
        mx1 = fmaxf(mx1, s[nb][2 + e]);
      }
    }
    const float mn0 = fmaxf(m0, quad_max(mx0)), mn1 = fmaxf(m1, quad_max(mx1));
    float t0 = 0.f, t1 = 0.f;
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
      t0 += ex2(s[nb][0] - mn0) + ex2(s[nb][1] - mn0);
      t1 += ex2(s[nb][2] - mn1) + ex2(s[nb][3] - mn1);
    }
    l0 = l0 * ex2(m0 - mn0) + t0;
    l1 = l1 * ex2(m1 - mn1) + t1;
    m0 = mn0;
    m1 = mn1;
  }
  cp_async_wait<0>();
  l0 = quad_sum(l0);
  l1 = quad_sum(l1);
  if (c == 0) {
    const int r0 = r_base + g, r1 = r0 + 8;
    if (r0 < M) { a.row_m[(size_t)prob * M + r0] = m0; a.row_l[(size_t)prob * M + r0] = l0; }
    if (r1 < M) { a.row_m[(size_t)prob * M + r1] = m1; a.row_l[(size_t)prob * M + r1] = l1; }
  }
}

// Pass 2: CTA = (64-key block, KV head, layer x sequence); the key tile stays
// in shared memory while the 4 warps sweep all M text rows 16 at a time.
template <int D>
__global__ void __launch_bounds__(128) colsum_bf16_kernel(const ScoreArgs a) {
  pdl_wait();  // memory of earlier kernels in the stream is visible from here on
  pdl_trigger();
  extern __shared__ __align__(128) uint8_t smem[];
  const int h = blockIdx.y, lb = blockIdx.z, b = lb % a.B;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, c = lane & 3;
  const int prob = lb * a.Hkv + h;
  const int M = a.G * a.T;
  int nv;
  if (!visual_ok(a, b, &nv)) return;  // pass 1 flagged it
  const int key0 = blockIdx.x * TKS;
  if (key0 >= nv) return;
  const __nv_bfloat16* kp = reinterpret_cast<const __nv_bfloat16*>(a.k_full) +
                               ((size_t)prob * a.cap + a.prefix) * D;  // visual key 0
  const __nv_bfloat16* qp = reinterpret_cast<const __nv_bfloat16*>(a.q_text) + (size_t)(lb * a.Hq + h * a.G) * a.T * D;
  const uint32_t sk = smem_u32(smem);
  load_ktile<D>(sk, kp, key0, nv, tid, 128);
  cp_async_commit();
  const float sc = kLog2e * rsqrtf((float)D);
  const float* rm = a.row_m + (size_t)prob * M;
  const float* rl = a.row_l + (size_t)prob * M;
  float col[8][2];
#pragma unroll
  for (int nb = 0; nb < 8; ++nb) col[nb][0] = col[nb][1] = 0.f;
  cp_async_wait<0>();
  __syncthreads();
  for (int rb = warp; rb * 16 < M; rb += 4) {
    uint32_t qf[D / 16][4];
    load_qfrag<D>(qf, qp, rb * 16, M, g, c);
    const int r0 = rb * 16 + g, r1 = r0 + 8;
    const float mr0 = r0 < M ? rm[r0] : 0.f, mr1 = r1 < M ? rm[r1] : 0.f;
    const float il0 = r0 < M ? 1.f / rl[r0] : 0.f, il1 = r1 < M ? 1.f / rl[r1] : 0.f;
    float s[8][4];
    tile_logits<D>(s, qf, sk, lane);
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        col[nb][e] += ex2(fmaf(s[nb][e], sc, -mr0)) * il0 + ex2(fmaf(s[nb][2 + e], sc, -mr1)) * il1;
      }
    }
  }
  // sum over the 8 row groups of the warp, then over the 4 warps
#pragma unroll
  for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float v = col[nb][e];
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      col[nb][e] = v;
    }
  }
  __syncthreads();
  float* cbuf = reinterpret_cast<float*>(smem);  // [4][64], reuses the key tile
  if (g == 0) {
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
      cbuf[warp * 64 + nb * 8 + 2 * c] = col[nb][0];
      cbuf[warp * 64 + nb * 8 + 2 * c + 1] = col[nb][1];
    }
  }
  __syncthreads();
  if (tid < TKS) {
    const int n = key0 + tid;
    if (n < nv) {
      const float tot = (cbuf[tid] + cbuf[64 + tid]) + (cbuf[128 + tid] + cbuf[192 + tid]);
      if (STD_DCHECK(n < a.nvis_max, a.err)) a.scores[(size_t)prob * a.nvis_max + n] = tot / (float)M;
    }
  }
}

// fp32 operands: pass 1 with one thread per text row.
template <int D>
__global__ void __launch_bounds__(128) rowstats_f32_kernel(const ScoreArgs a) {
  pdl_wait();  // memory of earlier kernels in the stream is visible from here on
  pdl_trigger();
  const int h = blockIdx.y, lb = blockIdx.z, b = lb % a.B;
  const int prob = lb * a.Hkv + h;
  const int M = a.G * a.T;
  int nv;
  if (!visual_ok(a, b, &nv)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) flag_error(a.err, nv > a.nvis_max ? STD_DEVERR_NVIS_MAX : STD_DEVERR_K_RANGE);
    return;
  }
  const int r = blockIdx.x * 128 + threadIdx.x;
  if (r >= M) return;
  const float* kp = reinterpret_cast<const float*>(a.k_full) + ((size_t)prob * a.cap + a.prefix) * D;  // visual key 0
  const float* qp = reinterpret_cast<const float*>(a.q_text) + ((size_t)(lb * a.Hq + h * a.G) * a.T + r) * D;
  float q[D];
#pragma unroll
  for (int j = 0; j < D; ++j) q[j] = qp[j];
  const float sc = kLog2e / sqrtf((float)D);
  float m = -INFINITY, l = 0.f;
  for (int n = 0; n < nv; ++n) {
    float x = 0.f;
#pragma unroll
    for (int j = 0; j < D; ++j) x = fmaf(q[j], kp[(size_t)n * D + j], x);
    x *= sc;
    const float mn = fmaxf(m, x);
    l = l * exp2f(m - mn) + exp2f(x - mn);
    m = mn;
  }
  a.row_m[(size_t)prob * M + r] = m;
  a.row_l[(size_t)prob * M + r] = l;
}

// fp32 operands: pass 2 with one thread per visual key.
template <int D>
__global__ void __launch_bounds__(128) colsum_f32_kernel(const ScoreArgs a) {
  pdl_wait();  // memory of earlier kernels in the stream is visible from here on
  pdl_trigger();
  const int h = blockIdx.y, lb = blockIdx.z, b = lb % a.B;
  const int prob = lb * a.Hkv + h;
  const int M = a.G * a.T;
  int nv;
  if (!visual_ok(a, b, &nv)) return;
  const int n = blockIdx.x * 128 + threadIdx.x;
  if (n >= nv) return;
  const float* kp = reinterpret_cast<const float*>(a.k_full) + ((size_t)prob * a.cap + a.prefix + n) * D;
  const float* qp = reinterpret_cast<const float*>(a.q_text) + (size_t)(lb * a.Hq + h * a.G) * a.T * D;
  float k[D];
#pragma unroll
  for (int j = 0; j < D; ++j) k[j] = kp[j];
  const float sc = kLog2e / sqrtf((float)D);
  float acc = 0.f;
  for (int r = 0; r < M; ++r) {
    float x = 0.f;
#pragma unroll
    for (int j = 0; j < D; ++j) x = fmaf(qp[(size_t)r * D + j], k[j], x);
    acc += exp2f(x * sc - a.row_m[(size_t)prob * M + r]) / a.row_l[(size_t)prob * M + r];
  }
  if (STD_DCHECK(n < a.nvis_max, a.err)) a.scores[(size_t)prob * a.nvis_max + n] = acc / (float)M;
}

template <int D>
cudaError_t launch_bf16_scores(const ScoreArgs& a, cudaStream_t s) {
  const int M = a.G * a.T;
  constexpr int smem1 = P1_STAGES * TKS * D * 2;
  cudaError_t e = cudaFuncSetAttribute(rowstats_bf16_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem1);
  if (e != cudaSuccess) return e;
  const int passes = a.passes ? a.passes : 3;
  if ((passes & 1) &&
      (e = launch_pdl(rowstats_bf16_kernel<D>, dim3((M + 63) / 64, a.Hkv, a.L * a.B), dim3(128), smem1, s, a)) != cudaSuccess)
    return e;
  if ((passes & 1) && a.causal_text && (e = launch_text_rowstats(a, s)) != cudaSuccess) return e;
  if (!(passes & 2)) return cudaSuccess;
  constexpr int smem2 = TKS * D * 2;
  return launch_pdl(colsum_bf16_kernel<D>, dim3((a.nvis_max + TKS - 1) / TKS, a.Hkv, a.L * a.B), dim3(128), smem2, s, a);
}

template <int D>
cudaError_t launch_f32_scores(const ScoreArgs& a, cudaStream_t s) {
  const int M = a.G * a.T;
  const int passes = a.passes ? a.passes : 3;
  cudaError_t e = cudaSuccess;
  if ((passes & 1) &&
      (e = launch_pdl(rowstats_f32_kernel<D>, dim3((M + 127) / 128, a.Hkv, a.L * a.B), dim3(128), 0, s, a)) != cudaSuccess)
    return e;
  if ((passes & 1) && a.causal_text && (e = launch_text_rowstats(a, s)) != cudaSuccess) return e;
  if (!(passes & 2)) return cudaSuccess;
  return launch_pdl(colsum_f32_kernel<D>, dim3((a.nvis_max + 127) / 128, a.Hkv, a.L * a.B), dim3(128), 0, s, a);
}

}  // namespace

cudaError_t launch_select_scores(const ScoreArgs& a, cudaStream_t s, bool* hist_done) {
  *hist_done = false;
  if (a.dtype == STD_BF16) {
    const cudaError_t e = launch_select_scores_tc(a, s);  // tensor-core path
    if (e != cudaErrorNotSupported) {
      *hist_done = e == cudaSuccess && a.hist != nullptr;
      return e;
    }
    if (a.d == 128) return launch_bf16_scores<128>(a, s);
    if (a.d == 64) return launch_bf16_scores<64>(a, s);
  } else {
    switch (a.d) {
      case 32: return launch_f32_scores<32>(a, s);
      case 64: return launch_f32_scores<64>(a, s);
      case 96: return launch_f32_scores<96>(a, s);
      case 128: return launch_f32_scores<128>(a, s);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace stdb
