// Split-K flash-decode attention for the sparse draft and the dense verify of
// Sparse-to-Dense decoding ("Methodik" items 2 and 3 of the gist.science
// summary: the draft attends to the selected top-K KV, the verifier attends
// to the full cache, gamma + 1 positions in one pass).
//
// One CTA handles one (split, KV head, layer x sequence).  All query rows that
// read the same KV head -- the G grouped query heads times the nq query
// positions -- are packed into 16-row MMA tiles, so every K/V byte of the
// split is fetched from HBM exactly once and reused from shared memory.
// Keys stream through a 3-stage cp.async pipeline of 64-key tiles stored with
// an XOR swizzle; S = Q K^T and O += P V run on mma.sync (bf16 in, fp32
// accumulate) with an online softmax in the exp2 domain.  Partial (m, l, o)
// of each split go to the workspace and a second kernel merges them.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace stdb {
namespace {

constexpr int TK = 64;      // keys per pipeline tile
constexpr int STAGES = 3;   // cp.async pipeline depth

template <int D, int RT, int KS>
struct Cfg {
  static constexpr int NW = RT * KS;  // warps: RT row tiles x KS key slices
  static constexpr int NT = NW * 32;
  static constexpr int KW = TK / KS;  // keys of a tile each warp handles
  static constexpr int CH = D / 8;    // 16-byte chunks per row
  static constexpr int TILE_BYTES = TK * D * 2;
  static constexpr int PIPE_BYTES = STAGES * 2 * TILE_BYTES;
  static constexpr int MERGE_BYTES = NW * 16 * (D + 2) * 4;
  static constexpr int SMEM = PIPE_BYTES > MERGE_BYTES ? PIPE_BYTES : MERGE_BYTES;
  static_assert(KW % 16 == 0, "each warp needs whole 16-key MMA steps");
};

struct Range {
  int base;     // key limit of query position 0
  int lim_max;  // key limit of the last query position
  int k_begin, k_end;
  bool bad;
};

__device__ __forceinline__ Range split_range(const AttnArgs& a, int b, int split, int tile) {
  Range r;
  r.base = a.len[b] + a.len_off;
  r.lim_max = r.base + a.nq - 1;
  r.bad = (r.base <= 0) || ((int64_t)r.lim_max > a.cap);
  int lim = r.bad ? 0 : r.lim_max;
  int chunk = ((lim + a.splits - 1) / a.splits + tile - 1) / tile * tile;
  r.k_begin = split * chunk;
  r.k_end = min(r.k_begin + chunk, lim);
  return r;
}

// Final write of one (row, column pair): normalised output when the call has
// one split, else the unnormalised partial and (m, l).
__device__ __forceinline__ void store_pair(const AttnArgs& a, int prob, int lb, int h, int split,
                                           int rows_pad, int row, int col, float o0, float o1,
                                           float m, float l) {
  if (a.splits == 1) {
    if (row >= a.rows) return;
    float inv = l > 0.f ? 1.f / l : 0.f;
    float* dst = a.o + ((size_t)(lb * a.Hq + h * a.G) * a.nq + row) * a.d + col;
    *reinterpret_cast<float2*>(dst) = make_float2(o0 * inv, o1 * inv);
  } else {
    size_t slot = ((size_t)prob * a.splits + split) * rows_pad + row;
    *reinterpret_cast<float2*>(a.ws + slot * a.d + col) = make_float2(o0, o1);
    if (col == 0) {
      float* ml = a.ws + (size_t)a.B * a.L * a.Hkv * a.splits * rows_pad * a.d;
      ml[slot * 2] = m;
      ml[slot * 2 + 1] = l;
    }
  }
}

template <int D, int RT, int KS>
__global__ void __launch_bounds__(Cfg<D, RT, KS>::NT)
attn_bf16_kernel(const AttnArgs a) {
  pdl_wait();  // memory of earlier kernels in the stream is visible from here on
  pdl_trigger();
  using C = Cfg<D, RT, KS>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int split = blockIdx.x, h = blockIdx.y, lb = blockIdx.z;
  const int b = lb % a.B;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rt = warp % RT, ks = warp / RT;
  const int g = lane >> 2, c = lane & 3;
  const int prob = lb * a.Hkv + h;
  const int rows_pad = RT * 16;

  const Range rg = split_range(a, b, split, TK);
  if (rg.bad && split == 0 && tid == 0) flag_error(a.err, STD_DEVERR_LENGTH);
  const int ntiles = rg.k_begin < rg.k_end ? (rg.k_end - rg.k_begin + TK - 1) / TK : 0;

  const __nv_bfloat16* kp = reinterpret_cast<const __nv_bfloat16*>(a.k) + (size_t)prob * a.cap * D;
  const __nv_bfloat16* vp = reinterpret_cast<const __nv_bfloat16*>(a.v) + (size_t)prob * a.cap * D;
  const __nv_bfloat16* qp =
      reinterpret_cast<const __nv_bfloat16*>(a.q) + (size_t)(lb * a.Hq + h * a.G) * a.nq * D;
  const uint32_t sbase = smem_u32(smem);

  auto load_tile = [&](int t, int st) {
    const int key0 = rg.k_begin + t * TK;
    const uint32_t sk = sbase + st * 2 * C::TILE_BYTES;
    const uint32_t sv = sk + C::TILE_BYTES;
#pragma unroll 4
    for (int i = tid; i < TK * C::CH; i += C::NT) {
      const int r = i / C::CH, ch = i % C::CH;
      const int key = key0 + r;
      const bool ok = key < rg.k_end;
      const size_t off = (size_t)(ok ? key : rg.k_begin) * D + ch * 8;
      cp_async16(sk + swz(r, ch, C::CH), kp + off, ok ? 16 : 0);
      cp_async16(sv + swz(r, ch, C::CH), vp + off, ok ? 16 : 0);
    }
  };

  // Q fragments of this warp's 16 rows (rows past the group are zero).
  const int r0 = rt * 16 + g, r1 = r0 + 8;
  uint32_t qf[D / 16][4];
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const int col = kk * 16 + 2 * c;
    qf[kk][0] = r0 < a.rows ? *reinterpret_cast<const uint32_t*>(qp + (size_t)r0 * D + col) : 0u;
    qf[kk][1] = r1 < a.rows ? *reinterpret_cast<const uint32_t*>(qp + (size_t)r1 * D + col) : 0u;
    qf[kk][2] = r0 < a.rows ? *reinterpret_cast<const uint32_t*>(qp + (size_t)r0 * D + col + 8) : 0u;
    qf[kk][3] = r1 < a.rows ? *reinterpret_cast<const uint32_t*>(qp + (size_t)r1 * D + col + 8) : 0u;
  }
  const int lim0 = rg.base + (r0 < a.rows ? r0 % a.nq : 0);
  const int lim1 = rg.base + (r1 < a.rows ? r1 % a.nq : 0);
  const float sc = kLog2e * rsqrtf((float)D);

  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float oacc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;

#pragma unroll
  for (int t = 0; t < STAGES - 1; ++t) {
    if (t < ntiles) load_tile(t, t);
    cp_async_commit();
  }

  const int kb = ks * C::KW;
  for (int t = 0; t < ntiles; ++t) {
    cp_async_wait<STAGES - 2>();
    __syncthreads();
    {
      const int tn = t + STAGES - 1;
      if (tn < ntiles) load_tile(tn, tn % STAGES);
      cp_async_commit();
    }
    const uint32_t sk = sbase + (t % STAGES) * 2 * C::TILE_BYTES;
    const uint32_t sv = sk + C::TILE_BYTES;
    const int key0 = rg.k_begin + t * TK;

    float s[C::KW / 8][4];
#pragma unroll
    for (int nb = 0; nb < C::KW / 8; ++nb) s[nb][0] = s[nb][1] = s[nb][2] = s[nb][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int nb = 0; nb < C::KW / 8; nb += 2) {
        const int mi = lane >> 3, ri = lane & 7;
        const int row = kb + (nb + (mi >> 1)) * 8 + ri;
        uint32_t x0, x1, x2, x3;
        ldsm_x4(sk + swz(row, kk * 2 + (mi & 1), C::CH), x0, x1, x2, x3);
        mma_bf16_16816(s[nb], qf[kk], x0, x1);
        mma_bf16_16816(s[nb + 1], qf[kk], x2, x3);
      }
    }

    // mask, scale to the exp2 domain, online softmax update
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nb = 0; nb < C::KW / 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int key = key0 + kb + nb * 8 + 2 * c + e;
        s[nb][e] = key < lim0 ? s[nb][e] * sc : -INFINITY;
        s[nb][2 + e] = key < lim1 ? s[nb][2 + e] * sc : -INFINITY;
        mx0 = fmaxf(mx0, s[nb][e]);
        mx1 = fmaxf(mx1, s[nb][2 + e]);
      }
    }
    mx0 = quad_max(mx0);
    mx1 = quad_max(mx1);
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float ref0 = mn0 == -INFINITY ? 0.f : mn0;
    const float ref1 = mn1 == -INFINITY ? 0.f : mn1;
    const float corr0 = ex2(m0 - ref0), corr1 = ex2(m1 - ref1);
    m0 = mn0;
    m1 = mn1;
    l0 *= corr0;
    l1 *= corr1;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      oacc[i][0] *= corr0;
      oacc[i][1] *= corr0;
      oacc[i][2] *= corr1;
      oacc[i][3] *= corr1;
    }

    uint32_t pa[C::KW / 16][4];
#pragma unroll
    for (int kt = 0; kt < C::KW / 16; ++kt) {
      const float p00 = ex2(s[2 * kt][0] - ref0), p01 = ex2(s[2 * kt][1] - ref0);
      const float p10 = ex2(s[2 * kt][2] - ref1), p11 = ex2(s[2 * kt][3] - ref1);
      const float p20 = ex2(s[2 * kt + 1][0] - ref0), p21 = ex2(s[2 * kt + 1][1] - ref0);
      const float p30 = ex2(s[2 * kt + 1][2] - ref1), p31 = ex2(s[2 * kt + 1][3] - ref1);
      l0 += (p00 + p01) + (p20 + p21);
      l1 += (p10 + p11) + (p30 + p31);
      pa[kt][0] = pack_bf16(p00, p01);
      pa[kt][1] = pack_bf16(p10, p11);
      pa[kt][2] = pack_bf16(p20, p21);
      pa[kt][3] = pack_bf16(p30, p31);
    }
#pragma unroll
    for (int kt = 0; kt < C::KW / 16; ++kt) {
#pragma unroll
      for (int db = 0; db < D / 8; db += 2) {
        const int mi = lane >> 3, ri = lane & 7;
        const int row = kb + kt * 16 + (mi & 1) * 8 + ri;
        uint32_t x0, x1, x2, x3;
        ldsm_x4_t(sv + swz(row, db + (mi >> 1), C::CH), x0, x1, x2, x3);
        mma_bf16_16816(oacc[db], pa[kt], x0, x1);
        mma_bf16_16816(oacc[db + 1], pa[kt], x2, x3);
      }
    }
  }
  cp_async_wait<0>();
  l0 = quad_sum(l0);
  l1 = quad_sum(l1);

  if constexpr (KS == 1) {
#pragma unroll
    for (int db = 0; db < D / 8; ++db) {
      const int col = db * 8 + 2 * c;
      store_pair(a, prob, lb, h, split, rows_pad, r0, col, oacc[db][0], oacc[db][1], m0, l0);
      store_pair(a, prob, lb, h, split, rows_pad, r1, col, oacc[db][2], oacc[db][3], m1, l1);
    }
  } else {
    // merge the KS key slices of each row tile through shared memory
    __syncthreads();
    float* mbuf = reinterpret_cast<float*>(smem);           // [NW][16]
    float* lbuf = mbuf + C::NW * 16;                          // [NW][16]
    float* obuf = lbuf + C::NW * 16;                          // [NW][16][D]
    if (c == 0) {
      mbuf[warp * 16 + g] = m0;
      mbuf[warp * 16 + g + 8] = m1;
      lbuf[warp * 16 + g] = l0;
      lbuf[warp * 16 + g + 8] = l1;
    }
#pragma unroll
    for (int db = 0; db < D / 8; ++db) {
      const int col = db * 8 + 2 * c;
      *reinterpret_cast<float2*>(obuf + (warp * 16 + g) * D + col) = make_float2(oacc[db][0], oacc[db][1]);
      *reinterpret_cast<float2*>(obuf + (warp * 16 + g + 8) * D + col) = make_float2(oacc[db][2], oacc[db][3]);
    }
    __syncthreads();
    for (int i = tid; i < RT * 16 * (D / 2); i += C::NT) {
      const int row = i / (D / 2), col = (i % (D / 2)) * 2;
      const int trt = row / 16, rr = row % 16;
      float M = -INFINITY;
#pragma unroll
      for (int k = 0; k < KS; ++k) M = fmaxf(M, mbuf[(k * RT + trt) * 16 + rr]);
      const float ref = M == -INFINITY ? 0.f : M;
      float L = 0.f, o0 = 0.f, o1 = 0.f;
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        const int w = k * RT + trt;
        const float sc_k = ex2(mbuf[w * 16 + rr] - ref);
        L += sc_k * lbuf[w * 16 + rr];
        o0 += sc_k * obuf[(w * 16 + rr) * D + col];
        o1 += sc_k * obuf[(w * 16 + rr) * D + col + 1];
      }
      store_pair(a, prob, lb, h, split, rows_pad, row, col, o0, o1, M, L);
    }
  }
}

// fp32 operands: one warp per query row, lanes over the head dimension, FFMA
// dot products and an online softmax with the accurate exp2f.
template <int D>
__global__ void __launch_bounds__(128) attn_f32_kernel(const AttnArgs a) {
  pdl_wait();  // memory of earlier kernels in the stream is visible from here on
  pdl_trigger();
  constexpr int PER = D / 32;
  const int split = blockIdx.x, h = blockIdx.y, lb = blockIdx.z;
  const int b = lb % a.B;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int prob = lb * a.Hkv + h;
  const Range rg = split_range(a, b, split, 1);
  if (rg.bad && split == 0 && threadIdx.x == 0) flag_error(a.err, STD_DEVERR_LENGTH);
  const float* kp = reinterpret_cast<const float*>(a.k) + (size_t)prob * a.cap * D;
  const float* vp = reinterpret_cast<const float*>(a.v) + (size_t)prob * a.cap * D;
  const float* qp = reinterpret_cast<const float*>(a.q) + (size_t)(lb * a.Hq + h * a.G) * a.nq * D;
  const float sc = kLog2e / sqrtf((float)D);
  for (int row = warp; row < a.rows; row += 4) {
    const int lim = min(rg.k_end, rg.base + row % a.nq);
    float q[PER], o[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      q[j] = qp[(size_t)row * D + lane + 32 * j] * sc;
      o[j] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    for (int key = rg.k_begin; key < lim; ++key) {
      float x = 0.f;
#pragma unroll
      for (int j = 0; j < PER; ++j) x = fmaf(q[j], kp[(size_t)key * D + lane + 32 * j], x);
      x = warp_sum(x);
      const float mn = fmaxf(m, x);
      const float corr = exp2f(m - mn);
      const float p = exp2f(x - mn);
      l = l * corr + p;
#pragma unroll
      for (int j = 0; j < PER; ++j) o[j] = fmaf(p, vp[(size_t)key * D + lane + 32 * j], o[j] * corr);
      m = mn;
    }
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int col = lane + 32 * j;
      if (a.splits == 1) {
        a.o[((size_t)(lb * a.Hq + h * a.G) * a.nq + row) * D + col] = l > 0.f ? o[j] / l : 0.f;
      } else {
        const size_t slot = ((size_t)prob * a.splits + split) * a.rows + row;
        a.ws[slot * D + col] = o[j];
        if (col == 0) {
          float* ml = a.ws + (size_t)a.B * a.L * a.Hkv * a.splits * a.rows * D;
          ml[slot * 2] = m;
          ml[slot * 2 + 1] = l;
        }
      }
    }
  }
}

// Merge split partials: m = max m_s, l = sum l_s 2^(m_s - m), o = sum o_s 2^(m_s - m) / l.
__global__ void __launch_bounds__(128) attn_reduce_kernel(const AttnArgs a, int rows_pad) {
  pdl_wait();  // memory of earlier kernels in the stream is visible from here on
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 4 + warp;
  const int h = blockIdx.y, lb = blockIdx.z;
  if (row >= a.rows) return;
  const int prob = lb * a.Hkv + h;
  const float* ml = a.ws + (size_t)a.B * a.L * a.Hkv * a.splits * rows_pad * a.d;
  const size_t slot0 = (size_t)prob * a.splits * rows_pad + row;
  float M = -INFINITY;
  for (int s = 0; s < a.splits; ++s) M = fmaxf(M, ml[(slot0 + (size_t)s * rows_pad) * 2]);
  const float ref = M == -INFINITY ? 0.f : M;
  float L = 0.f;
  for (int s = 0; s < a.splits; ++s) {
    const size_t slot = slot0 + (size_t)s * rows_pad;
    L += ex2(ml[slot * 2] - ref) * ml[slot * 2 + 1];
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  float* dst = a.o + ((size_t)(lb * a.Hq + h * a.G) * a.nq + row) * a.d;
  for (int col = lane; col < a.d; col += 32) {
    float acc = 0.f;
    for (int s = 0; s < a.splits; ++s) {
      const size_t slot = slot0 + (size_t)s * rows_pad;
      acc += ex2(ml[slot * 2] - ref) * a.ws[slot * a.d + col];
    }
    dst[col] = acc * inv;
  }
}

template <int D, int RT, int KS>
cudaError_t launch_bf16(const AttnArgs& a, cudaStream_t s) {
  using C = Cfg<D, RT, KS>;
  auto kern = attn_bf16_kernel<D, RT, KS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid(a.splits, a.Hkv, a.L * a.B);
  return launch_pdl(kern, grid, dim3(C::NT), C::SMEM, s, a);
}

template <int D>
cudaError_t dispatch_rt(const AttnArgs& a, cudaStream_t s) {
  switch ((a.rows + 15) / 16) {
    case 1: return launch_bf16<D, 1, 4>(a, s);
    case 2: return launch_bf16<D, 2, 2>(a, s);
    case 3: return launch_bf16<D, 3, 1>(a, s);
    case 4: return launch_bf16<D, 4, 1>(a, s);
    case 5: return launch_bf16<D, 5, 1>(a, s);
    case 6: return launch_bf16<D, 6, 1>(a, s);
    case 7: return launch_bf16<D, 7, 1>(a, s);
    case 8: return launch_bf16<D, 8, 1>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int attn_rows_pad(int rows, int dtype) { return dtype == STD_BF16 ? (rows + 15) / 16 * 16 : rows; }

size_t attn_ws_floats(int probs, int splits, int rows, int d, int dtype) {
  if (splits <= 1) return 0;
  const size_t slots = (size_t)probs * splits * attn_rows_pad(rows, dtype);
  return slots * d + slots * 2;
}

cudaError_t launch_decode_attn(const AttnArgs& a, cudaStream_t s) {
  cudaError_t e;
  if (a.dtype == STD_BF16) {
    e = a.d == 128 ? dispatch_rt<128>(a, s) : a.d == 64 ? dispatch_rt<64>(a, s) : cudaErrorInvalidValue;
  } else {
    dim3 grid(a.splits, a.Hkv, a.L * a.B);
    switch (a.d) {
      case 32: e = launch_pdl(attn_f32_kernel<32>, grid, dim3(128), 0, s, a); break;
      case 64: e = launch_pdl(attn_f32_kernel<64>, grid, dim3(128), 0, s, a); break;
      case 96: e = launch_pdl(attn_f32_kernel<96>, grid, dim3(128), 0, s, a); break;
      case 128: e = launch_pdl(attn_f32_kernel<128>, grid, dim3(128), 0, s, a); break;
      default: return cudaErrorInvalidValue;
    }
  }
  if (e != cudaSuccess || a.splits == 1) return e;
  dim3 rgrid((a.rows + 3) / 4, a.Hkv, a.L * a.B);
  return launch_pdl(attn_reduce_kernel, rgrid, dim3(128), 0, s, a, attn_rows_pad(a.rows, a.dtype));
}

}  // namespace stdb
