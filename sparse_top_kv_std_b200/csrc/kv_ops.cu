// Cache bookkeeping and acceptance of Sparse-to-Dense decoding (gist.science
// summary, "Methodik" items 3 and 4): gather of the selected KV into the
// compacted sparse cache, appends of new rows, greedy longest-prefix
// acceptance with one bonus token, and the commit that appends the accepted
// inputs to the context.  Row copies move 16-byte vectors, one warp per row.
#include "common.cuh"
#include "internal.h"

namespace stdb {
namespace {

constexpr int ROWS_PER_CTA = 8;  // one warp per row

__device__ __forceinline__ void copy_row(uint8_t* dst, const uint8_t* src, int bytes, int lane) {
  for (int off = lane * 16; off < bytes; off += 32 * 16)
    *reinterpret_cast<uint4*>(dst + off) = *reinterpret_cast<const uint4*>(src + off);
}

__device__ __forceinline__ void zero_row(uint8_t* dst, int bytes, int lane) {
  for (int off = lane * 16; off < bytes; off += 32 * 16) *reinterpret_cast<uint4*>(dst + off) = make_uint4(0, 0, 0, 0);
}

// Sparse cache rows [0, K) <- full rows idx[0..K); rows [K, K + T) <- text rows.
__global__ void __launch_bounds__(ROWS_PER_CTA * 32) gather_kernel(const GatherArgs a) {
  pdl_wait();  // memory of earlier kernels in the stream is visible from here on
  pdl_trigger();
  const int h = blockIdx.y, lb = blockIdx.z, b = lb % a.B;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * ROWS_PER_CTA + warp;
  const int prob = lb * a.Hkv + h;
  const int nv = a.nvis[b];
  // (a part holds only [part_pos0, part_pos0 + part_rows) of the cache: no extent check here)
  if (a.K > nv || (a.part_rows == 0 && (int64_t)a.prefix + nv + a.T > a.cap_full)) {
    if (j == 0 && h == 0 && lane == 0) flag_error(a.err, STD_DEVERR_K_RANGE);
    return;
  }
  if (j >= a.prefix + a.K + a.T) return;
  int src;  // full-cache row: [prefix | visual | text] -> sparse [prefix | K selected | text]
  if (j < a.prefix) {
    src = j;
  } else if (j < a.prefix + a.K) {
    src = a.idx[(size_t)prob * a.K + (j - a.prefix)];
    if (src < 0 || src >= nv) {  // an index outside the visual block
      if (lane == 0) flag_error(a.err, STD_DEVERR_K_RANGE);
      return;
    }
    src += a.prefix;
  } else {
    src = a.prefix + nv + (j - a.prefix - a.K);
  }
  const size_t dof = ((size_t)prob * a.cap_sparse + j) * a.row_bytes;
  if (a.part_rows > 0) {
    if (src < a.part_pos0 || src >= a.part_pos0 + a.part_rows) {  // another part's row: zeros here
      zero_row(static_cast<uint8_t*>(a.k_sp) + dof, a.row_bytes, lane);
      zero_row(static_cast<uint8_t*>(a.v_sp) + dof, a.row_bytes, lane);
      if (blockIdx.x == 0 && h == 0 && blockIdx.z / a.B == 0 && threadIdx.x == 0) a.len_sparse[b] = a.prefix + a.K + a.T;
      return;
    }
    src -= (int)a.part_pos0;
  }
  if (!STD_DCHECK(src >= 0 && src < a.cap_full && j < a.cap_sparse, a.err)) return;
  const size_t so = ((size_t)prob * a.cap_full + src) * a.row_bytes;
  copy_row(static_cast<uint8_t*>(a.k_sp) + dof, static_cast<const uint8_t*>(a.k_full) + so, a.row_bytes, lane);
  copy_row(static_cast<uint8_t*>(a.v_sp) + dof, static_cast<const uint8_t*>(a.v_full) + so, a.row_bytes, lane);
  if (blockIdx.x == 0 && h == 0 && blockIdx.z / a.B == 0 && threadIdx.x == 0) a.len_sparse[b] = a.prefix + a.K + a.T;
}

// cache rows len[b] + off + r <- new rows r (r < n_new).
__global__ void __launch_bounds__(ROWS_PER_CTA * 32)
append_kernel(uint8_t* kc, uint8_t* vc, int64_t cap, const int32_t* len, int off,
              const uint8_t* kn, const uint8_t* vn, int n_new, int B, int Hkv, int row_bytes, int* err) {
  pdl_wait();  // memory of earlier kernels in the stream is visible from here on
  pdl_trigger();
  const int h = blockIdx.y, lb = blockIdx.z, b = lb % B;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * ROWS_PER_CTA + warp;
  if (r >= n_new) return;
  const int64_t pos0 = (int64_t)len[b] + off;
  if (pos0 < 0 || pos0 + n_new > cap) {
    if (r == 0 && h == 0 && lane == 0) flag_error(err, STD_DEVERR_CAPACITY);
    return;
  }
  const int prob = lb * Hkv + h;
  if (!STD_DCHECK(pos0 + r < cap, err)) return;
  const size_t dof = ((size_t)prob * cap + pos0 + r) * row_bytes;
  const size_t so = ((size_t)prob * n_new + r) * row_bytes;
  copy_row(kc + dof, kn + so, row_bytes, lane);
  copy_row(vc + dof, vn + so, row_bytes, lane);
}

// sparse rows [len_sp, len_sp + n) <- full rows [len_full, len_full + n).
__global__ void __launch_bounds__(ROWS_PER_CTA * 32)
commit_copy_kernel(const uint8_t* kf, const uint8_t* vf, uint8_t* ks, uint8_t* vs, const int32_t* len_full,
                   const int32_t* len_sp, const int32_t* n_plus_1, int max_n, int B, int Hkv,
                   int row_bytes, int64_t cap_full, int64_t cap_sparse, int* err) {
  pdl_wait();  // memory of earlier kernels in the stream is visible from here on
  pdl_trigger();
  const int h = blockIdx.y, lb = blockIdx.z, b = lb % B;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * ROWS_PER_CTA + warp;
  const int n = n_plus_1[b];
  if (r >= n && r > 0) return;
  const int64_t a0 = len_full[b], s0 = len_sp[b];
  if (n < 0 || n > max_n || a0 < 0 || s0 < 0 || a0 + n > cap_full || s0 + n > cap_sparse) {
    if (r == 0 && h == 0 && lane == 0) flag_error(err, STD_DEVERR_CAPACITY);
    return;
  }
  if (r >= n) return;
  const int prob = lb * Hkv + h;
  if (!STD_DCHECK(a0 + r < cap_full && s0 + r < cap_sparse, err)) return;
  const size_t so = ((size_t)prob * cap_full + a0 + r) * row_bytes;
  const size_t dof = ((size_t)prob * cap_sparse + s0 + r) * row_bytes;
  copy_row(ks + dof, kf + so, row_bytes, lane);
  copy_row(vs + dof, vf + so, row_bytes, lane);
}

// Both lengths advance by n + 1 (after every copy of the commit has read them).
__global__ void commit_len_kernel(int32_t* len_full, int32_t* len_sp, const int32_t* n_plus_1, int max_n,
                                  int B, int64_t cap_full, int64_t cap_sparse) {
  pdl_wait();  // memory of earlier kernels in the stream is visible from here on
  pdl_trigger();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int n = n_plus_1[b];
  if (n < 0 || n > max_n || len_full[b] < 0 || len_sp[b] < 0 || (int64_t)len_full[b] + n > cap_full ||
      (int64_t)len_sp[b] + n > cap_sparse)
    return;  // the copy kernel flagged it
  len_full[b] += n;
  len_sp[b] += n;
}

// One warp per sequence: n = index of the first mismatch (gamma if none).
__global__ void accept_kernel(int B, int gamma, const int32_t* draft, const int32_t* dense,
                              int32_t* n_plus_1, int32_t* accepted) {
  pdl_wait();  // memory of earlier kernels in the stream is visible from here on
  pdl_trigger();
  const int b = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (b >= B) return;
  const bool mismatch = lane < gamma && draft[(size_t)b * gamma + lane] != dense[(size_t)b * (gamma + 1) + lane];
  const uint32_t mm = __ballot_sync(0xffffffffu, mismatch);
  const int n = mm ? __ffs(mm) - 1 : gamma;
  if (lane == 0) n_plus_1[b] = n + 1;
  if (lane <= gamma) accepted[(size_t)b * (gamma + 1) + lane] = lane <= n ? dense[(size_t)b * (gamma + 1) + lane] : -1;
}

}  // namespace

cudaError_t launch_gather(const GatherArgs& a, cudaStream_t s) {
  dim3 grid((a.prefix + a.K + a.T + ROWS_PER_CTA - 1) / ROWS_PER_CTA, a.Hkv, a.L * a.B);
  return launch_pdl(gather_kernel, grid, dim3(ROWS_PER_CTA * 32), 0, s, a);
}

cudaError_t launch_append(void* k_cache, void* v_cache, int64_t cap, const int32_t* len, int off,
                          const void* k_new, const void* v_new, int n_new, int L, int B, int Hkv,
                          int row_bytes, int* err, cudaStream_t s) {
  if (n_new <= 0) return cudaSuccess;
  dim3 grid((n_new + ROWS_PER_CTA - 1) / ROWS_PER_CTA, Hkv, L * B);
  return launch_pdl(append_kernel, grid, dim3(ROWS_PER_CTA * 32), 0, s, static_cast<uint8_t*>(k_cache),
                    static_cast<uint8_t*>(v_cache), cap, len, off, static_cast<const uint8_t*>(k_new),
                    static_cast<const uint8_t*>(v_new), n_new, B, Hkv, row_bytes, err);
}

cudaError_t launch_commit(void* k_full, void* v_full, void* k_sp, void* v_sp, int32_t* len_full,
                          int32_t* len_sp, const int32_t* n_plus_1, int max_n, int L, int B,
                          int Hkv, int row_bytes, int64_t cap_full, int64_t cap_sparse, int* err,
                          cudaStream_t s) {
  dim3 grid((max_n + ROWS_PER_CTA - 1) / ROWS_PER_CTA, Hkv, L * B);
  cudaError_t e = launch_pdl(commit_copy_kernel, grid, dim3(ROWS_PER_CTA * 32), 0, s, static_cast<const uint8_t*>(k_full),
                             static_cast<const uint8_t*>(v_full), static_cast<uint8_t*>(k_sp), static_cast<uint8_t*>(v_sp),
                             len_full, len_sp, n_plus_1, max_n, B, Hkv, row_bytes, cap_full, cap_sparse, err);
  if (e != cudaSuccess) return e;
  return launch_pdl(commit_len_kernel, dim3((B + 127) / 128), dim3(128), 0, s, len_full, len_sp, n_plus_1, max_n, B,
                    cap_full, cap_sparse);
}

cudaError_t launch_accept(int B, int gamma, const int32_t* draft, const int32_t* dense,
                          int32_t* n_plus_1, int32_t* accepted, cudaStream_t s) {
  return launch_pdl(accept_kernel, dim3((B + 3) / 4), dim3(128), 0, s, B, gamma, draft, dense, n_plus_1, accepted);
}

}  // namespace stdb
