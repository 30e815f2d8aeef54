// Device helpers shared by the kernels of the Sparse-to-Dense library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/std_b200.h"

namespace stdb {

// log2(e): softmax is evaluated as 2^(x*log2e - m) with ex2.
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void flag_error(int* err, int bits) {
  if (err) atomicOr(err, bits);
}

// Debug builds (compiled with -DSTD_DEBUG into libstd_b200_debug.so) check, on the device,
// that every index and cache row a kernel is about to use lies inside its buffer: a failed
// check sets STD_DEVERR_DEBUG and the caller skips the access.  Never a trap.  In the
// product build the check is the constant true and costs nothing.
#ifdef STD_DEBUG
__device__ __forceinline__ bool std_dcheck(bool ok, int* err) {
  if (!ok) flag_error(err, STD_DEVERR_DEBUG);
  return ok;
}
#define STD_DCHECK(cond, err) ::stdb::std_dcheck((cond), (err))
#else
#define STD_DCHECK(cond, err) true
#endif

// Programmatic dependent launch: every kernel of the library is launched so
// that it may start while the previous kernel in the stream finishes.  It must
// call pdl_wait() before touching memory a previous kernel writes or reads, and
// calls pdl_trigger() to let the next kernel start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Order-preserving 32-bit key of a float (larger float -> larger key; -0.0 maps like
// +0.0): the radix of the top-K select, and the digit the selection's score pass counts.
__device__ __forceinline__ uint32_t score_order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------- loads
template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte global->shared async copy; src_bytes = 0 zero-fills the destination.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D = A(16x16 bf16, row) * B(16x8 bf16, col) + D, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 2^x on the special-function unit (flushes subnormals; 2^-inf = 0).
// (not volatile: no side effects, so the compiler may schedule, predicate or speculate it)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}
// Maximum of v over the 32 lanes of the warp, in every lane (all lanes must be converged).
__device__ __forceinline__ float warp_max_f32(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// ---------------------------------------------------------------- packed fp32 pairs (sm_100)
// Two fp32 lanes in one 64-bit register: one instruction does both.
typedef unsigned long long f32x2;
__device__ __forceinline__ f32x2 f2_make(float lo, float hi) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_split(f32x2 v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f32x2 f2_fma(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ f32x2 f2_add(f32x2 a, f32x2 b) {
  f32x2 r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x for a pair of x <= 0 on the FMA pipe (used beside ex2() to split the
// exponential work between the special-function unit and the FP32 pipe).
// Method: round x to the nearest integer j with the 1.5 * 2^23 shifter
// (Cody-Waite style reduction, f = x - j in [-1/2, 1/2]), evaluate 2^f with a
// degree-4 polynomial fitted for least relative error on [-1/2, 1/2]
// (iteratively reweighted least squares on 4001 Chebyshev points, our own fit;
// 2.6e-6 relative in exact arithmetic, 2.7e-6 in fp32 Horner steps -- the
// selection scores it feeds are compared at 2e-3), then add j to the exponent
// field.  That last step uses
// (t_bits - bits(1.5 * 2^23)) << 23 == t_bits << 23 (mod 2^32), since the
// shifter's low nine bits are zero.  Inputs below -125 are clamped (result
// ~2e-38, negligible next to the row maximum's 2^0).
__device__ __forceinline__ f32x2 exp2_fma2(f32x2 x) {
  float x0, x1;
  f2_split(x, x0, x1);
  x = f2_make(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const f32x2 t = f2_add(x, f2_make(12582912.f, 12582912.f));
  const f32x2 j = f2_add(t, f2_make(-12582912.f, -12582912.f));
  const f32x2 f = f2_fma(j, f2_make(-1.f, -1.f), x);
  f32x2 p = f2_make(9.570097072e-03f, 9.570097072e-03f);
  p = f2_fma(p, f, f2_make(5.591786329e-02f, 5.591786329e-02f));
  p = f2_fma(p, f, f2_make(2.402474498e-01f, 2.402474498e-01f));
  p = f2_fma(p, f, f2_make(6.931218144e-01f, 6.931218144e-01f));
  p = f2_fma(p, f, f2_make(9.999992614e-01f, 9.999992614e-01f));
  float p0, p1, t0, t1;
  f2_split(p, p0, p1);
  f2_split(t, t0, t1);
  return f2_make(__int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23)),
                 __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23)));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float quad_max(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
  return v;
}
__device__ __forceinline__ float quad_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Byte offset of 16-byte chunk `c` of row `r` in a shared tile whose rows are
// `chunks` x 16 bytes; chunk index XOR (r mod 8) keeps ldmatrix conflict-free.
__device__ __forceinline__ uint32_t swz(int r, int c, int chunks) {
  return static_cast<uint32_t>((r * chunks + (c ^ (r & 7))) * 16);
}

}  // namespace stdb
