// Shared device helpers of the tree-verify kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tsd.h"

namespace tsd {

// Programmatic dependent launch.  Every kernel of the library is launched with programmatic
// stream serialisation: it may be scheduled while the previous kernel in the stream is still
// running.  pdl_trigger() lets the next kernel be scheduled; pdl_wait() blocks until the previous
// kernel has completed and its writes are visible.  Every kernel calls pdl_wait() on every path
// before it writes anything an earlier kernel may read, and before it reads anything an earlier
// kernel writes, so "previous kernel complete" stays transitive down the stream.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }

// Record a device-detected error for sequence b unless an earlier one is already there.
__device__ __forceinline__ void flag_status(int32_t* status, int b, int code, int detail = 0) {
  atomicCAS(status + b, 0, code | (detail << 8));
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// 16-byte asynchronous global->shared copy; src_bytes = 0 zero-fills without reading.
__device__ __forceinline__ void cp_async_16(void* smem, const void* gmem, int src_bytes) {
  uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// Larger-value-wins argmax merge with the lower index winning ties.
__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

// Paired fp32 arithmetic of sm_100 (two lanes of work per instruction), round to nearest.
__device__ __forceinline__ void padd2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n.reg .b64 ra, rb, rd;\nmov.b64 ra, {%2, %3};\nmov.b64 rb, {%4, %5};\n"
      "add.rn.f32x2 rd, ra, rb;\nmov.b64 {%0, %1}, rd;\n}\n"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void pmul2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n.reg .b64 ra, rb, rd;\nmov.b64 ra, {%2, %3};\nmov.b64 rb, {%4, %5};\n"
      "mul.rn.f32x2 rd, ra, rb;\nmov.b64 {%0, %1}, rd;\n}\n"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void pfma2(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0, float c1) {
  asm("{\n.reg .b64 ra, rb, rc, rd;\nmov.b64 ra, {%2, %3};\nmov.b64 rb, {%4, %5};\nmov.b64 rc, {%6, %7};\n"
      "fma.rn.f32x2 rd, ra, rb, rc;\nmov.b64 {%0, %1}, rd;\n}\n"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
// 2^x by the hardware approximation, results below 2^-126 flushed to zero (a sum whose largest term
// is 1 does not see them); 2^-inf = 0.
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}
// sum over e of 2^((x[e] - m) * (chi + clo)) for 8 values x[e] <= m: x - m in one rounding (exact
// for bf16 logits), the two-term constant applied as d*chi + d*clo, paired instructions.
__device__ __forceinline__ float sum_ex2_8(const float (&x)[8], float m, float chi, float clo) {
  float t0 = 0.f, t1 = 0.f;
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    float d0, d1, u0, u1, a0, a1;
    padd2(d0, d1, x[e], x[e + 1], -m, -m);
    pmul2(u0, u1, d0, d1, clo, clo);
    pfma2(a0, a1, d0, d1, chi, chi, u0, u1);
    padd2(t0, t1, t0, t1, ex2_ftz(a0), ex2_ftz(a1));
  }
  return t0 + t1;
}

// The same sum with the library exp2f for each term (its accuracy where a sampler's decisions are
// compared with an fp64 oracle at tight margins).
__device__ __forceinline__ float sum_exp2f_8(const float (&x)[8], float m, float chi, float clo) {
  float t0 = 0.f, t1 = 0.f;
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    float d0, d1, u0, u1, a0, a1;
    padd2(d0, d1, x[e], x[e + 1], -m, -m);
    pmul2(u0, u1, d0, d1, clo, clo);
    pfma2(a0, a1, d0, d1, chi, chi, u0, u1);
    padd2(t0, t1, t0, t1, exp2f(a0), exp2f(a1));
  }
  return t0 + t1;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Load 8 consecutive logits starting at element `v` of a row (v % 8 == 0, 16-byte aligned row).
template <typename T>
__device__ __forceinline__ void load8(const T* row, int v, float (&x)[8]);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* row, int v, float (&x)[8]) {
  const uint4 w = __ldg(reinterpret_cast<const uint4*>(row + v));
  x[0] = bf16_lo(w.x), x[1] = bf16_hi(w.x), x[2] = bf16_lo(w.y), x[3] = bf16_hi(w.y);
  x[4] = bf16_lo(w.z), x[5] = bf16_hi(w.z), x[6] = bf16_lo(w.w), x[7] = bf16_hi(w.w);
}
template <>
__device__ __forceinline__ void load8<float>(const float* row, int v, float (&x)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(row + v));
  const float4 c = __ldg(reinterpret_cast<const float4*>(row + v + 4));
  x[0] = a.x, x[1] = a.y, x[2] = a.z, x[3] = a.w, x[4] = c.x, x[5] = c.y, x[6] = c.z, x[7] = c.w;
}
__device__ __forceinline__ float load1(const __nv_bfloat16* row, int v) { return __bfloat162float(row[v]); }
__device__ __forceinline__ float load1(const float* row, int v) { return row[v]; }

}  // namespace tsd
