// fastmath.cuh -- element-wise helpers shared by the prefill and backward
// kernels: packed fp32 pair arithmetic (sm_100 f32x2 instructions), a
// polynomial 2^x on the FMA pipe, and bf16 pair packing.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

namespace eio {

// Packed fp32 pair arithmetic (sm_100): one instruction for two lanes of work.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// 2^x on the FMA pipe, two lanes at a time: x = j + f with j = rint(x)
// (added to 1.5 * 2^23, whose low mantissa bits then hold j) and f in
// [-1/2, 1/2]; 2^f by a degree-3 minimax polynomial (relative error 7.5e-5,
// Remez exchange, coefficients from gen_exp2_poly.py); j is added to the
// exponent field.  Results below 2^-126 (and -inf inputs) give 0.  A fixed
// share of each tile's exponentials may go here instead of the MUFU unit
// (the prefill kernel's Cfg::kPolyPairs, the backward's kPolyPairsB).
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  const float2 magic = make_float2(12582912.0f, 12582912.0f);
  const float2 xc = make_float2(fmaxf(x.x, -126.0f), fmaxf(x.y, -126.0f));
  const float2 t = fadd2(xc, magic);
  const float2 jf = fadd2(t, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = ffma2(jf, make_float2(-1.0f, -1.0f), xc);
  float2 p = ffma2(make_float2(0.055171669f, 0.055171669f), f, make_float2(0.24261112f, 0.24261112f));
  p = ffma2(p, f, make_float2(0.69326099f, 0.69326099f));
  p = ffma2(p, f, make_float2(0.99992807f, 0.99992807f));
  // Below 2^-126 the result is flushed to zero, as ex2.approx.ftz does; a
  // masked score (-inf) gives exactly 0.
  return make_float2(x.x < -126.0f ? 0.f : __uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     x.y < -126.0f ? 0.f : __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

}  // namespace eio
