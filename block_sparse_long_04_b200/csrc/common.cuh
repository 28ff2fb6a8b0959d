// Shared device helpers for the xattn kernels (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace xattn {

typedef __nv_bfloat16 bf16;

constexpr float kNegInf = -__builtin_huge_valf();
constexpr float kLog2e = 1.4426950408889634f;   // log2(e)
constexpr float kLn2 = 0.6931471805599453f;     // ln(2)

// Per-device error word, raised by kernels for conditions only the device sees
// (list capacity, a bounded wait that ran out); read and cleared by
// xattn_get_device_error.
__device__ int g_device_error;

__device__ __forceinline__ void raise_device_error(int code) {
  atomicCAS(&g_device_error, 0, code);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Hardware base-2 exponential / logarithm (MUFU.EX2 / MUFU.LG2 via PTX).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// max of three fp32 values in one instruction (sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// packed fp32x2 arithmetic (two lanes per instruction, sm_100)
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  unsigned long long ua, ub, uc, ud;
  ua = *reinterpret_cast<unsigned long long*>(&a);
  ub = *reinterpret_cast<unsigned long long*>(&b);
  uc = *reinterpret_cast<unsigned long long*>(&c);
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(ud) : "l"(ua), "l"(ub), "l"(uc));
  return *reinterpret_cast<float2*>(&ud);
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  unsigned long long ua, ub, ud;
  ua = *reinterpret_cast<unsigned long long*>(&a);
  ub = *reinterpret_cast<unsigned long long*>(&b);
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(ud) : "l"(ua), "l"(ub));
  return *reinterpret_cast<float2*>(&ud);
}

// 2^x for two lanes on the FMA and integer pipes instead of MUFU, for x <= 127
// (-inf allowed). Range reduction: n = round-to-nearest(x) via the 1.5 * 2^23
// addition, f = x - n in [-1/2, 1/2], both exact; 2^f = 1 + f(c1 + f(c2 + f c3)),
// the cubic of least maximum relative error on [-1/2, 1/2] with constant term 1
// (fit_exp2_poly.py, relative error 1.01e-4 in fp32); 2^n is added to the
// exponent field as an integer. x is clamped to -127 first, where that sum is
// the bit pattern of +0, so -inf and every x <= -127 give exactly 0.
__device__ __forceinline__ float2 ex2_poly2(float2 x) {
  constexpr float kRound = 12582912.f;   // 1.5 * 2^23
  constexpr float c1 = 0.6932829022407532f, c2 = 0.2422109693288803f,
                  c3 = 0.055009059607982635f;
  x.x = fmaxf(x.x, -127.f);
  x.y = fmaxf(x.y, -127.f);
  const float2 t = fadd2(x, make_float2(kRound, kRound));
  const float2 n = fadd2(t, make_float2(-kRound, -kRound));
  const float2 f = ffma2(n, make_float2(-1.f, -1.f), x);
  float2 p = ffma2(make_float2(c3, c3), f, make_float2(c2, c2));
  p = ffma2(p, f, make_float2(c1, c1));
  p = ffma2(p, f, make_float2(1.f, 1.f));
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

}  // namespace xattn
