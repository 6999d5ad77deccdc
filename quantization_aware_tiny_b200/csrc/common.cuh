// Shared device/host helpers of the sm_100a library (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/qat.h"

namespace qat {

// ~2 s: the limit after which any device-side wait gives up.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

// Address (on the current device) of the library's device-side error flag,
// set to QAT_ERR_TIMEOUT by a kernel whose bounded wait gave up.
int* device_error_ptr();

void count_launch();  // bumps the process-wide launch counter

inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? QAT_OK : QAT_ERR_CUDA; }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sm_count();  // SMs of the current device (cached per device)

// One bit per device of a once-per-device flag (e.g. a kernel attribute, which
// belongs to each device's context).  device_flag_once returns whether the
// current device's bit is set and reports the device; device_flag_set sets it.
bool device_flag_once(std::atomic<uint64_t>& done, int* dev_out);
void device_flag_set(std::atomic<uint64_t>& done, int dev);

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void record_timeout(int* err) {
  if (err) atomicExch(err, QAT_ERR_TIMEOUT);
}

// IEEE fp32 helpers, written so the compiler can neither contract nor
// approximate them.
__device__ __forceinline__ float div_rn(float a, float b) { return __fdiv_rn(a, b); }
__device__ __forceinline__ float mul_rn(float a, float b) { return __fmul_rn(a, b); }

// fl32(w / s) given r = fl32(1 / s), by Markstein's correction step
// (P. Markstein, "Computation of elementary functions on the IBM RISC
// System/6000 processor", IBM J. Res. Develop. 34(1), 1990): q0 = fl(w * r) is
// within one ulp of w / s, the residual w - s * q0 is exact in one fused
// multiply-add, and q0 + residual * r rounded once is the correctly rounded
// quotient.  (Outside the normal range the result may differ from the true
// quotient only where |w / s| is far below 1/2, where every code is 0.)
__device__ __forceinline__ float div_by_scale(float w, float s, float r) {
  const float q0 = __fmul_rn(w, r);
  const float rem = __fmaf_rn(-q0, s, w);
  return __fmaf_rn(rem, r, q0);
}

// Levels of a grid's scale, s = amax / levels: 15 for int5, 127 for int6 and
// int8 (the int6 grid is every fourth int8 level).
__device__ __forceinline__ float grid_levels(int bits) { return bits == 5 ? 15.0f : 127.0f; }

// ---- paired fp32 arithmetic (two IEEE round-to-nearest operations per instruction)
__device__ __forceinline__ uint64_t f2u(float2 v) { return *reinterpret_cast<uint64_t*>(&v); }
__device__ __forceinline__ float2 u2f(uint64_t v) { return *reinterpret_cast<float2*>(&v); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2u(a)), "l"(f2u(b)));
  return u2f(d);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2u(a)), "l"(f2u(b)));
  return u2f(d);
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(f2u(a)), "l"(f2u(b)), "l"(f2u(c)));
  return u2f(d);
}

// 1.5 * 2^23: for |x| < 2^22, fl32(x + kOff) = kOff + rne(x) (the sum's ulp is 1,
// and ties go to even since kOff is even), whose bit pattern is 0x4B400000 + rne(x).
constexpr float kOff = 12582912.0f;

// Codes of two weights as exact float values, for a row scale s = fl32(amax / L)
// (L = 127, or 15 for int5) and r = fl32(1 / s): kOff + rne(fl32(w / s)) from
// the Markstein-corrected quotient (see div_by_scale), done pairwise; for int6
// kOff + rne(k / 4) (the fma forms k / 4 exactly) and 4 * (that - kOff) by one
// exact fma.  With that scale every |fl32(w / s)| < L + 1/2, so rne(w / s) is
// already in [-L, L] and only int6's second rounding can leave the grid
// (4 * rne(127 / 4) = 128 -> 124).
template <int BITS>
__device__ __forceinline__ float2 grid_code_values2(float a, float b, float s, float r) {
  const float2 w = make_float2(a, b), r2 = make_float2(r, r);
  const float2 q0 = mul2(w, r2);
  const float2 rem = fma2(q0, make_float2(-s, -s), w);
  const float2 t = add2(fma2(rem, r2, q0), make_float2(kOff, kOff));
  if constexpr (BITS == 6) {
    const float2 y = fma2(t, make_float2(0.25f, 0.25f), make_float2(-kOff / 4, -kOff / 4));
    const float2 u = add2(y, make_float2(kOff, kOff));
    const float2 c = fma2(u, make_float2(4.0f, 4.0f), make_float2(-4.0f * kOff, -4.0f * kOff));
    return make_float2(fminf(c.x, 124.0f), fminf(c.y, 124.0f));
  } else {
    return add2(t, make_float2(-kOff, -kOff));
  }
}

}  // namespace qat
