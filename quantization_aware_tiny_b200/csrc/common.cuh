// Shared device/host helpers of the sm_100a library (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

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

int sm_count();

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void record_timeout(int* err) {
  if (err) atomicExch(err, QAT_ERR_TIMEOUT);
}

// IEEE fp32 division and rounding helpers, written so the compiler can
// neither contract nor approximate them.
__device__ __forceinline__ float div_rn(float a, float b) { return __fdiv_rn(a, b); }
__device__ __forceinline__ float mul_rn(float a, float b) { return __fmul_rn(a, b); }
__device__ __forceinline__ float rne(float x) { return rintf(x); }  // round half to even

// Code of one weight on the int6 / int8 grid (see qat_quantize_weights).
__device__ __forceinline__ int quant_code(float w, float s, int bits) {
  float q = rne(div_rn(w, s));
  if (bits == 6) {
    q = mul_rn(rne(mul_rn(q, 0.25f)), 4.0f);  // q/4 and *4 are exact in fp32
    q = fminf(fmaxf(q, -128.0f), 124.0f);
  } else {
    q = fminf(fmaxf(q, -127.0f), 127.0f);
  }
  return __float2int_rn(q);
}

}  // namespace qat
