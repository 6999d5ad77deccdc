// HBM-bound quantizer kernels: training-time weight quantization (the GEMM
// operand / recurrence cache), the export quantizer with its per-row quantile
// clip, fp16 passthrough, and the roundtrip dequantizer.
//
// One warp per row: coalesced 16-byte loads (512 B per warp instruction), warp
// shuffle reductions, rows cached in registers between the reduction pass and
// the quantization pass (up to 2048 columns; longer rows re-read from L2).
#include <algorithm>
#include <cmath>

#include "quant.cuh"

namespace qat {

namespace {

constexpr int kQThreads = 256;  // 8 warps per block
constexpr int kRegV4 = 16;      // float4 per lane kept in registers (2048 columns)

__device__ __forceinline__ float amax4(float4 v) {
  return fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
}

__device__ __forceinline__ uint32_t pack_codes(int a, int b, int c, int d) {
  return (static_cast<uint32_t>(a) & 0xffu) | ((static_cast<uint32_t>(b) & 0xffu) << 8) |
         ((static_cast<uint32_t>(c) & 0xffu) << 16) | ((static_cast<uint32_t>(d) & 0xffu) << 24);
}

__device__ __forceinline__ uint2 operand4(int c0, int c1, int c2, int c3, float s) {
  // bf16_rne(fl32(c * s)) for four codes
  __nv_bfloat162 lo = __floats2bfloat162_rn(mul_rn(static_cast<float>(c0), s),
                                            mul_rn(static_cast<float>(c1), s));
  __nv_bfloat162 hi = __floats2bfloat162_rn(mul_rn(static_cast<float>(c2), s),
                                            mul_rn(static_cast<float>(c3), s));
  uint2 r;
  r.x = *reinterpret_cast<uint32_t*>(&lo);
  r.y = *reinterpret_cast<uint32_t*>(&hi);
  return r;
}

// ------------------------------------------------------------------ QAT quantize
__global__ void __launch_bounds__(kQThreads)
    quantize_weights_kernel(const float* __restrict__ W, int N, int K, int bits,
                            int8_t* __restrict__ codes, float* __restrict__ scales,
                            __nv_bfloat16* __restrict__ operand) {
  const int lane = threadIdx.x & 31;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  const int K4 = K >> 2;
  for (int row = warp; row < N; row += nwarps) {
    const float4* r = reinterpret_cast<const float4*>(W + static_cast<int64_t>(row) * K);
    float4 cache[kRegV4];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < kRegV4; ++i) {
      const int j = lane + 32 * i;
      if (j < K4) {
        cache[i] = __ldg(r + j);
        amax = fmaxf(amax, amax4(cache[i]));
      }
    }
    for (int j = lane + 32 * kRegV4; j < K4; j += 32) amax = fmaxf(amax, amax4(__ldg(r + j)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    amax = fmaxf(amax, 1e-12f);
    const float s = div_rn(amax, 127.0f);
    if (lane == 0) scales[row] = s;
    auto emit = [&](int j, float4 v) {
      const int c0 = quant_code(v.x, s, bits), c1 = quant_code(v.y, s, bits);
      const int c2 = quant_code(v.z, s, bits), c3 = quant_code(v.w, s, bits);
      const int64_t e = static_cast<int64_t>(row) * K + 4 * j;
      if (codes) *reinterpret_cast<uint32_t*>(codes + e) = pack_codes(c0, c1, c2, c3);
      if (operand) *reinterpret_cast<uint2*>(operand + e) = operand4(c0, c1, c2, c3, s);
    };
#pragma unroll
    for (int i = 0; i < kRegV4; ++i) {
      const int j = lane + 32 * i;
      if (j < K4) emit(j, cache[i]);
    }
    for (int j = lane + 32 * kRegV4; j < K4; j += 32) emit(j, __ldg(r + j));
  }
}

// ------------------------------------------------------------------ export
// Running top-2 of |w| (with multiplicity): t1 >= t2.
__device__ __forceinline__ void top2_push(float a, float& t1, float& t2) {
  if (a > t1) {
    t2 = t1;
    t1 = a;
  } else if (a > t2) {
    t2 = a;
  }
}
__device__ __forceinline__ void top2_push4(float4 v, float& t1, float& t2) {
  top2_push(fabsf(v.x), t1, t2);
  top2_push(fabsf(v.y), t1, t2);
  top2_push(fabsf(v.z), t1, t2);
  top2_push(fabsf(v.w), t1, t2);
}

__device__ __forceinline__ void export_quant_row(const ExportDescDev& d, int64_t row, int lane) {
  const int64_t cols = d.cols;
  const int K4 = static_cast<int>(cols >> 2);
  const float4* r = reinterpret_cast<const float4*>(d.src + row * cols);
  float4 cache[kRegV4];
  float t1 = 0.0f, t2 = 0.0f;
#pragma unroll
  for (int i = 0; i < kRegV4; ++i) {
    const int j = lane + 32 * i;
    if (j < K4) {
      cache[i] = __ldg(r + j);
      top2_push4(cache[i], t1, t2);
    }
  }
  for (int j = lane + 32 * kRegV4; j < K4; j += 32) top2_push4(__ldg(r + j), t1, t2);
  // merge the lanes' top-2 lists
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float b1 = __shfl_xor_sync(0xffffffffu, t1, o);
    const float b2 = __shfl_xor_sync(0xffffffffu, t2, o);
    const float n1 = fmaxf(t1, b1);
    const float n2 = fmaxf(fminf(t1, b1), fmaxf(t2, b2));
    t1 = n1;
    t2 = n2;
  }
  // v_hi = largest, v_lo = the (cols - lo)-th largest (top2 = 2, top1 = 1)
  const float v_hi = t1;
  const float v_lo = (d.m == 2) ? t2 : t1;
  const float clip = __fadd_rn(v_lo, __fmul_rn(d.frac, __fsub_rn(v_hi, v_lo)));
  const float s = div_rn(fmaxf(clip, 1e-12f), 127.0f);
  if (lane == 0) d.scales[row] = __float2half_rn(s);
  int8_t* out = reinterpret_cast<int8_t*>(d.dst) + row * cols;
  const int bits = d.mode;
  auto emit = [&](int j, float4 v) {
    const int c0 = quant_code(fminf(fmaxf(v.x, -clip), clip), s, bits);
    const int c1 = quant_code(fminf(fmaxf(v.y, -clip), clip), s, bits);
    const int c2 = quant_code(fminf(fmaxf(v.z, -clip), clip), s, bits);
    const int c3 = quant_code(fminf(fmaxf(v.w, -clip), clip), s, bits);
    *reinterpret_cast<uint32_t*>(out + 4 * j) = pack_codes(c0, c1, c2, c3);
  };
#pragma unroll
  for (int i = 0; i < kRegV4; ++i) {
    const int j = lane + 32 * i;
    if (j < K4) emit(j, cache[i]);
  }
  for (int j = lane + 32 * kRegV4; j < K4; j += 32) emit(j, __ldg(r + j));
}

// fp16 passthrough of one chunk ("row") of a flat tensor.
__device__ __forceinline__ void export_fp16_chunk(const ExportDescDev& d, int64_t row, int lane) {
  const int64_t begin = row * d.cols;
  const int64_t end = min(begin + d.cols, d.numel);
  const float* src = d.src;
  __half* dst = reinterpret_cast<__half*>(d.dst);
  // chunk starts are multiples of cols (a multiple of 8), so 8-element groups
  // are 16-byte aligned in the source and the destination
  const int64_t n8 = (end - begin) >> 3;
  for (int64_t g = lane; g < n8; g += 32) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(src + begin) + 2 * g);
    const float4 b = __ldg(reinterpret_cast<const float4*>(src + begin) + 2 * g + 1);
    __half2 h0 = __floats2half2_rn(a.x, a.y), h1 = __floats2half2_rn(a.z, a.w);
    __half2 h2 = __floats2half2_rn(b.x, b.y), h3 = __floats2half2_rn(b.z, b.w);
    uint4 w;
    w.x = *reinterpret_cast<uint32_t*>(&h0);
    w.y = *reinterpret_cast<uint32_t*>(&h1);
    w.z = *reinterpret_cast<uint32_t*>(&h2);
    w.w = *reinterpret_cast<uint32_t*>(&h3);
    *reinterpret_cast<uint4*>(dst + begin + 8 * g) = w;
  }
  for (int64_t e = begin + 8 * n8 + lane; e < end; e += 32) dst[e] = __float2half_rn(src[e]);
}

__global__ void __launch_bounds__(kQThreads) export_batch_kernel(const ExportBatch b) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t g = warp; g < b.total_rows; g += nwarps) {
    // descriptor owning global row g (row_begin is increasing)
    int lo = 0, hi = b.n - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (b.d[mid].row_begin <= g) lo = mid; else hi = mid - 1;
    }
    const ExportDescDev& d = b.d[lo];
    const int64_t row = g - d.row_begin;
    if (d.mode == QAT_EXPORT_FP16) export_fp16_chunk(d, row, lane);
    else export_quant_row(d, row, lane);
  }
}

// ------------------------------------------------------------------ dequantize
__global__ void __launch_bounds__(kQThreads)
    dequant_kernel(const int8_t* __restrict__ codes, const __half* __restrict__ scales,
                   int64_t rows, int64_t cols, int out_bf16, void* __restrict__ out) {
  const int64_t n8_row = cols >> 3;
  const int64_t total = rows * n8_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = i / n8_row;
    const int64_t e = i * 8;
    const float s = __half2float(scales[row]);
    const uint2 cc = *reinterpret_cast<const uint2*>(codes + e);
    const int8_t* c = reinterpret_cast<const int8_t*>(&cc);
    float v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = mul_rn(static_cast<float>(c[k]), s);
    if (out_bf16) {
      __nv_bfloat162 p0 = __floats2bfloat162_rn(v[0], v[1]), p1 = __floats2bfloat162_rn(v[2], v[3]);
      __nv_bfloat162 p2 = __floats2bfloat162_rn(v[4], v[5]), p3 = __floats2bfloat162_rn(v[6], v[7]);
      uint4 w;
      w.x = *reinterpret_cast<uint32_t*>(&p0);
      w.y = *reinterpret_cast<uint32_t*>(&p1);
      w.z = *reinterpret_cast<uint32_t*>(&p2);
      w.w = *reinterpret_cast<uint32_t*>(&p3);
      *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(out) + e) = w;
    } else {
      float4* o = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + e);
      o[0] = make_float4(v[0], v[1], v[2], v[3]);
      o[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
  }
}

int grid_for_rows(int64_t rows_or_items, int items_per_block) {
  const int64_t want = (rows_or_items + items_per_block - 1) / items_per_block;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  return static_cast<int>(std::max<int64_t>(1, std::min(want, cap)));
}

}  // namespace

int launch_quantize_weights(const float* W, int N, int K, int bits, int8_t* codes, float* scales,
                            __nv_bfloat16* operand, cudaStream_t s) {
  quantize_weights_kernel<<<grid_for_rows(N, kQThreads / 32), kQThreads, 0, s>>>(
      W, N, K, bits, codes, scales, operand);
  count_launch();
  return cuda_status(cudaGetLastError());
}

// Order statistic (m = cols - lo, 1 or 2) and interpolation fraction of the
// export quantile for rows of `cols` entries, from the position q*(cols-1)
// computed in double.
int export_quantile_params(int64_t cols, int* m, float* frac) {
  const double pos = 0.9999984 * static_cast<double>(cols - 1);
  int64_t lo = static_cast<int64_t>(std::floor(pos));
  lo = std::max<int64_t>(0, std::min<int64_t>(lo, cols - 1));
  const int64_t mm = cols - lo;
  if (mm > 2) return QAT_ERR_SHAPE;
  *m = static_cast<int>(mm);
  *frac = static_cast<float>(pos - static_cast<double>(lo));
  return QAT_OK;
}

int launch_export_batch(const ExportBatch& b, cudaStream_t s) {
  if (b.total_rows == 0) return QAT_OK;
  export_batch_kernel<<<grid_for_rows(b.total_rows, kQThreads / 32), kQThreads, 0, s>>>(b);
  count_launch();
  return cuda_status(cudaGetLastError());
}

int launch_dequant(const int8_t* codes, const __half* scales, int64_t rows, int64_t cols,
                   int out_bf16, void* out, cudaStream_t s) {
  const int64_t items = rows * (cols >> 3);
  if (items == 0) return QAT_OK;
  dequant_kernel<<<grid_for_rows(items, kQThreads), kQThreads, 0, s>>>(codes, scales, rows, cols,
                                                                       out_bf16, out);
  count_launch();
  return cuda_status(cudaGetLastError());
}

}  // namespace qat
