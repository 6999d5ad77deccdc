// HBM-bound quantizer kernels: training-time weight quantization (the GEMM
// operand / recurrence cache), the export quantizer with its per-row quantile
// clip, fp16 passthrough, and the roundtrip dequantizer.
//
// Quantization uses one warp per row.  The export kernel stages rows in shared
// memory with 1-D bulk async copies (the copy engine, completing on an
// mbarrier) one work unit ahead of the unit being quantized, with up to 16 warps per
// SM; the training-time kernel caches the row in registers between its
// reduction and quantization passes.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <type_traits>

#include "quant.cuh"
#include "sm100_ptx.cuh"

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

// Two floats as one word of bf16 (round to nearest even), the first in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// ------------------------------------------------------------------ Noisy QAT
// Philox-4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
// easy as 1, 2, 3", SC'11): ten rounds of the multiply-xor round function on a
// 4-word counter under a 2-word key bumped by the Weyl constants each round.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t hi0 = __umulhi(0xD2511F53u, c.x), lo0 = 0xD2511F53u * c.x;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c.z), lo1 = 0xCD9E8D57u * c.z;
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}

// fl32(w + fl32(fl32(u - 1/2) * s)) with u = (x >> 8) * 2^-24 in [0, 1).
__device__ __forceinline__ float noisy_value(float w, uint32_t x, float s) {
  const float u = __uint2float_rn(x >> 8) * 5.9604644775390625e-08f;  // exact
  return __fadd_rn(w, __fmul_rn(__fsub_rn(u, 0.5f), s));
}

// Noisy-QAT forward operand ("Depth Recurrence + Mixed-Precision Quant",
// "幸存发现 1 Noisy QAT"): per row s = max(amax, 1e-12) / 127 (the int8 step;
// amax / 15, the int5 step, for bits = 5), every weight gets (u - 1/2) * s of
// uniform noise, the result is cast to bf16.  Element e
// of the row-major weight takes word e % 4 of the Philox block with counter
// (e / 4, offset) and key seed.  One warp per row, the row cached in registers
// between the amax and the noise passes.
__global__ void __launch_bounds__(kQThreads)
    noisy_operand_kernel(const float* __restrict__ W, int N, int K, int bits, uint64_t seed,
                         uint64_t offset, float* __restrict__ scales,
                         __nv_bfloat16* __restrict__ operand) {
  const int lane = threadIdx.x & 31;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  const int K4 = K >> 2;
  const uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
  const uint32_t o0 = static_cast<uint32_t>(offset), o1 = static_cast<uint32_t>(offset >> 32);
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
    const float s = div_rn(fmaxf(amax, 1e-12f), grid_levels(bits));
    if (lane == 0 && scales) scales[row] = s;
    auto emit = [&](int j, float4 v) {
      const uint64_t g = static_cast<uint64_t>(row) * static_cast<uint64_t>(K4) + j;  // e / 4
      const uint4 x = philox4x32_10(
          make_uint4(static_cast<uint32_t>(g), static_cast<uint32_t>(g >> 32), o0, o1), k0, k1);
      __nv_bfloat162 lo = __floats2bfloat162_rn(noisy_value(v.x, x.x, s), noisy_value(v.y, x.y, s));
      __nv_bfloat162 hi = __floats2bfloat162_rn(noisy_value(v.z, x.z, s), noisy_value(v.w, x.w, s));
      uint2 o;
      o.x = *reinterpret_cast<uint32_t*>(&lo);
      o.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(operand + static_cast<int64_t>(row) * K + 4 * j) = o;
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
  const float lo = fminf(a, t1);
  t1 = fmaxf(a, t1);
  t2 = fmaxf(t2, lo);
}
__device__ __forceinline__ void top2_push4(float4 v, float& t1, float& t2) {
  top2_push(fabsf(v.x), t1, t2);
  top2_push(fabsf(v.y), t1, t2);
  top2_push(fabsf(v.z), t1, t2);
  top2_push(fabsf(v.w), t1, t2);
}
// Merge the 32 lanes' top-2 lists; every lane ends with the row's top two.
// The values are >= 0, so their bit patterns order like unsigned integers and
// one warp-wide integer max finds the largest, M.  The second largest (with
// multiplicity) is M when two lanes hold M, else the largest of every lane's
// list with one M removed.
__device__ __forceinline__ void top2_warp(float& t1, float& t2) {
  const uint32_t m = __reduce_max_sync(0xffffffffu, __float_as_uint(t1));
  const bool has = __float_as_uint(t1) == m;
  const uint32_t holders = __ballot_sync(0xffffffffu, has);
  const uint32_t cand = __float_as_uint(has ? t2 : t1);
  const uint32_t second = __reduce_max_sync(0xffffffffu, cand);
  t1 = __uint_as_float(m);
  t2 = __popc(holders) >= 2 ? t1 : __uint_as_float(second);
}

// fl32(1 / 127) and fl32(1 / 15), correctly rounded (0x3C010204, 0x3D888889).
constexpr float kRcp127 = 0.00787401571869850158691406f;
constexpr float kRcp15 = 0.066666670143604278564453125f;

struct RowQuant {
  float clip, s, rs;
  int bits;
};

// Clip and scales of one row from its top two |w| (see quantize_rows_export).
__device__ __forceinline__ RowQuant row_params(const ExportDescDev& d, float t1, float t2) {
  const float v_hi = t1;
  const float v_lo = (d.m == 2) ? t2 : t1;
  RowQuant q;
  q.clip = __fadd_rn(v_lo, __fmul_rn(d.frac, __fsub_rn(v_hi, v_lo)));
  q.s = d.mode == 5 ? div_by_scale(fmaxf(q.clip, 1e-12f), 15.0f, kRcp15)
                    : div_by_scale(fmaxf(q.clip, 1e-12f), 127.0f, kRcp127);
  q.rs = __frcp_rn(q.s);
  q.bits = d.mode;
  return q;
}

// Which clamps a row's codes need (chosen per row from its largest |w| a1 and
// its clip; see row_range):
//   kClampW    -- clamp w to [-clip, clip], then the grid's clamp;
//   kClampGrid -- the grid's clamp only.  Exact when a1 <= 2 clip: only entries
//                 with |w| > clip differ, their quotient |w / s| then lies in
//                 (L, 2L] (L = 127, or 15 for int5), and after the grid's clamp
//                 their code equals the code of +-clip itself (+124 / -128 for
//                 int6, +-127 for int8, +-15 for int5);
//   kNarrow    -- no clamp can bind except int6's top: when a1 <= fl32(1.0039 *
//                 clip), every |fl32(w / s)| < L + 1/2 (s = fl32(clip / L) is
//                 within 2^-24 of clip / L and the quotient adds one more
//                 rounding: |w / s| < 1.0039003 L, i.e. 127.4953 or 15.0585),
//                 so rne(w / s) is already in [-L, L]; int6's second rounding
//                 can still give 4 * 32 = 128 (-> 124), never below -128.
// The row clips of the pages' quantile sit within 0.3 % of the row maximum for
// rows of up to 1536 columns, so nearly every row is kNarrow.
constexpr int kClampW = 0, kClampGrid = 1, kNarrow = 2;
constexpr float kNarrowRatio = 1.0039f;

__device__ __forceinline__ int row_range(float a1, const RowQuant& q) {
  if (a1 > 2.0f * q.clip) return kClampW;
  return a1 <= __fmul_rn(kNarrowRatio, q.clip) ? kNarrow : kClampGrid;
}


// kOff + rne(fl32(w / s)) for two weights: the Markstein-corrected quotient
// (see div_by_scale) done pairwise, then the rounding offset kOff = 1.5 * 2^23
// (common.cuh); the float's bit pattern is 0x4B400000 + rne(w / s).
template <int R>
__device__ __forceinline__ float2 rne_quot2(const RowQuant& q, float a, float b) {
  const float2 w = R == kClampW ? make_float2(fminf(fmaxf(a, -q.clip), q.clip),
                                              fminf(fmaxf(b, -q.clip), q.clip))
                                : make_float2(a, b);
  const float2 s2 = make_float2(-q.s, -q.s), r2 = make_float2(q.rs, q.rs);
  const float2 q0 = mul2(w, r2);
  const float2 rem = fma2(q0, s2, w);
  const float2 x = fma2(rem, r2, q0);
  return add2(x, make_float2(kOff, kOff));
}

// int6: kOff + rne(k / 4) from t = kOff + k; the fma forms k / 4 exactly.
__device__ __forceinline__ float2 rne_quarter2(float2 t) {
  const float2 y = fma2(t, make_float2(0.25f, 0.25f), make_float2(-kOff / 4, -kOff / 4));
  return add2(y, make_float2(kOff, kOff));
}

// Integer codes of two weights on the row's grid, with the clamps the row's
// range needs: k = rne(fl32(w / s)); int6: 4 * rne(k / 4) clamped to
// [-128, 124], formed as 4 * (bits of kOff + rne(k / 4)) minus 4 * (bits of
// kOff) modulo 2^32; int8 / int5: k clamped to [-L, L].
template <int BITS, int R>
__device__ __forceinline__ void codes2(const RowQuant& q, float a, float b, int& ca, int& cb) {
  const float2 t = rne_quot2<R>(q, a, b);
  if constexpr (BITS == 6) {
    const float2 u = rne_quarter2(t);
    ca = static_cast<int>(__float_as_uint(u.x) * 4u - 0x2D000000u);
    cb = static_cast<int>(__float_as_uint(u.y) * 4u - 0x2D000000u);
    if constexpr (R == kNarrow) {
      ca = min(ca, 124);
      cb = min(cb, 124);
    } else {  // k = rne(x) >= -254 gives 4 rne(k / 4) >= -256: both clamps can bind
      ca = min(max(ca, -128), 124);
      cb = min(max(cb, -128), 124);
    }
  } else {
    constexpr int L = BITS == 5 ? 15 : 127;
    ca = __float_as_int(t.x) - 0x4B400000;
    cb = __float_as_int(t.y) - 0x4B400000;
    if constexpr (R != kNarrow) {
      ca = min(max(ca, -L), L);
      cb = min(max(cb, -L), L);
    }
  }
}

// Calls f(integral_constant<int, bits>, integral_constant<int, range>) for a
// row's grid and clamp range.
template <typename F>
__device__ __forceinline__ void with_grid(int bits, int range, F&& f) {
  using T5 = std::integral_constant<int, 5>;
  using T6 = std::integral_constant<int, 6>;
  using T8 = std::integral_constant<int, 8>;
  using R0 = std::integral_constant<int, kClampW>;
  using R1 = std::integral_constant<int, kClampGrid>;
  using R2 = std::integral_constant<int, kNarrow>;
  auto by_range = [&](auto bt) {
    if (range == kNarrow) f(bt, R2{});
    else if (range == kClampGrid) f(bt, R1{});
    else f(bt, R0{});
  };
  if (bits == 6) by_range(T6{});
  else if (bits == 5) by_range(T5{});
  else by_range(T8{});
}

// Four codes packed little-endian into a word (byte permutes).
__device__ __forceinline__ uint32_t pack4(int c0, int c1, int c2, int c3) {
  const uint32_t lo = __byte_perm(static_cast<uint32_t>(c0), static_cast<uint32_t>(c1), 0x0040);
  const uint32_t hi = __byte_perm(static_cast<uint32_t>(c2), static_cast<uint32_t>(c3), 0x0040);
  return __byte_perm(lo, hi, 0x5410);
}

// The codes c_i = MUL (x_i - B) of four words x_i (int6: x_i the bit pattern
// of kOff + rne(k / 4), B = 0x4B400000, MUL = 4), each in [-128, 127], as one
// word of their two's-complement bytes.  sum_i (c_i + 128) 2^(8i) has no
// carries between bytes, so four multiply-adds form it (modulo 2^32, B's
// share folded into the constant), and flipping each byte's top bit turns
// c + 128 into c's byte: no per-code byte permutes.
template <uint32_t MUL, uint32_t B>
__device__ __forceinline__ uint32_t pack_offset4(uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3) {
  constexpr uint32_t kC = (128u - MUL * B) * 0x01010101u;  // modulo 2^32
  uint32_t acc = x3 * (MUL << 24) + kC;
  acc = x2 * (MUL << 16) + acc;
  acc = x1 * (MUL << 8) + acc;
  acc = x0 * MUL + acc;
  return acc ^ 0x80808080u;
}

template <int BITS, int R>
__device__ __forceinline__ uint32_t codes4_t(const RowQuant& q, float4 v) {
  if constexpr (R == kNarrow && BITS != 6) {
    // no clamp binds: the code's byte is the low byte of kOff + rne(w / s)
    // (0x4B400000 has a zero low byte), so the offset need not be removed
    const float2 t0 = rne_quot2<R>(q, v.x, v.y), t1 = rne_quot2<R>(q, v.z, v.w);
    return pack4(__float_as_int(t0.x), __float_as_int(t0.y), __float_as_int(t1.x),
                 __float_as_int(t1.y));
  } else if constexpr (R == kNarrow) {
    // int6: only the top clamp can bind, 4 rne(k / 4) <= 124, i.e. the
    // pattern kOff + rne(k / 4) at most 0x4B40001F; then the bytes 4 rne(k / 4)
    const float2 u0 = rne_quarter2(rne_quot2<R>(q, v.x, v.y));
    const float2 u1 = rne_quarter2(rne_quot2<R>(q, v.z, v.w));
    return pack_offset4<4u, 0x4B400000u>(
        min(__float_as_uint(u0.x), 0x4B40001Fu), min(__float_as_uint(u0.y), 0x4B40001Fu),
        min(__float_as_uint(u1.x), 0x4B40001Fu), min(__float_as_uint(u1.y), 0x4B40001Fu));
  } else {
    int c0, c1, c2, c3;
    codes2<BITS, R>(q, v.x, v.y, c0, c1);
    codes2<BITS, R>(q, v.z, v.w, c2, c3);
    return pack4(c0, c1, c2, c3);
  }
}

// ------------------------------------------------------------------ QAT quantize
// Rows in segments of 512 columns (128 float4 groups, four per lane), a warp
// per segment: a row of K columns takes S = ceil(K / 512) segments, and a
// block of 8 warps takes 8 / min(S, 8) rows with min(S, 8) warps each, so
// every warp issues its four loads at once whatever the row length (a warp
// looping over a 2,048-column row waited on memory four times in a row).  The
// warps of a row merge their amax through shared memory; each keeps its first
// segment in registers for the code pass and reads any further segments (rows
// over 4,096 columns) a second time.
template <int BITS>
__device__ __forceinline__ void quantize_tile(const QuantDescDev& d, int64_t tile, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int K = d.K, K4 = K >> 2;
  const int S = (K4 + 127) >> 7;
  const int wpr = min(S, kQuantTileRows);  // warps per row
  const int rpb = kQuantTileRows / wpr;    // rows per block
  const int rib = warp / wpr, wir = warp - rib * wpr;
  const int64_t row = tile * rpb + rib;
  const bool active = rib < rpb && row < d.N;
  const float4* r = reinterpret_cast<const float4*>(d.W + (active ? row : 0) * static_cast<int64_t>(K));
  float4 v[4];
  float amax = 0.0f;
  if (active) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = wir * 128 + lane + 32 * u;
      v[u] = j < K4 ? __ldg(r + j) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
    amax = fmaxf(fmaxf(amax4(v[0]), amax4(v[1])), fmaxf(amax4(v[2]), amax4(v[3])));
    for (int sg = wir + wpr; sg < S; sg += wpr) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = sg * 128 + lane + 32 * u;
        if (j < K4) amax = fmaxf(amax, amax4(__ldg(r + j)));
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) red[warp] = amax;
  __syncthreads();
  if (!active) return;
  for (int w = rib * wpr; w < rib * wpr + wpr; ++w) amax = fmaxf(amax, red[w]);
  const float s = div_rn(fmaxf(amax, 1e-12f), grid_levels(BITS));
  const float rs = __frcp_rn(s);
  if (wir == 0 && lane == 0) d.scales[row] = s;
  const float2 s2 = make_float2(s, s);
  auto emit = [&](int j, float4 x) {
    const float2 c01 = grid_code_values2<BITS>(x.x, x.y, s, rs);
    const float2 c23 = grid_code_values2<BITS>(x.z, x.w, s, rs);
    const int64_t e = row * K + 4 * j;
    if (d.codes)
      *reinterpret_cast<uint32_t*>(d.codes + e) =
          pack_codes(__float2int_rn(c01.x), __float2int_rn(c01.y), __float2int_rn(c23.x),
                     __float2int_rn(c23.y));
    if (d.operand) {
      const float2 w01 = mul2(c01, s2), w23 = mul2(c23, s2);
      uint2 o;
      o.x = pack_bf16x2(w01.x, w01.y);
      o.y = pack_bf16x2(w23.x, w23.y);
      *reinterpret_cast<uint2*>(d.operand + e) = o;
    }
  };
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int j = wir * 128 + lane + 32 * u;
    if (j < K4) emit(j, v[u]);
  }
  for (int sg = wir + wpr; sg < S; sg += wpr) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = sg * 128 + lane + 32 * u;
      if (j < K4) emit(j, __ldg(r + j));
    }
  }
}

// The batch's weights in tiles (8 / min(S, 8) rows of one weight each), one
// thread block per tile: the tile's descriptor is block-uniform, found by a
// binary search on the tile index.
__global__ void __launch_bounds__(kQThreads, 6)
    quantize_batch_kernel(const __grid_constant__ QuantBatch b) {
  __shared__ float red[kQuantTileRows];
  const int64_t t = blockIdx.x;
  int lo = 0, hi = b.n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (b.tile_begin[mid] <= t) lo = mid; else hi = mid - 1;
  }
  const QuantDescDev& d = b.d[lo];
  const int64_t tile = t - b.tile_begin[lo];
  if (d.bits == 6) quantize_tile<6>(d, tile, red);
  else if (d.bits == 5) quantize_tile<5>(d, tile, red);
  else quantize_tile<8>(d, tile, red);
}

// ---- 6-bit packing of int6 / int5 codes: one 6-bit two's-complement field per
// code (c / 4 for int6, c for int5), field i at bits 6i .. 6i+5 of a
// little-endian bit stream; four codes make 24 bits, three bytes.

// The 24 packed bits of the four codes in the bytes of x (byte i = code i).
template <int BITS>
__device__ __forceinline__ uint32_t pack24(uint32_t x) {
  // per byte: the field in bits 0..5 (int6: the byte's bits 2..7, i.e. c / 4)
  const uint32_t y = (BITS == 6 ? (x >> 2) : x) & 0x3F3F3F3Fu;
  return (y & 0x3Fu) | ((y >> 2) & 0xFC0u) | ((y >> 4) & 0x3F000u) | ((y >> 6) & 0xFC0000u);
}

// Stores the 24-bit values p of the warp's first n lanes (n even, <= 32) as
// 3n contiguous bytes at dst (2-byte aligned).  Output word w (of 32 or 16
// bits) starts at stream bit 32w (16w), inside lane a = 4w / 3 (2w / 3)'s
// value at bit offset `off`; its remaining high bits come from lane a + 1.
// Full 32-lane chunks at 4-byte aligned addresses go out as 24 words, the
// rest as 16-bit halves.  Every lane must call this (shuffles).
__device__ __forceinline__ void store_pack6_chunk(uint8_t* dst, uint32_t p, int n, int lane) {
  if (n == 32 && (reinterpret_cast<uintptr_t>(dst) & 3u) == 0) {
    const int a = (4 * lane) / 3;
    const int off = 8 * (4 * lane - 3 * a);  // 0, 8 or 16
    const uint32_t lo = __shfl_sync(0xffffffffu, p, a & 31);
    const uint32_t hi = __shfl_sync(0xffffffffu, p, (a + 1) & 31);
    if (lane < 24) reinterpret_cast<uint32_t*>(dst)[lane] = (lo >> off) | (hi << (24 - off));
  } else {
    const int halves = 3 * n / 2;
    for (int h0 = 0; h0 < halves; h0 += 32) {
      const int h = h0 + lane;
      const int a = (2 * h) / 3;
      const int off = 8 * (2 * h - 3 * a);  // 0, 8 or 16
      const uint32_t lo = __shfl_sync(0xffffffffu, p, a & 31);
      const uint32_t hi = __shfl_sync(0xffffffffu, p, (a + 1) & 31);
      if (h < halves)
        reinterpret_cast<uint16_t*>(dst)[h] =
            static_cast<uint16_t>((lo >> off) | (hi << (24 - off)));
    }
  }
}

// float4 groups per lane and loop iteration in the shared-memory passes: more
// independent dependency chains per warp.
constexpr int kUnroll = 4;

template <int BITS, int R>
__device__ __forceinline__ void quantize_smem_row(const RowQuant& q, const float4* buf, int K4,
                                                  uint32_t* out, int lane) {
  int j = lane;
  for (; j + 32 * (kUnroll - 1) < K4; j += 32 * kUnroll) {
    float4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) v[u] = buf[j + 32 * u];
    uint32_t c[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) c[u] = codes4_t<BITS, R>(q, v[u]);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) out[j + 32 * u] = c[u];
  }
  for (; j < K4; j += 32) out[j] = codes4_t<BITS, R>(q, buf[j]);
}

// The same codes stored 6-bit packed: NR rows of K4 float4 groups (K4 even),
// row k read through src(k, j) and written to bytes [3 * K4) at out[k] (2-byte
// aligned).  The rows are interleaved, 4 / NR chunks of 32 groups each per
// iteration, so every lane has four independent groups in flight; chunks are
// warp-uniform, so the packing shuffles see every lane.
template <int BITS, int R, int NR, typename Src>
__device__ __forceinline__ void quantize_rows_pack6(const RowQuant (&q)[NR], Src src, int K4,
                                                    uint8_t* const (&out)[NR], int lane) {
  constexpr int U = 4 / NR;
  for (int base = 0; base < K4; base += 32 * U) {
    uint32_t p[NR][U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = base + 32 * u + lane;
#pragma unroll
      for (int k = 0; k < NR; ++k)
        p[k][u] = j < K4 ? pack24<BITS>(codes4_t<BITS, R>(q[k], src(k, j))) : 0u;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c0 = base + 32 * u;
      if (c0 < K4) {
#pragma unroll
        for (int k = 0; k < NR; ++k)
          store_pack6_chunk(out[k] + 3 * c0, p[k][u], min(32, K4 - c0), lane);
      }
    }
  }
}

// A quantized row staged in shared memory (cols <= the batch's buffer).
// PACK: the kernel also serves 6-bit packed descriptors.
template <bool PACK>
__device__ __forceinline__ void export_row_smem(const ExportDescDev& d, int64_t row,
                                                const float4* buf, int lane) {
  const int K4 = static_cast<int>(d.cols >> 2);
  float t1[kUnroll], t2[kUnroll];
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) t1[u] = t2[u] = 0.0f;
  int j = lane;
  for (; j + 32 * (kUnroll - 1) < K4; j += 32 * kUnroll) {
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) top2_push4(buf[j + 32 * u], t1[u], t2[u]);
  }
  for (; j < K4; j += 32) top2_push4(buf[j], t1[0], t2[0]);
  // merge this lane's partial lists
#pragma unroll
  for (int u = 1; u < kUnroll; ++u) {
    const float n2 = fmaxf(fminf(t1[0], t1[u]), fmaxf(t2[0], t2[u]));
    t1[0] = fmaxf(t1[0], t1[u]);
    t2[0] = n2;
  }
  float a1 = t1[0], a2 = t2[0];
  top2_warp(a1, a2);
  const RowQuant q = row_params(d, a1, a2);
  if (lane == 0) d.scales[row] = __float2half_rn(q.s);
  const int range = row_range(a1, q);
  if (PACK && d.pack6) {
    const RowQuant qs[1] = {q};
    uint8_t* const out[1] = {reinterpret_cast<uint8_t*>(d.dst) + row * 3 * K4};
    with_grid(q.bits, range, [&](auto bits_tag, auto range_tag) {
      constexpr int B = decltype(bits_tag)::value;
      if constexpr (B != 8)
        quantize_rows_pack6<B, decltype(range_tag)::value, 1>(
            qs, [&](int, int j) { return buf[j]; }, K4, out, lane);
    });
    return;
  }
  uint32_t* out = reinterpret_cast<uint32_t*>(reinterpret_cast<int8_t*>(d.dst) + row * d.cols);
  with_grid(q.bits, range, [&](auto bits_tag, auto range_tag) {
    quantize_smem_row<decltype(bits_tag)::value, decltype(range_tag)::value>(q, buf, K4, out, lane);
  });
}

// NR rows of the same tensor staged in shared memory (consecutive rows of one
// work unit), processed together so their top-2 passes, warp merges, scale
// computations and quantization passes interleave (NR independent dependency
// chains through every phase).  The rows share the strictest clamp range.
template <bool PACK, int NR>
__device__ __forceinline__ void export_rows_smem(const ExportDescDev& d, int64_t row,
                                                 const float4* buf, int lane) {
  const int K4 = static_cast<int>(d.cols >> 2);
  float t1[NR], t2[NR], u1[NR], u2[NR];
#pragma unroll
  for (int k = 0; k < NR; ++k) t1[k] = t2[k] = u1[k] = u2[k] = 0.0f;
  int j = lane;
  for (; j + 32 < K4; j += 64) {
#pragma unroll
    for (int k = 0; k < NR; ++k) {
      top2_push4(buf[k * K4 + j], t1[k], t2[k]);
      top2_push4(buf[k * K4 + j + 32], u1[k], u2[k]);
    }
  }
  if (j < K4) {
#pragma unroll
    for (int k = 0; k < NR; ++k) top2_push4(buf[k * K4 + j], t1[k], t2[k]);
  }
  RowQuant q[NR];
  int range = kNarrow;
#pragma unroll
  for (int k = 0; k < NR; ++k) {
    const float n2 = fmaxf(fminf(t1[k], u1[k]), fmaxf(t2[k], u2[k]));
    t1[k] = fmaxf(t1[k], u1[k]);
    t2[k] = n2;
    top2_warp(t1[k], t2[k]);
    q[k] = row_params(d, t1[k], t2[k]);
    range = min(range, row_range(t1[k], q[k]));
  }
  if (lane == 0) {
#pragma unroll
    for (int k = 0; k < NR; ++k) d.scales[row + k] = __float2half_rn(q[k].s);
  }
  if (PACK && d.pack6) {
    uint8_t* const out0 = reinterpret_cast<uint8_t*>(d.dst) + row * 3 * K4;
    uint8_t* out[NR];
#pragma unroll
    for (int k = 0; k < NR; ++k) out[k] = out0 + k * 3 * K4;
    with_grid(q[0].bits, range, [&](auto bits_tag, auto range_tag) {
      constexpr int B = decltype(bits_tag)::value;
      if constexpr (B != 8)
        quantize_rows_pack6<B, decltype(range_tag)::value, NR>(
            q, [&](int k, int jj) { return buf[k * K4 + jj]; }, K4, out, lane);
    });
    return;
  }
  uint32_t* out = reinterpret_cast<uint32_t*>(reinterpret_cast<int8_t*>(d.dst) + row * d.cols);
  auto run = [&](auto bits_tag, auto range_tag) {
    constexpr int BITS = decltype(bits_tag)::value;
    constexpr int R = decltype(range_tag)::value;
    int jj = lane;
    for (; jj + 32 < K4; jj += 64) {
      float4 v[NR][2];
#pragma unroll
      for (int k = 0; k < NR; ++k) {
        v[k][0] = buf[k * K4 + jj];
        v[k][1] = buf[k * K4 + jj + 32];
      }
      uint32_t c[NR][2];
#pragma unroll
      for (int k = 0; k < NR; ++k) {
        c[k][0] = codes4_t<BITS, R>(q[k], v[k][0]);
        c[k][1] = codes4_t<BITS, R>(q[k], v[k][1]);
      }
#pragma unroll
      for (int k = 0; k < NR; ++k) {
        out[k * K4 + jj] = c[k][0];
        out[k * K4 + jj + 32] = c[k][1];
      }
    }
    if (jj < K4) {
#pragma unroll
      for (int k = 0; k < NR; ++k) out[k * K4 + jj] = codes4_t<BITS, R>(q[k], buf[k * K4 + jj]);
    }
  };
  with_grid(q[0].bits, range, run);
}

// ---- full units of the common widths, specialised: 384 float4 groups, as
// three rows of 512 columns or one of 1,536 -- nearly every unit of the
// 11-layer d = 512 state dict.  Every offset is a compile-time constant,
// which takes the generic loops' counters and address arithmetic out of the
// per-element work, and each unit's per-row scalar work runs once, on lanes
// 0 to NR - 1, instead of on the whole warp per row.

// Three-input max (sm_100): max(a, b, c) in one instruction.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Running top-2 of |w| (with multiplicity) over four more weights, by sorted
// pairs: (h, l) = sorted |v.x|, |v.y| and |v.z|, |v.w|; the four's largest is
// max(h_xy, h_zw) and their second max(min(h_xy, h_zw), l_xy, l_zw); merging
// two sorted pairs (t1, t2), (X1, X2) gives max(t1, X1) and
// max(t2, X2, min(t1, X1)).  Ten min / max operations for four weights.
__device__ __forceinline__ void top2_push4_pairs(float4 v, float& t1, float& t2) {
  const float a = fabsf(v.x), b = fabsf(v.y), c = fabsf(v.z), e = fabsf(v.w);
  const float hab = fmaxf(a, b), lab = fminf(a, b);
  const float hce = fmaxf(c, e), lce = fminf(c, e);
  const float x1 = fmaxf(hab, hce);
  const float x2 = fmax3(fminf(hab, hce), lab, lce);
  const float y = fminf(t1, x1);
  t1 = fmaxf(t1, x1);
  t2 = fmax3(t2, y, x2);
}

// Merge of two top-2 lists (t1 >= t2, u1 >= u2) into (t1, t2).
__device__ __forceinline__ void top2_merge(float& t1, float& t2, float u1, float u2) {
  const float y = fminf(t1, u1);
  t1 = fmaxf(t1, u1);
  t2 = fmax3(t2, u2, y);
}

// A full unit of NR rows staged at buf (NR = 3: rows of 128 groups; NR = 1:
// one row of 384): lane holds groups lane + 32 i, i < 12; row k owns i in
// [12k / NR, 12(k + 1) / NR).
template <int NR>
__device__ __forceinline__ void export_unit384(const ExportDescDev& d, int64_t row0,
                                               const float4* __restrict__ buf, int lane) {
  // three chains of four groups: chain c = row c (NR = 3) or a third of the row
  float t1[3], t2[3];
#pragma unroll
  for (int c = 0; c < 3; ++c) t1[c] = t2[c] = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int c = 0; c < 3; ++c) top2_push4_pairs(buf[lane + 32 * (4 * c + i)], t1[c], t2[c]);
  }
  if constexpr (NR == 1) {
    top2_merge(t1[0], t2[0], t1[1], t2[1]);
    top2_merge(t1[0], t2[0], t1[2], t2[2]);
  }
#pragma unroll
  for (int k = 0; k < NR; ++k) top2_warp(t1[k], t2[k]);
  // lane k works out row k's clip, scales and clamp range once for the warp
  float m1 = t1[0], m2 = t2[0];
#pragma unroll
  for (int k = 1; k < NR; ++k) {
    if (lane == k) {
      m1 = t1[k];
      m2 = t2[k];
    }
  }
  const RowQuant mine = row_params(d, m1, m2);
  const int my_range = row_range(m1, mine);
  if (lane < NR) d.scales[row0 + lane] = __float2half_rn(mine.s);
  RowQuant q[NR];
  int range = kNarrow;
#pragma unroll
  for (int k = 0; k < NR; ++k) {
    q[k].clip = __shfl_sync(0xffffffffu, mine.clip, k);
    q[k].s = __shfl_sync(0xffffffffu, mine.s, k);
    q[k].rs = __shfl_sync(0xffffffffu, mine.rs, k);
    q[k].bits = mine.bits;
    range = min(range, __shfl_sync(0xffffffffu, my_range, k));
  }
  uint32_t* out = reinterpret_cast<uint32_t*>(reinterpret_cast<int8_t*>(d.dst) + row0 * d.cols) + lane;
  const float4* src = buf + lane;
  with_grid(q[0].bits, range, [&](auto bits_tag, auto range_tag) {
    constexpr int BITS = decltype(bits_tag)::value;
    constexpr int R = decltype(range_tag)::value;
#pragma unroll 1
    for (int c = 0; c < 3; ++c) {
      RowQuant qc = q[0];  // selects, not an indexed (local-memory) array
      if constexpr (NR == 3) {
        if (c == 1) qc = q[1];
        if (c == 2) qc = q[NR - 1];
      }
      const float4* sc = src + 128 * c;
      uint32_t* oc = out + 128 * c;
      float4 v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = sc[32 * i];
#pragma unroll
      for (int i = 0; i < 4; ++i) oc[32 * i] = codes4_t<BITS, R>(qc, v[i]);
    }
  });
}

// ---- clip search (the leaderboard's "GPTQ-lite" clip search, read as: per row,
// export at each candidate quantile and keep the first candidate of least
// squared error of the stored row, sum_j (w_j - c_j * fp16(s))^2).

// The candidate quantiles, in search order (the same values on the host).
__device__ __forceinline__ double clip_candidate(int k) {
  switch (k) {
    case 0: return 1.0;
    case 1: return 0.9999984;
    case 2: return 0.99999;
    case 3: return 0.9999;
    case 4: return 0.9995;
    default: return 0.999;
  }
}

// Running top-4 of |w| (with multiplicity), t[0] >= t[1] >= t[2] >= t[3].
__device__ __forceinline__ void top4_push(float a, float (&t)[kClipSearchTop]) {
#pragma unroll
  for (int i = 0; i < kClipSearchTop; ++i) {
    const float hi = fmaxf(a, t[i]);
    a = fminf(a, t[i]);
    t[i] = hi;
  }
}

// The row's top four from the lanes' sorted lists: four rounds, each taking
// the warp-wide largest head (values >= 0 order like their bit patterns) and
// popping it from one lane that holds it.
__device__ __forceinline__ void top4_warp(float (&t)[kClipSearchTop], float (&top)[kClipSearchTop],
                                          int lane) {
#pragma unroll
  for (int r = 0; r < kClipSearchTop; ++r) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, __float_as_uint(t[0]));
    const uint32_t holders = __ballot_sync(0xffffffffu, __float_as_uint(t[0]) == m);
    if (lane == __ffs(holders) - 1) {
#pragma unroll
      for (int i = 0; i + 1 < kClipSearchTop; ++i) t[i] = t[i + 1];
      t[kClipSearchTop - 1] = 0.0f;
    }
    top[r] = __uint_as_float(m);
  }
}

__device__ __forceinline__ float top_at(const float (&top)[kClipSearchTop], int64_t k) {
  return k == 0 ? top[0] : k == 1 ? top[1] : k == 2 ? top[2] : top[3];
}

// Grid parameters of candidate k for a row of n entries with top four `top`:
// the quantile as in quantize_rows_export (pos = q (n - 1) in double, linear
// interpolation in three fp32 roundings), then the row's scales.
__device__ __forceinline__ RowQuant candidate_params(const float (&top)[kClipSearchTop], int64_t n,
                                                     int k, int bits) {
  const double pos = clip_candidate(k) * static_cast<double>(n - 1);
  int64_t lo = static_cast<int64_t>(floor(pos));
  lo = lo < 0 ? 0 : (lo > n - 1 ? n - 1 : lo);
  const int64_t hi = lo + 1 < n ? lo + 1 : lo;
  const float frac = static_cast<float>(pos - static_cast<double>(lo));
  const float v_lo = top_at(top, n - 1 - lo), v_hi = top_at(top, n - 1 - hi);
  RowQuant q;
  q.clip = __fadd_rn(v_lo, __fmul_rn(frac, __fsub_rn(v_hi, v_lo)));
  q.s = bits == 5 ? div_by_scale(fmaxf(q.clip, 1e-12f), 15.0f, kRcp15)
                  : div_by_scale(fmaxf(q.clip, 1e-12f), 127.0f, kRcp127);
  q.rs = __frcp_rn(q.s);
  q.bits = bits;
  return q;
}

// Squared error of four weights against their codes times the stored scale sh.
template <int BITS>
__device__ __forceinline__ float sq_err4(const RowQuant& q, float sh, float4 v, float e) {
  int c0, c1, c2, c3;
  codes2<BITS, kClampW>(q, v.x, v.y, c0, c1);
  codes2<BITS, kClampW>(q, v.z, v.w, c2, c3);
  const float d0 = __fmaf_rn(-static_cast<float>(c0), sh, v.x);
  const float d1 = __fmaf_rn(-static_cast<float>(c1), sh, v.y);
  const float d2 = __fmaf_rn(-static_cast<float>(c2), sh, v.z);
  const float d3 = __fmaf_rn(-static_cast<float>(c3), sh, v.w);
  e = __fmaf_rn(d0, d0, e);
  e = __fmaf_rn(d1, d1, e);
  e = __fmaf_rn(d2, d2, e);
  return __fmaf_rn(d3, d3, e);
}

// One staged row under the clip search: top four of |w|, the candidates'
// errors in one pass (fp32, per-lane sums reduced by a butterfly so every
// lane holds the same totals and takes the same decision), then the row
// quantized with the kept candidate.
template <int BITS>
__device__ __forceinline__ void export_row_search_t(const ExportDescDev& d, int64_t row,
                                                    const float4* buf, int lane) {
  const int K4 = static_cast<int>(d.cols >> 2);
  float t[kClipSearchTop] = {0.0f, 0.0f, 0.0f, 0.0f};
  for (int j = lane; j < K4; j += 32) {
    const float4 v = buf[j];
    top4_push(fabsf(v.x), t);
    top4_push(fabsf(v.y), t);
    top4_push(fabsf(v.z), t);
    top4_push(fabsf(v.w), t);
  }
  float top[kClipSearchTop];
  top4_warp(t, top, lane);
  RowQuant q[kClipCandidates];
  float sh[kClipCandidates], e[kClipCandidates];
#pragma unroll
  for (int k = 0; k < kClipCandidates; ++k) {
    q[k] = candidate_params(top, d.cols, k, BITS);
    sh[k] = __half2float(__float2half_rn(q[k].s));
    e[k] = 0.0f;
  }
  for (int j = lane; j < K4; j += 32) {
    const float4 v = buf[j];
#pragma unroll
    for (int k = 0; k < kClipCandidates; ++k) e[k] = sq_err4<BITS>(q[k], sh[k], v, e[k]);
  }
  int best = 0;
  float best_e = 0.0f;
#pragma unroll
  for (int k = 0; k < kClipCandidates; ++k) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) e[k] += __shfl_xor_sync(0xffffffffu, e[k], o);
    if (k == 0 || e[k] < best_e) {
      best_e = e[k];
      best = k;
    }
  }
  const RowQuant qb = candidate_params(top, d.cols, best, BITS);
  if (lane == 0) d.scales[row] = __float2half_rn(qb.s);
  if (d.pack6) {
    if constexpr (BITS != 8) {
      const RowQuant qs[1] = {qb};
      uint8_t* const out[1] = {reinterpret_cast<uint8_t*>(d.dst) + row * 3 * K4};
      quantize_rows_pack6<BITS, kClampW, 1>(qs, [&](int, int j) { return buf[j]; }, K4, out, lane);
    }
    return;
  }
  uint32_t* out = reinterpret_cast<uint32_t*>(reinterpret_cast<int8_t*>(d.dst) + row * d.cols);
  quantize_smem_row<BITS, kClampW>(qb, buf, K4, out, lane);
}

__device__ __forceinline__ void export_row_search(const ExportDescDev& d, int64_t row,
                                                  const float4* buf, int lane) {
  if (d.mode == 6) export_row_search_t<6>(d, row, buf, lane);
  else if (d.mode == 5) export_row_search_t<5>(d, row, buf, lane);
  else export_row_search_t<8>(d, row, buf, lane);
}

// A quantized row read from global memory (rows longer than the staging buffer).
template <bool PACK>
__device__ __forceinline__ void export_row_global(const ExportDescDev& d, int64_t row, int lane) {
  const int K4 = static_cast<int>(d.cols >> 2);
  const float4* r = reinterpret_cast<const float4*>(d.src + row * d.cols);
  float t1 = 0.0f, t2 = 0.0f;
  for (int j = lane; j < K4; j += 32) top2_push4(__ldg(r + j), t1, t2);
  top2_warp(t1, t2);
  const RowQuant q = row_params(d, t1, t2);
  if (lane == 0) d.scales[row] = __float2half_rn(q.s);
  if (PACK && d.pack6) {
    const RowQuant qs[1] = {q};
    uint8_t* const out[1] = {reinterpret_cast<uint8_t*>(d.dst) + row * 3 * K4};
    with_grid(q.bits, kClampW, [&](auto bits_tag, auto range_tag) {
      constexpr int B = decltype(bits_tag)::value;
      if constexpr (B != 8)
        quantize_rows_pack6<B, decltype(range_tag)::value, 1>(
            qs, [&](int, int j) { return __ldg(r + j); }, K4, out, lane);
    });
    return;
  }
  uint32_t* out = reinterpret_cast<uint32_t*>(reinterpret_cast<int8_t*>(d.dst) + row * d.cols);
  with_grid(q.bits, row_range(t1, q), [&](auto bits_tag, auto range_tag) {
    constexpr int B = decltype(bits_tag)::value;
    constexpr int R = decltype(range_tag)::value;
    for (int j = lane; j < K4; j += 32) out[j] = codes4_t<B, R>(q, __ldg(r + j));
  });
}

// fp16 passthrough of one chunk ("row") of a flat tensor.
__device__ __forceinline__ void export_fp16_chunk(const ExportDescDev& d, int64_t row, int lane) {
  const int64_t begin = row * d.cols;
  const int64_t end = min(begin + d.cols, d.numel);
  const float* src = d.src + begin;
  __half* dst = reinterpret_cast<__half*>(d.dst) + begin;
  // chunk starts are multiples of cols (a multiple of 8): 8-element groups are
  // 16-byte aligned in the source and the destination
  const int n8 = static_cast<int>((end - begin) >> 3);
  constexpr int U = 4;
  for (int g0 = lane; g0 < n8; g0 += 32 * U) {
    float4 a[U], b[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int g = g0 + 32 * u;
      if (g < n8) {
        a[u] = __ldg(reinterpret_cast<const float4*>(src) + 2 * g);
        b[u] = __ldg(reinterpret_cast<const float4*>(src) + 2 * g + 1);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int g = g0 + 32 * u;
      if (g < n8) {
        __half2 h0 = __floats2half2_rn(a[u].x, a[u].y), h1 = __floats2half2_rn(a[u].z, a[u].w);
        __half2 h2 = __floats2half2_rn(b[u].x, b[u].y), h3 = __floats2half2_rn(b[u].z, b[u].w);
        uint4 w;
        w.x = *reinterpret_cast<uint32_t*>(&h0);
        w.y = *reinterpret_cast<uint32_t*>(&h1);
        w.z = *reinterpret_cast<uint32_t*>(&h2);
        w.w = *reinterpret_cast<uint32_t*>(&h3);
        *reinterpret_cast<uint4*>(dst + 8 * g) = w;
      }
    }
  }
  for (int64_t e = begin + 8 * static_cast<int64_t>(n8) + lane; e < end; e += 32)
    reinterpret_cast<__half*>(d.dst)[e] = __float2half_rn(d.src[e]);
}

// Descriptor owning work unit u (unit_begin is non-decreasing; the last
// descriptor with unit_begin <= u).
template <class Batch>
__device__ __forceinline__ int find_desc(const Batch& b, int64_t u) {
  int lo = 0, hi = b.n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (b.d[mid].unit_begin <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ bool staged(const ExportDescDev& d) {
  return d.mode != QAT_EXPORT_FP16 && d.cols <= kExportMaxStagedCols;
}
// (the host sizes buf_bytes for the longest staged row, so staged rows fit)

// A work unit: rows [row0, row0 + nrows) of descriptor d (d < 0: no more work).
struct UnitPos {
  int64_t row0;
  int nrows;
  int d;
};

// One launch over all descriptors.  Work units are runs of consecutive rows of
// one tensor -- as many as fit kExportUnitBytes for rows staged in shared
// memory, one row otherwise, one chunk of about the same bytes for fp16
// passthrough -- so units cost about the same.  Warp w of the grid takes the
// w-th run of ceil(units / W) consecutive units (W = warps in the grid; a
// static assignment: one shared work counter would serialise the warps on its
// atomics); a staged unit
// arrives in one bulk copy into one of the warp's kExportBufs buffers while
// the warp quantizes the previous one.  Units that are not staged still arrive once on their buffer's
// mbarrier so every buffer's phases stay in step with the unit count.
// KIND selects the code a batch needs, so a plain export carries neither the
// packing nor the search code (registers, instruction cache): kExportPlain,
// kExportPacked (some descriptors 6-bit packed), kExportSearch (some with the
// clip search; packing included).
constexpr int kExportPlain = 0, kExportPacked = 1, kExportSearch = 2;
template <int KIND, int CAP>
__global__ void __launch_bounds__(kExportMaxWarps * 32, 1)
    export_batch_kernel(const __grid_constant__ ExportBatchT<CAP> b, int* err) {
  extern __shared__ __align__(128) uint8_t xsmem[];
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  float4* bufs = reinterpret_cast<float4*>(xsmem + wib * kExportBufs * b.buf_bytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(xsmem + nw * kExportBufs * b.buf_bytes) +
                   wib * kExportBufs;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) abort_flag = 0;
  if (lane == 0) {
    for (int i = 0; i < kExportBufs; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  __syncthreads();

  // Warp gw takes the consecutive units [gw * per, (gw + 1) * per): units cost
  // about the same, and consecutive units mostly share their descriptor, so
  // a cursor replaces a search per unit.
  const int64_t W = static_cast<int64_t>(gridDim.x) * nw;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * nw + wib;
  const int64_t per = (b.total_units + W - 1) / W;
  const int64_t u_end = min(b.total_units, (gw + 1) * per);
  const int stride = b.buf_bytes / 16;
  int dcur = find_desc(b, min(gw * per, b.total_units - 1));
  auto next_unit = [&](int64_t u) {
    UnitPos p;
    if (u >= u_end) {
      p.d = -1;
      p.row0 = 0;
      p.nrows = 0;
      return p;
    }
    while (dcur + 1 < b.n && b.d[dcur + 1].unit_begin <= u) ++dcur;
    p.d = dcur;
    const ExportDescDev& d = b.d[dcur];
    p.row0 = (u - d.unit_begin) * d.unit_rows;
    p.nrows = static_cast<int>(min(d.unit_rows, d.rows - p.row0));
    return p;
  };

  auto issue = [&](const UnitPos& p, int slot) {
    if (p.d < 0 || lane != 0) return;
    const ExportDescDev& d = b.d[p.d];
    if (staged(d)) {
      const uint32_t bytes = static_cast<uint32_t>(p.nrows * d.cols * 4);
      mbar_arrive_expect_tx(&bars[slot], bytes);
      bulk_load_1d(bufs + slot * stride, d.src + p.row0 * d.cols, bytes, &bars[slot]);
    } else {
      mbar_arrive(&bars[slot]);
    }
  };

  // ring of kExportBufs units: pos[k] is the unit in buffer (i + k) % kExportBufs
  UnitPos pos[kExportBufs];
  int64_t next_u = gw * per;
  for (int k = 0; k < kExportBufs; ++k) {
    pos[k] = next_unit(next_u);
    ++next_u;
    issue(pos[k], k);
  }
  int i = 0;
  for (; pos[0].d >= 0; ++i) {
    const int slot = i % kExportBufs;
    if (!mbar_wait(&bars[slot], static_cast<uint32_t>((i / kExportBufs) & 1), &abort_flag, err))
      break;
    const ExportDescDev& d = b.d[pos[0].d];
    if (d.mode == QAT_EXPORT_FP16) {
      export_fp16_chunk(d, pos[0].row0, lane);
    } else if (staged(d)) {
      const int K4 = static_cast<int>(d.cols >> 2);
      const float4* ub = bufs + slot * stride;
      int r = 0;
      constexpr bool PACK = KIND != kExportPlain;
      if (KIND == kExportSearch && d.search) {
        for (; r < pos[0].nrows; ++r) export_row_search(d, pos[0].row0 + r, ub + r * K4, lane);
      } else if (KIND == kExportPlain && pos[0].nrows * K4 == 384 && (K4 == 128 || K4 == 384)) {
        if (K4 == 128) export_unit384<3>(d, pos[0].row0, ub, lane);
        else export_unit384<1>(d, pos[0].row0, ub, lane);
      } else {
        for (; r + 2 < pos[0].nrows; r += 3)
          export_rows_smem<PACK, 3>(d, pos[0].row0 + r, ub + r * K4, lane);
        if (r + 1 < pos[0].nrows) {
          export_rows_smem<PACK, 2>(d, pos[0].row0 + r, ub + r * K4, lane);
          r += 2;
        }
        if (r < pos[0].nrows) export_row_smem<PACK>(d, pos[0].row0 + r, ub + r * K4, lane);
      }
    } else {
      export_row_global<KIND != kExportPlain>(d, pos[0].row0, lane);
    }
    // the buffer is read; order those reads before the copy engine refills it
    fence_proxy_async_smem();
    __syncwarp();
    const UnitPos nn = next_unit(next_u);
    ++next_u;
    issue(nn, slot);
#pragma unroll
    for (int k = 0; k + 1 < kExportBufs; ++k) pos[k] = pos[k + 1];
    pos[kExportBufs - 1] = nn;
  }
  if (lane == 0) {
    // After a timeout: let the copies this warp still has in flight land
    // (bounded) before the block's shared memory is released.
    for (int k = 0; k < kExportBufs; ++k)
      if (pos[k].d >= 0)
        mbar_drain(&bars[(i + k) % kExportBufs], static_cast<uint32_t>(((i + k) / kExportBufs) & 1));
  }
}

// ------------------------------------------------------------------ dequantize
// Items of four consecutive codes of a row (item l of a tensor: elements
// 4l .. 4l + 3; cols a multiple of 8, so the four share the row's scale): the
// codes as one 32-bit load, fl32(c * fp32(scale_fp16)) stored as one 16-byte
// fp32 word (or 8 bytes of bf16), so a warp's loads and stores are
// contiguous.  A thread block takes one tile of kDequantTile items; each
// thread issues its kDequantPerThread items' loads before any store.  The row
// index comes from a multiply-high by row_magic instead of a 64-bit division,
// and every descriptor field a tile needs is block-uniform.
struct DequantItem {
  uint32_t c;  // four codes, little-endian bytes
  float s;     // the row's scale
};

__device__ __forceinline__ DequantItem dequant_load(const int8_t* __restrict__ codes,
                                                    const __half* __restrict__ scales,
                                                    uint64_t row_magic, int64_t l) {
  DequantItem it;
  it.c = __ldg(reinterpret_cast<const uint32_t*>(codes) + l);
  it.s = __half2float(__ldg(scales + __umul64hi(static_cast<uint64_t>(l), row_magic)));
  return it;
}

__device__ __forceinline__ void dequant_store(const DequantItem& it, int out_bf16,
                                              void* __restrict__ out, int64_t l) {
  const float v0 = mul_rn(static_cast<float>(static_cast<int8_t>(it.c & 0xFFu)), it.s);
  const float v1 = mul_rn(static_cast<float>(static_cast<int8_t>((it.c >> 8) & 0xFFu)), it.s);
  const float v2 = mul_rn(static_cast<float>(static_cast<int8_t>((it.c >> 16) & 0xFFu)), it.s);
  const float v3 = mul_rn(static_cast<float>(static_cast<int8_t>(it.c >> 24)), it.s);
  if (out_bf16) {
    uint2 w;
    w.x = pack_bf16x2(v0, v1);
    w.y = pack_bf16x2(v2, v3);
    reinterpret_cast<uint2*>(out)[l] = w;
  } else {
    reinterpret_cast<float4*>(out)[l] = make_float4(v0, v1, v2, v3);
  }
}

static_assert(kDequantTile == kQThreads * kDequantPerThread, "one tile per block of kQThreads");
static_assert(kQuantTileRows * 32 == kQThreads, "a warp per row of a quantize tile");

// Tile `tile` of one tensor's items.
__device__ __forceinline__ void dequant_tile(const int8_t* __restrict__ codes,
                                             const __half* __restrict__ scales, int64_t items,
                                             uint64_t row_magic, int out_bf16,
                                             void* __restrict__ out, int64_t tile) {
  const int64_t base = tile * kDequantTile + threadIdx.x;
  DequantItem it[kDequantPerThread];
#pragma unroll
  for (int j = 0; j < kDequantPerThread; ++j) {
    const int64_t l = base + j * kQThreads;
    if (l < items) it[j] = dequant_load(codes, scales, row_magic, l);
  }
#pragma unroll
  for (int j = 0; j < kDequantPerThread; ++j) {
    const int64_t l = base + j * kQThreads;
    if (l < items) dequant_store(it[j], out_bf16, out, l);
  }
}

__global__ void __launch_bounds__(kQThreads)
    dequant_kernel(const int8_t* __restrict__ codes, const __half* __restrict__ scales,
                   int64_t items, uint64_t row_magic, int out_bf16, void* __restrict__ out) {
  dequant_tile(codes, scales, items, row_magic, out_bf16, out, blockIdx.x);
}

// One block per tile of the concatenation; its descriptor is the last k with
// tile_begin[k] <= tile (tensors without items own no tile).
template <int CAP>
__global__ void __launch_bounds__(kQThreads)
    dequant_batch_kernel(const __grid_constant__ DequantBatchT<CAP> b) {
  const int64_t t = blockIdx.x;
  int lo = 0, hi = b.n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (b.tile_begin[mid] <= t) lo = mid; else hi = mid - 1;
  }
  const DequantDescDev& d = b.d[lo];
  dequant_tile(d.codes, d.scales, d.items, d.row_magic, d.out_bf16, d.out, t - b.tile_begin[lo]);
}

// 6-bit packed codes back to int8 codes: thread per 8 codes (6 bytes read as
// three 16-bit halves, 2-byte aligned; 8 codes written as one 8-byte word).
__global__ void __launch_bounds__(kQThreads)
    unpack6_kernel(const uint16_t* __restrict__ packed, int64_t n8, int bits,
                   uint2* __restrict__ codes) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint64_t v = static_cast<uint64_t>(packed[3 * i]) |
                       (static_cast<uint64_t>(packed[3 * i + 1]) << 16) |
                       (static_cast<uint64_t>(packed[3 * i + 2]) << 32);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int f = static_cast<int>((v >> (6 * k)) & 63u);
      const int c = (f >= 32 ? f - 64 : f) * (bits == 6 ? 4 : 1);
      w[k >> 2] |= (static_cast<uint32_t>(c) & 0xFFu) << (8 * (k & 3));
    }
    codes[i] = make_uint2(w[0], w[1]);
  }
}

int grid_for_rows(int64_t rows_or_items, int items_per_block) {
  const int64_t want = (rows_or_items + items_per_block - 1) / items_per_block;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  return static_cast<int>(std::max<int64_t>(1, std::min(want, cap)));
}

}  // namespace

int launch_quantize_batch(const QuantBatch& b, cudaStream_t s) {
  const int64_t tiles = b.tile_begin[b.n];
  if (tiles == 0) return QAT_OK;
  if (tiles > 0x7FFFFFFF) return QAT_ERR_SHAPE;
  quantize_batch_kernel<<<static_cast<unsigned>(tiles), kQThreads, 0, s>>>(b);
  count_launch();
  return cuda_status(cudaGetLastError());
}

int launch_quantize_weights(const float* W, int N, int K, int bits, int8_t* codes, float* scales,
                            __nv_bfloat16* operand, cudaStream_t s) {
  QuantBatch b;
  b.n = 1;
  b.tile_begin[0] = 0;
  b.tile_begin[1] = quant_tiles(N, K);
  b.d[0] = QuantDescDev{W, codes, scales, operand, N, K, bits, 0};
  return launch_quantize_batch(b, s);
}

int launch_noisy_operand(const float* W, int N, int K, int bits, uint64_t seed, uint64_t offset,
                         float* scales, __nv_bfloat16* operand, cudaStream_t s) {
  noisy_operand_kernel<<<grid_for_rows(N, kQThreads / 32), kQThreads, 0, s>>>(
      W, N, K, bits, seed, offset, scales, operand);
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

// Whether the clip search covers rows of `cols` entries: the row is staged in
// shared memory and every candidate's quantile needs only the top four order
// statistics (the same double arithmetic as the kernel's).
int clip_search_supported(int64_t cols) {
  if (cols < 2 || cols > kExportMaxStagedCols) return 0;
  static const double cand[kClipCandidates] = {1.0, 0.9999984, 0.99999, 0.9999, 0.9995, 0.999};
  for (int k = 0; k < kClipCandidates; ++k) {
    const int64_t lo = static_cast<int64_t>(std::floor(cand[k] * static_cast<double>(cols - 1)));
    if (cols - 1 - lo > kClipSearchTop - 1) return 0;
  }
  return 1;
}

// Descriptor capacities the batched kernels are built for, smallest first.
constexpr int kBatchCapSmall = 24, kBatchCapMid = 96;

// The export kernel of kind KIND at capacity CAP, its shared-memory limit
// raised once per device.
template <int KIND, int CAP>
int export_launch_kind(const ExportBatchT<CAP>& t, int grid, int warps, int smem, cudaStream_t s) {
  static std::atomic<uint64_t> attr_done{0};  // per device: attributes live in its context
  int dev = 0;
  if (!device_flag_once(attr_done, &dev)) {
    if (cudaFuncSetAttribute(export_batch_kernel<KIND, CAP>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kExportSmemBudget) != cudaSuccess)
      return QAT_ERR_CUDA;
    device_flag_set(attr_done, dev);
  }
  export_batch_kernel<KIND, CAP><<<grid, warps * 32, smem, s>>>(t, device_error_ptr());
  return QAT_OK;
}

// The batch copied into a parameter block of capacity CAP (n <= CAP).
template <int CAP>
int export_launch_cap(const ExportBatch& b, int kind, int grid, int warps, int smem,
                      cudaStream_t s) {
  static thread_local ExportBatchT<CAP> t;
  t.n = b.n;
  t.buf_bytes = b.buf_bytes;
  t.total_units = b.total_units;
  std::copy(b.d, b.d + b.n, t.d);
  if (kind == kExportSearch) return export_launch_kind<kExportSearch, CAP>(t, grid, warps, smem, s);
  if (kind == kExportPacked) return export_launch_kind<kExportPacked, CAP>(t, grid, warps, smem, s);
  return export_launch_kind<kExportPlain, CAP>(t, grid, warps, smem, s);
}

int launch_export_batch(ExportBatch& b, cudaStream_t s) {
  if (b.total_units == 0) return QAT_OK;
  int64_t longest = 16;  // bytes of the longest staged unit
  for (int i = 0; i < b.n; ++i)
    if (b.d[i].mode != QAT_EXPORT_FP16 && b.d[i].cols <= kExportMaxStagedCols)
      longest = std::max(longest, b.d[i].unit_rows * b.d[i].cols * 4);
  b.buf_bytes = static_cast<int>((longest + 127) / 128 * 128);
  const int per_warp = kExportBufs * (b.buf_bytes + 8);
  const int warps = std::max(1, std::min(kExportMaxWarps, kExportSmemBudget / per_warp));
  const int smem = warps * per_warp;
  const int64_t want = (b.total_units + warps - 1) / warps;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, sm_count())));
  bool search = false, packed = false;
  for (int i = 0; i < b.n; ++i) {
    search = search || b.d[i].search;
    packed = packed || b.d[i].pack6;
  }
  const int kind = search ? kExportSearch : packed ? kExportPacked : kExportPlain;
  int rc;
  if (b.n <= kBatchCapSmall) rc = export_launch_cap<kBatchCapSmall>(b, kind, grid, warps, smem, s);
  else if (b.n <= kBatchCapMid) rc = export_launch_cap<kBatchCapMid>(b, kind, grid, warps, smem, s);
  else rc = export_launch_cap<QAT_EXPORT_BATCH_CAP>(b, kind, grid, warps, smem, s);
  if (rc != QAT_OK) return rc;
  count_launch();
  return cuda_status(cudaGetLastError());
}

int launch_dequant(const int8_t* codes, const __half* scales, int64_t rows, int64_t cols,
                   int out_bf16, void* out, cudaStream_t s) {
  const int64_t items = rows * (cols >> 2);
  if (items == 0) return QAT_OK;
  const int64_t tiles = (items + kDequantTile - 1) / kDequantTile;
  if (tiles > 0x7FFFFFFF) return QAT_ERR_SHAPE;
  dequant_kernel<<<static_cast<unsigned>(tiles), kQThreads, 0, s>>>(
      codes, scales, items, dequant_row_magic(cols >> 2), out_bf16, out);
  count_launch();
  return cuda_status(cudaGetLastError());
}

// The batch copied into a parameter block of capacity CAP (n <= CAP).
template <int CAP>
void dequant_launch_cap(const DequantBatch& b, unsigned grid, cudaStream_t s) {
  static thread_local DequantBatchT<CAP> t;
  t.n = b.n;
  std::copy(b.tile_begin, b.tile_begin + b.n + 1, t.tile_begin);
  std::copy(b.d, b.d + b.n, t.d);
  dequant_batch_kernel<CAP><<<grid, kQThreads, 0, s>>>(t);
}

int launch_dequant_batch(const DequantBatch& b, cudaStream_t s) {
  const int64_t tiles = b.tile_begin[b.n];
  if (tiles == 0) return QAT_OK;
  if (tiles > 0x7FFFFFFF) return QAT_ERR_SHAPE;
  const unsigned grid = static_cast<unsigned>(tiles);
  if (b.n <= kBatchCapSmall) dequant_launch_cap<kBatchCapSmall>(b, grid, s);
  else if (b.n <= kBatchCapMid) dequant_launch_cap<kBatchCapMid>(b, grid, s);
  else dequant_launch_cap<kDequantMaxDescs>(b, grid, s);
  count_launch();
  return cuda_status(cudaGetLastError());
}

int launch_unpack6(const uint8_t* packed, int64_t n, int bits, int8_t* codes, cudaStream_t s) {
  const int64_t n8 = n / 8;
  if (n8 == 0) return QAT_OK;
  unpack6_kernel<<<grid_for_rows(n8, kQThreads), kQThreads, 0, s>>>(
      reinterpret_cast<const uint16_t*>(packed), n8, bits, reinterpret_cast<uint2*>(codes));
  count_launch();
  return cuda_status(cudaGetLastError());
}

}  // namespace qat
