/*
 * CPU oracle for the int6 quantization-aware linear and its export quantizer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the tests, the package's smoke check and the CPU
 * baseline leg of the benchmark do.  It shares no code, header, table or
 * constant with the CUDA path.
 *
 * Plain scalar C99.  Every floating-point step is one IEEE binary32 operation
 * (build with -O2 -ffp-contract=off, never -ffast-math), rounding is the
 * default round-to-nearest-even mode, so each result below is the correctly
 * rounded value fl32(.) of the operation it names.
 *
 * Sources (page title, section):
 *  - "parameter-golf 16MB 极限压缩实战：11L MLP3x + Int6 QAT + zstd-22 记录详解",
 *    section "训练时的模拟量化": per-row amax, scale = amax/127,
 *    q_raw = round(w/scale), int6: q = round(q_raw/4)*4 clamped to [-128,124];
 *    STE forward uses the quantized weight.
 *  - same page, section "后训练量化导出": per-row clip at the 99.99984
 *    percentile, one fp16 scale per row, int8 or int6 codes, small tensors
 *    and the tied embedding pass through as fp16, with the same rounding
 *    logic as training.
 *  - "Depth Recurrence + Mixed-Precision Quant" write-up (PR #363), section
 *    "幸存发现 1 Noisy QAT" code: amax is clamp_min(1e-12) before /127.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - .round() is round-half-to-even (torch semantics) for both roundings;
 *  - w/scale and amax/127 are true IEEE divisions;
 *  - int8 codes clamp to [-127,127];
 *  - the quantile is linear interpolation on the sorted |w| at position
 *    q*(n-1) (computed in double), interpolated with three fp32 operations;
 *  - export codes use the fp32 scale, the stored scale is fp16(rne) of it.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_AMAX_FLOOR 1e-12f

/* ---- bit-level conversions (from the IEEE 754 definitions) -------------- */

static uint32_t f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float u2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* Round a binary32 value to bfloat16 (8-bit significand), nearest-even.
 * bfloat16 is the upper half of binary32, so rounding is done on the
 * discarded low 16 bits: above half -> up, below -> down, exactly half ->
 * to the even upper half.  NaN stays a quiet NaN. */
uint16_t oracle_bf16_rne(float x) {
  uint32_t u = f2u(x);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) {
    return (uint16_t)((u >> 16) | 0x0040u);
  }
  uint32_t upper = u >> 16;
  uint32_t lower = u & 0xffffu;
  if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;
  return (uint16_t)upper;
}

float oracle_bf16_to_f32(uint16_t b) { return u2f(((uint32_t)b) << 16); }

/* Round a binary32 value to binary16, nearest-even, with gradual underflow
 * and overflow to infinity.  Works on the exact value m * 2^e. */
uint16_t oracle_fp16_rne(float x) {
  uint32_t u = f2u(x);
  uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
  uint32_t ex = (u >> 23) & 0xffu;
  uint32_t man = u & 0x7fffffu;
  if (ex == 0xffu) return (uint16_t)(sign | 0x7c00u | (man ? 0x200u : 0u));
  if (ex == 0 && man == 0) return sign;
  /* value = sig * 2^(E) with sig an integer of 24 bits (normal) */
  int32_t E;
  uint64_t sig;
  if (ex == 0) { sig = man; E = -149; } else { sig = man | 0x800000u; E = (int32_t)ex - 150; }
  /* target: half value = hs * 2^(he - 24) with quantum depending on range.
   * The half quantum is 2^(e16 - 10) for normal exponents e16 >= -14,
   * and 2^-24 for subnormals. */
  /* exponent of the leading bit of the value */
  int32_t lead = E;
  { uint64_t t = sig; while (t > 1) { t >>= 1; lead++; } }
  int32_t q = (lead < -14) ? -24 : lead - 10; /* log2 of the half ulp grid */
  /* integer n = value / 2^q, rounded to nearest even */
  uint64_t n;
  int32_t sh = q - E;
  if (sh <= 0) {
    n = sig << (uint32_t)(-sh);
  } else if (sh >= 63) {
    n = 0; /* far below half the smallest subnormal */
    if (sh == 63) { /* cannot happen for binary32 inputs */ }
  } else {
    uint64_t keep = sig >> (uint32_t)sh;
    uint64_t rem = sig & ((1ull << (uint32_t)sh) - 1ull);
    uint64_t half = 1ull << (uint32_t)(sh - 1);
    if (rem > half || (rem == half && (keep & 1ull))) keep += 1ull;
    n = keep;
  }
  /* n * 2^q ; encode */
  if (q == -24) {
    /* subnormal grid; n may have rounded up to the smallest normal 1024 */
    return (uint16_t)(sign | (uint16_t)n); /* n <= 1024 -> 0x0400 is min normal */
  }
  /* normal: n in [1024, 2048]; rounding may carry into the next binade */
  int32_t e16 = q + 10;
  if (n == 2048u) { n = 1024u; e16 += 1; }
  if (e16 > 15) return (uint16_t)(sign | 0x7c00u);
  return (uint16_t)(sign | (uint16_t)((uint32_t)(e16 + 15) << 10) | (uint16_t)(n - 1024u));
}

float oracle_fp16_to_f32(uint16_t h) {
  uint32_t sign = ((uint32_t)h & 0x8000u) << 16;
  uint32_t ex = (h >> 10) & 0x1fu;
  uint32_t man = h & 0x3ffu;
  if (ex == 0x1fu) return u2f(sign | 0x7f800000u | (man << 13));
  if (ex == 0) {
    /* subnormal: man * 2^-24, exactly representable in binary32 */
    float v = (float)man * 5.9604644775390625e-08f;
    return sign ? -v : v;
  }
  return u2f(sign | ((ex + 112u) << 23) | (man << 13));
}

/* ---- QAT fake quantization (training-time simulated quantization) -------- */

/* Levels of a grid: the scale is amax / levels.  int6 and int8 use 127 (the
 * int6 grid is every fourth int8 level); int5 uses 15 (reading of the page-1
 * remark that an int5-calibrated step would be amax / 15: codes in [-15, 15]). */
static float oracle_levels(int bits) { return bits == 5 ? 15.0f : 127.0f; }

/* Per-row amax clamped below at 1e-12, scale = amax / levels. */
void oracle_qat_scales_bits(const float* W, int64_t N, int64_t K, int bits, float* scale) {
  const float levels = oracle_levels(bits);
  for (int64_t i = 0; i < N; ++i) {
    float amax = 0.0f;
    for (int64_t j = 0; j < K; ++j) {
      float a = fabsf(W[i * K + j]);
      if (a > amax) amax = a;
    }
    if (amax < ORACLE_AMAX_FLOOR) amax = ORACLE_AMAX_FLOOR;
    scale[i] = amax / levels;
  }
}

/* The int6 / int8 scale, amax / 127. */
void oracle_qat_scales(const float* W, int64_t N, int64_t K, float* scale) {
  oracle_qat_scales_bits(W, N, K, 8, scale);
}

/* One code from a weight value and its row scale.
 * bits == 6: rne(rne(w/s)/4)*4 clamped to [-128, 124] (64 levels, multiples
 *            of 4 stored in an int8);
 * bits == 8: rne(w/s) clamped to [-127, 127];
 * bits == 5: rne(w/s) clamped to [-15, 15] (s = amax / 15). */
static int oracle_code(float w, float s, int bits) {
  float q_raw = nearbyintf(w / s);
  if (bits == 5) {
    if (q_raw < -15.0f) q_raw = -15.0f;
    if (q_raw > 15.0f) q_raw = 15.0f;
    return (int)q_raw;
  }
  if (bits == 6) {
    float q = nearbyintf(q_raw / 4.0f) * 4.0f;
    if (q < -128.0f) q = -128.0f;
    if (q > 124.0f) q = 124.0f;
    return (int)q;
  }
  if (q_raw < -127.0f) q_raw = -127.0f;
  if (q_raw > 127.0f) q_raw = 127.0f;
  return (int)q_raw;
}

int oracle_qat_codes(const float* W, int64_t N, int64_t K, const float* scale, int bits,
                     int8_t* codes) {
  if (bits != 5 && bits != 6 && bits != 8) return -1;
  for (int64_t i = 0; i < N; ++i)
    for (int64_t j = 0; j < K; ++j)
      codes[i * K + j] = (int8_t)oracle_code(W[i * K + j], scale[i], bits);
  return 0;
}

/* STE forward value: the dequantized weight fl32(c * s). */
void oracle_dequant_f32(const int8_t* codes, const float* scale, int64_t N, int64_t K,
                        float* out) {
  for (int64_t i = 0; i < N; ++i)
    for (int64_t j = 0; j < K; ++j)
      out[i * K + j] = (float)codes[i * K + j] * scale[i];
}

/* The bf16 GEMM operand: bf16_rne(fl32(c * s)) (CastedLinear casts the
 * quantized fp32 weight to the activation dtype). */
void oracle_operand_bf16(const int8_t* codes, const float* scale, int64_t N, int64_t K,
                         uint16_t* out) {
  for (int64_t i = 0; i < N; ++i)
    for (int64_t j = 0; j < K; ++j)
      out[i * K + j] = oracle_bf16_rne((float)codes[i * K + j] * scale[i]);
}

/* ---- export quantizer ------------------------------------------------------ */

static int cmp_float(const void* a, const void* b) {
  float x = *(const float*)a, y = *(const float*)b;
  return (x > y) - (x < y);
}

/* Linear-interpolated quantile of |row| at fraction qf: sort ascending,
 * pos = qf*(n-1) in double, lo = floor(pos), hi = min(lo+1, n-1),
 * frac = fl32(pos - lo), clip = v_lo + frac*(v_hi - v_lo) in three
 * separately rounded fp32 operations. */
float oracle_row_quantile_abs(const float* row, int64_t n, double qf) {
  float* v = (float*)malloc((size_t)n * sizeof(float));
  for (int64_t j = 0; j < n; ++j) v[j] = fabsf(row[j]);
  qsort(v, (size_t)n, sizeof(float), cmp_float);
  double pos = qf * (double)(n - 1);
  int64_t lo = (int64_t)floor(pos);
  if (lo < 0) lo = 0;
  if (lo > n - 1) lo = n - 1;
  int64_t hi = (lo + 1 < n) ? lo + 1 : lo;
  float frac = (float)(pos - (double)lo);
  float d = v[hi] - v[lo];
  float t = frac * d;
  float clip = v[lo] + t;
  free(v);
  return clip;
}

/* Export one matrix: per row clip, fp32 scale s = max(clip,1e-12)/127,
 * codes of clamp(w, -clip, clip) with the same rounding as training,
 * stored scale fp16_rne(s).  scale32 may be NULL. */
static void export_one_row(const float* r, int64_t cols, int bits, double qf, int8_t* codes,
                           uint16_t* scale16, float* scale32) {
  float clip = oracle_row_quantile_abs(r, cols, qf);
  float c = clip < ORACLE_AMAX_FLOOR ? ORACLE_AMAX_FLOOR : clip;
  float s = c / oracle_levels(bits);
  for (int64_t j = 0; j < cols; ++j) {
    float w = r[j];
    if (w > clip) w = clip;
    if (w < -clip) w = -clip;
    codes[j] = (int8_t)oracle_code(w, s, bits);
  }
  *scale16 = oracle_fp16_rne(s);
  *scale32 = s;
}

int oracle_export_rows(const float* W, int64_t rows, int64_t cols, int bits, double qf,
                       int8_t* codes, uint16_t* scale16, float* scale32) {
  if (bits != 5 && bits != 6 && bits != 8) return -1;
  for (int64_t i = 0; i < rows; ++i) {
    float s32;
    export_one_row(W + i * cols, cols, bits, qf, codes + i * cols, scale16 + i, &s32);
    if (scale32) scale32[i] = s32;
  }
  return 0;
}

/* Clip search of the export ("GPTQ-lite 裁剪搜索" of the parameter-golf
 * leaderboard, record "11L EMA + GPTQ-lite + warmdown3500"; the pages name it
 * without defining it).  Reading: per row, each candidate quantile q_k of
 * `cand` (n_cand of them, in the order given) is exported exactly as above;
 * its reconstruction error is E_k = sum_j (w_j - c_j * s16_k)^2, with s16_k
 * the stored fp16 scale read back as fp32 -- what a dequantizing reader gets
 * -- evaluated in double; the row keeps the first candidate of smallest
 * E_k.  Outputs the kept codes and scales, the kept index and every E_k
 * (errs [rows, n_cand]; nullable). */
int oracle_export_rows_search(const float* W, int64_t rows, int64_t cols, int bits,
                              const double* cand, int n_cand, int8_t* codes, uint16_t* scale16,
                              float* scale32, int32_t* chosen, double* errs) {
  if (bits != 5 && bits != 6 && bits != 8) return -1;
  if (n_cand < 1) return -1;
  int8_t* tmp = (int8_t*)malloc((size_t)cols);
  for (int64_t i = 0; i < rows; ++i) {
    const float* r = W + i * cols;
    double best = 0.0;
    int kbest = -1;
    for (int k = 0; k < n_cand; ++k) {
      uint16_t h;
      float s32;
      export_one_row(r, cols, bits, cand[k], tmp, &h, &s32);
      const double sh = (double)oracle_fp16_to_f32(h);
      double e = 0.0;
      for (int64_t j = 0; j < cols; ++j) {
        const double d = (double)r[j] - (double)tmp[j] * sh;
        e += d * d;
      }
      if (errs) errs[i * n_cand + k] = e;
      if (kbest < 0 || e < best) {
        best = e;
        kbest = k;
        for (int64_t j = 0; j < cols; ++j) codes[i * cols + j] = tmp[j];
        scale16[i] = h;
        if (scale32) scale32[i] = s32;
      }
    }
    if (chosen) chosen[i] = kbest;
  }
  free(tmp);
  return 0;
}

/* 6-bit packing of int6 / int5 codes (the bit-packing of the depth-recurrence
 * write-up's Day 0 compression study, which puts int6 codes at about 2.94
 * bits of entropy each; the pages give no format).  Reading: each code
 * becomes one 6-bit two's-complement field -- c / 4 for int6 (codes are
 * multiples of 4 in [-128, 124], so c / 4 is in [-32, 31]), c itself for int5
 * ([-15, 15]) -- and field i occupies bits 6i .. 6i+5 of a little-endian bit
 * stream: bit k of the stream is bit (k mod 8) of byte k / 8.  n codes (n a
 * multiple of 4) give 3n/4 bytes.  Written bit by bit, as the definition. */
int oracle_pack6(const int8_t* codes, int64_t n, int bits, uint8_t* out) {
  if ((bits != 5 && bits != 6) || n % 4 != 0) return -1;
  for (int64_t b = 0; b < 3 * n / 4; ++b) out[b] = 0;
  for (int64_t i = 0; i < n; ++i) {
    const int c = codes[i];
    const int v = bits == 6 ? c / 4 : c;            /* exact: c is a multiple of 4 */
    const unsigned field = (unsigned)v & 63u;       /* two's complement, 6 bits */
    for (int k = 0; k < 6; ++k) {
      const int64_t pos = 6 * i + k;
      if ((field >> k) & 1u) out[pos / 8] |= (uint8_t)(1u << (pos % 8));
    }
  }
  return 0;
}

/* Inverse of oracle_pack6: field i read back bit by bit, sign-extended from 6
 * bits, times 4 for int6. */
int oracle_unpack6(const uint8_t* in, int64_t n, int bits, int8_t* codes) {
  if ((bits != 5 && bits != 6) || n % 4 != 0) return -1;
  for (int64_t i = 0; i < n; ++i) {
    unsigned field = 0;
    for (int k = 0; k < 6; ++k) {
      const int64_t pos = 6 * i + k;
      field |= (unsigned)((in[pos / 8] >> (pos % 8)) & 1u) << k;
    }
    const int v = field >= 32u ? (int)field - 64 : (int)field;
    codes[i] = (int8_t)(bits == 6 ? 4 * v : v);
  }
  return 0;
}

/* Roundtrip dequantize: fl32(c * fp32(scale16)). */
void oracle_dequant_export(const int8_t* codes, const uint16_t* scale16, int64_t rows,
                           int64_t cols, float* out) {
  for (int64_t i = 0; i < rows; ++i) {
    float s = oracle_fp16_to_f32(scale16[i]);
    for (int64_t j = 0; j < cols; ++j) out[i * cols + j] = (float)codes[i * cols + j] * s;
  }
}

/* fp16 passthrough of a whole tensor. */
void oracle_fp16_array(const float* in, int64_t n, uint16_t* out) {
  for (int64_t j = 0; j < n; ++j) out[j] = oracle_fp16_rne(in[j]);
}

void oracle_bf16_array(const float* in, int64_t n, uint16_t* out) {
  for (int64_t j = 0; j < n; ++j) out[j] = oracle_bf16_rne(in[j]);
}

/* ---- Noisy QAT (training-time noise for depth-recurrent cores) ------------ */
/* Source: "Depth Recurrence + Mixed-Precision Quant" write-up (PR #363),
 * section "幸存发现 1 Noisy QAT": for the shared core blocks the forward weight
 * is w + (U(0,1) - 0.5) * amax/127 (per-row amax clamped at 1e-12), the noise
 * drawn without gradient, so the backward is the identity in w.
 *
 * The uniform draws come from Philox-4x32-10 (J. K. Salmon, M. A. Moraes,
 * R. O. Dror, D. E. Shaw, "Parallel random numbers: as easy as 1, 2, 3",
 * SC'11), written here from that definition: ten rounds of
 *   (c0,c1,c2,c3) -> (hi(M1*c2) ^ c1 ^ k0, lo(M1*c2), hi(M0*c0) ^ c3 ^ k1, lo(M0*c0))
 * with M0 = 0xD2511F53, M1 = 0xCD9E8D57, the key bumped by
 * (0x9E3779B9, 0xBB67AE85) before every round after the first.
 * Element e of the row-major [N,K] weight uses output word e % 4 of the block
 * with counter (g, g >> 32, offset, offset >> 32), g = e / 4, and key
 * (seed, seed >> 32); the word x becomes u = (x >> 8) * 2^-24 in [0, 1). */
void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
  uint32_t k0 = key[0], k1 = key[1];
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    uint64_t p0 = (uint64_t)0xD2511F53u * (uint64_t)c0;
    uint64_t p1 = (uint64_t)0xCD9E8D57u * (uint64_t)c2;
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ c1 ^ k0, n1 = lo1, n2 = hi0 ^ c3 ^ k1, n3 = lo0;
    c0 = n0; c1 = n1; c2 = n2; c3 = n3;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* Noisy forward weight of every element and its bf16 operand:
 *   s = fl32(max(amax, 1e-12) / levels), levels 127 (noise at the int8 step, as
 *   the page's code) or 15 (bits == 5: at the int5 step, the page's remark);
 *   noise = fl32(fl32(u - 0.5) * s);
 *   w' = fl32(w + noise);  operand = bf16_rne(w').  (u - 0.5 is exact.) */
void oracle_noisy_operand(const float* W, int64_t N, int64_t K, int bits, uint64_t seed,
                          uint64_t offset, float* scale, float* noisy, uint16_t* operand) {
  oracle_qat_scales_bits(W, N, K, bits, scale);
  uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  for (int64_t i = 0; i < N; ++i) {
    for (int64_t j = 0; j < K; ++j) {
      int64_t e = i * K + j;
      uint64_t g = (uint64_t)e >> 2;
      uint32_t ctr[4] = {(uint32_t)g, (uint32_t)(g >> 32), (uint32_t)offset,
                         (uint32_t)(offset >> 32)};
      uint32_t x[4];
      oracle_philox4x32_10(ctr, key, x);
      float u = (float)(x[e & 3] >> 8) * 5.9604644775390625e-08f;
      float noise = (u - 0.5f) * scale[i];
      float w = W[e] + noise;
      if (noisy) noisy[e] = w;
      if (operand) operand[e] = oracle_bf16_rne(w);
    }
  }
}
