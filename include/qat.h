/*
 * qat.h -- C ABI of the B200 (sm_100a) int6 quantization-aware linear, ReLU^2
 * MLP, recurrent-core weight cache and export quantizer (with the int5 grid,
 * Noisy QAT and the LeakyReLU(0.5)^2 MLP of the depth-recurrence write-up).
 *
 * Page references used below (title, section):
 *   [P5] "parameter-golf 16MB 极限压缩实战：11L MLP3x + Int6 QAT + zstd-22 记录详解"
 *   [P1] "Depth Recurrence + Mixed-Precision Quant" write-up of PR #363
 *   [P4] "openai/parameter-golf" README mirror, leaderboard table
 *
 * Conventions shared by every call
 *   - Every pointer is a caller-owned DEVICE pointer unless stated otherwise,
 *     row-major and contiguous (a leading-dimension argument says otherwise),
 *     16-byte aligned.  Nothing is retained after a call returns.
 *   - bf16 / fp16 tensors are passed as their 16-bit storage (qat_bf16 /
 *     qat_fp16).  fp32 is IEEE binary32.
 *   - Every call is asynchronous on the given CUDA stream and never
 *     synchronizes.  The library never allocates device memory: scratch
 *     comes from the caller's workspace, sized by qat_workspace_size().
 *   - Arguments are validated on the host before any launch; on error
 *     nothing is launched and a QAT_ERR_* code is returned.
 *   - bits = 6 selects the int6 grid (multiples of 4 in [-128,124], 64
 *     levels in an int8 container); bits = 8 the int8 grid [-127,127];
 *     bits = 5 the int5 grid [-15,15] with scale amax/15 ([P1] "幸存发现 1
 *     Noisy QAT" gives amax/15 as the int5 step; its reproduction commands
 *     switch MLP and attention weights to int5 with MLP_INT5 / ATTN_INT5).
 *   - Shapes: feature dimensions (N, K, d, H, cols) must be multiples of 8
 *     (16-byte rows for bf16, as the tensor-memory-access engine requires);
 *     the token count T may be anything >= 0 (T = 0 is a no-op).
 *   - Bounded device waits: every wait inside a kernel gives up after ~2 s,
 *     records QAT_ERR_TIMEOUT in a device flag and lets the kernel return;
 *     qat_device_error() reads and clears that flag.
 */
#ifndef QAT_B200_H
#define QAT_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* qat_stream_t; /* a cudaStream_t; NULL = legacy default stream */
typedef uint16_t qat_bf16;                /* bfloat16 bit pattern */
typedef uint16_t qat_fp16;                /* IEEE binary16 bit pattern */

enum {
  QAT_OK = 0,
  QAT_ERR_ARG = 1,        /* null pointer, non-positive size, bits not in {5,6,8} */
  QAT_ERR_ALIGN = 2,      /* a pointer is not 16-byte aligned */
  QAT_ERR_SHAPE = 3,      /* a feature dimension is not a multiple of 8, or too large */
  QAT_ERR_WORKSPACE = 4,  /* workspace missing or smaller than qat_workspace_size() */
  QAT_ERR_CUDA = 5,       /* a CUDA runtime call or kernel launch failed */
  QAT_ERR_TIMEOUT = 6,    /* a bounded device wait gave up (see qat_device_error) */
  QAT_ERR_UNSUPPORTED = 7 /* no sm_100 device, or driver entry point missing */
};

/* Human-readable text of a QAT_* code (static storage, never NULL). */
const char* qat_strerror(int code);

/* Number of kernels this library has launched in this process (all streams). */
int64_t qat_launch_count(void);

/* Synchronizes `stream`, then returns QAT_OK, or QAT_ERR_TIMEOUT if any kernel
 * of this library recorded a timed-out device wait since the last call
 * (the flag is cleared), or QAT_ERR_CUDA if the stream reports an error. */
int qat_device_error(qat_stream_t stream);

/* ---------------------------------------------------------------------------
 * Quantized weight: the STE forward operand of one weight matrix.
 * Produced by qat_quantize_weights(); it is also the recurrence cache of [P1]
 * "税 1" (shared weights are stored once and quantized once, then reused by
 * every application of the block).
 *   operand : [N,K] bf16 = bf16_rne(fl32(c * s)), required by every GEMM call
 *   scales  : [N] fp32 per-row scales s (may be NULL)
 *   codes   : [N,K] int8 codes c (may be NULL)
 * ------------------------------------------------------------------------- */
typedef struct qat_qweight {
  const qat_bf16* operand;
  const float* scales;
  const int8_t* codes;
  int32_t N, K, bits;
} qat_qweight;

/* [P5] "训练时的模拟量化": per row i of W [N,K] fp32,
 *   amax_i = max(max_j |W_ij|, 1e-12)      (floor from [P1] "修复" code)
 *   s_i    = fl32(amax_i / 127)             (IEEE division; / 15 for int5)
 *   int6:  c = clamp(4*rne(rne(fl32(W/s))/4), -128, 124);  int8: clamp(rne(W/s), -127, 127)
 *   int5:  c = clamp(rne(fl32(W/s)), -15, 15)
 *   operand = bf16_rne(fl32(c * s))         (the STE forward value cast to bf16)
 * Outputs: scales [N] (required), codes [N,K] (nullable), operand [N,K] (nullable).
 * Bit-exact with the CPU oracle. */
int qat_quantize_weights(const float* W, int32_t N, int32_t K, int32_t bits, int8_t* codes,
                         float* scales, qat_bf16* operand, qat_stream_t stream);

/* [P5] "训练时的模拟量化", as qat_quantize_weights, for several weights in one
 * launch (all of a training step's weights, each on its own grid; the pages
 * quantize every CastedLinear weight at every step): descs[i] holds W [N,K] fp32, bits,
 * scales [N] (required), codes [N,K] and operand [N,K] (nullable) exactly as
 * qat_quantize_weights takes them.  1 <= n <= QAT_QUANT_MAX_DESCS; the
 * descriptor array is read on the host during the call.  Each weight's
 * outputs are bit-identical to a qat_quantize_weights call on it; outputs
 * must not overlap one another or any W. */
#define QAT_QUANT_MAX_DESCS 16
typedef struct qat_quant_desc {
  const float* W;
  int8_t* codes;
  float* scales;
  qat_bf16* operand;
  int32_t N, K, bits, pad;
} qat_quant_desc;
int qat_quantize_weights_batch(const qat_quant_desc* descs, int32_t n, qat_stream_t stream);

/* Noisy QAT for the shared blocks of a depth-recurrent core ([P1] "幸存发现 1
 * Noisy QAT"): instead of the STE fake quantization, the forward weight is
 *   w' = fl32(w + fl32(fl32(u - 1/2) * s)),  s = fl32(max(amax_row, 1e-12) / L),
 * L = 127 (the int8 step of the page's code) for bits 6 or 8, L = 15 for
 * bits = 5 (the int5-matched step the page proposes for an int5 export),
 * u uniform in [0,1), and the gradient flows through w' to w unchanged (the
 * noise carries none), so the backward is qat_linear_bwd with this operand.
 * u comes from Philox-4x32-10 (Salmon et al., SC'11): element e of the
 * row-major [N,K] weight uses word e % 4 of the block with counter
 * (e/4 low, e/4 high, offset low, offset high) and key (seed low, seed high);
 * u = (word >> 8) * 2^-24.  Outputs: operand [N,K] bf16 = bf16_rne(w')
 * (required; pass it as qat_qweight.operand), scales [N] fp32 (nullable).
 * Bit-exact with the CPU oracle.  Use a fresh offset per draw. */
int qat_noisy_operand(const float* W, int32_t N, int32_t K, int32_t bits, uint64_t seed,
                      uint64_t offset, float* scales, qat_bf16* operand, qat_stream_t stream);

/* Workspace sizes (bytes) for the calls below.  `raw_weights` != 0 means the
 * call is given fp32 weights to quantize itself (the workspace then also
 * holds the bf16 operands and scales); 0 means qat_qweight operands. */
enum { QAT_OP_LINEAR_FWD = 1, QAT_OP_LINEAR_BWD = 2, QAT_OP_MLP_FWD = 3, QAT_OP_MLP_BWD = 4 };
size_t qat_workspace_size(int32_t op, int32_t N_or_d, int32_t K_or_H, int64_t T,
                          int32_t raw_weights);

/* [P5] CastedLinear forward with QAT: Y[T,N] = bf16( X[T,K] . Wq^T (+ residual) ),
 * fp32 accumulation on the tensor cores.  Weights: either W (fp32 [N,K],
 * quantized inside the call) or qw (pre-quantized; W must then be NULL).
 * ldx = row stride of X in elements (0 -> K); residual (nullable) is [T,N]
 * bf16 and may alias Y exactly.
 * With W, one of two paths, both giving bf16(fl32(c * s)) as the operand:
 *   - with a workspace (qat_workspace_size() bytes), the weight is quantized
 *     into it first and the GEMM reads the bf16 operand from there -- the
 *     faster path on B200 at every measured size;
 *   - with workspace == NULL, the fused quantizing producer: the GEMM itself
 *     computes each row's amax, scale, codes and bf16 operand in shared
 *     memory, so the quantized weight never reaches global memory and no
 *     scratch is needed.  Needs T >= 256 and K <= 1024 (a CTA pair holds the
 *     whole B_ROWS x K slice of its N block); otherwise QAT_ERR_WORKSPACE. */
int qat_linear_fwd(const float* W, const qat_qweight* qw, int32_t N, int32_t K, int32_t bits,
                   const qat_bf16* X, int64_t ldx, int64_t T, const qat_bf16* residual,
                   qat_bf16* Y, void* workspace, size_t ws_bytes, qat_stream_t stream);

/* STE backward of qat_linear_fwd ([P5]: the forward uses the quantized weight,
 * the gradient flows to the fp32 weight unchanged):
 *   dX[T,K] = bf16( dY[T,N] . Wq (+ dX_residual) )   (nullable)
 *   dW[N,K] (+)= dY^T . X   in fp32                   (nullable; accumulate_dW != 0
 *                                                      adds into dW, e.g. over the
 *                                                      R uses of a recurrent weight)
 * dX needs W or qw; dW needs neither.  ldx = row stride of X in elements
 * (0 -> K; a multiple of 8, >= K), so X may be a column slice of a wider
 * activation.  dX_residual (nullable, [T,K] bf16, needs dX) is added to the
 * fp32 product before the bf16 rounding -- the gradient of a residual
 * connection around the linear -- and may alias dX exactly.  With T = 0, dW
 * is zeroed unless accumulate_dW. */
int qat_linear_bwd(const float* W, const qat_qweight* qw, int32_t N, int32_t K, int32_t bits,
                   const qat_bf16* X, int64_t ldx, const qat_bf16* dY, int64_t T,
                   const qat_bf16* dX_residual, qat_bf16* dX, float* dW, int32_t accumulate_dW,
                   void* workspace, size_t ws_bytes, qat_stream_t stream);

/* MLP activations: [P5] "架构" relu(x)^2, and leaky_relu(x, 0.5)^2 ([P1]
 * negative result #9 "LeakyReLU(0.5)²"; [P4] leaderboard entries use it). */
enum { QAT_ACT_RELU2 = 0, QAT_ACT_LEAKY_RELU2 = 1 };

/* [P5] "架构" ReLU^2 MLP forward, both linears int5/int6/int8 QAT
 * (given Wfc and workspace == NULL, the fc GEMM quantizes Wfc in its own
 * producer as qat_linear_fwd does; proj then needs qproj and h_save):
 *   pre = X . Wfc_q^T  [T,H];  h = act(pre) (fused in the fc epilogue, from the
 *   fp32 accumulator: relu(pre)^2, or for QAT_ACT_LEAKY_RELU2 t^2 with t = pre
 *   (pre > 0) else pre/2);  Y = bf16(h . Wproj_q^T (+ residual))  [T,d].
 * Weights: (Wfc [H,d], Wproj [d,H]) fp32, or (qfc, qproj).  pre_save [T,H]
 * (nullable) and h_save [T,H] (nullable; the workspace holds h otherwise)
 * keep the activations for the backward.  residual may alias Y exactly. */
int qat_mlp_fwd(const float* Wfc, const float* Wproj, const qat_qweight* qfc,
                const qat_qweight* qproj, int32_t d, int32_t H, int32_t bits, int32_t act,
                const qat_bf16* X, int64_t T, const qat_bf16* residual, qat_bf16* Y,
                qat_bf16* pre_save, qat_bf16* h_save, void* workspace, size_t ws_bytes,
                qat_stream_t stream);

/* STE backward of qat_mlp_fwd from the saved pre and h:
 *   dh = dY . Wproj_q;  dpre = dh * act'(pre) (fused in the dh epilogue:
 *   2*relu(pre), or for QAT_ACT_LEAKY_RELU2 2*pre (pre > 0) else pre/2);
 *   dWproj (+)= dY^T . h;  dWfc (+)= dpre^T . X;
 *   dX = bf16( dpre . Wfc_q (+ dX_residual) ).
 * dX, dWfc, dWproj may each be NULL.  dX_residual (nullable, [T,d] bf16,
 * needs dX; may alias dX exactly) adds the gradient that bypasses the MLP
 * through a residual connection.  dpre_save (nullable, [T,H] bf16) receives
 * dpre -- e.g. to form dWfc later over several token batches in one call --
 * else the workspace holds it (qat_workspace_size counts it either way). */
int qat_mlp_bwd(const float* Wfc, const float* Wproj, const qat_qweight* qfc,
                const qat_qweight* qproj, int32_t d, int32_t H, int32_t bits, int32_t act,
                const qat_bf16* X, const qat_bf16* pre, const qat_bf16* h, const qat_bf16* dY,
                int64_t T, const qat_bf16* dX_residual, qat_bf16* dX, qat_bf16* dpre_save,
                float* dWfc, float* dWproj, int32_t accumulate_dW, void* workspace,
                size_t ws_bytes, qat_stream_t stream);

/* Diagnostic (the pages have no counterpart): runs the library's bounded
 * device wait on a barrier that nothing arrives on, with a limit of limit_ns
 * (1 us .. 10 s, else QAT_ERR_ARG).  The wait gives up, records
 * QAT_ERR_TIMEOUT in the device error flag and the kernel returns: the next
 * qat_device_error() returns QAT_ERR_TIMEOUT (and clears the flag) and the
 * context stays usable.  Lets a caller check its failure handling without a
 * GPU fault. */
int qat_selftest_wait_timeout(int64_t limit_ns, qat_stream_t stream);

/* ---------------------------------------------------------------------------
 * qat_linear_fwd_noalloc -- the QAT linear forward from fp32 weights that
 * allocates nothing and takes no workspace.  The pages have no counterpart:
 * this is a library convenience for callers that cannot allocate device
 * memory themselves (a plugin inside a framework that owns all device memory
 * through its own pool, a fixed-budget service that allocates only at
 * start-up, latency-critical code that cannot afford the synchronization
 * cudaMalloc / cudaFree may cause).
 *   Computes what qat_linear_fwd computes when given W, always by quantizing
 *   into the array first and then running the GEMM:
 *   Y[T,N] = bf16( X[T,K] . bf16(fl32(c*s))^T (+ residual) ).
 *   Scratch: a fixed device array inside the library holds the bf16 operand and
 *   the scales -- at most QAT_NOALLOC_MAX_ELEMS weights (N*K) and
 *   QAT_NOALLOC_MAX_ROWS rows; larger weights return QAT_ERR_SHAPE.  Every GPU
 *   that loads the library holds this array (8 MiB + 64 KiB) until exit.
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current); make that first call
 *   before any stream capture.  The address is cached per process and per
 *   device's primary context: after cudaDeviceReset on a device, the cached
 *   address is stale and this entry point must not be called there again.
 *   All calls share the array and each rewrites what it reads, so nothing
 *   must start at zero; calls whose kernels overlap on the GPU (other streams
 *   or host threads on the same device) race on it -- serialize them.
 * Other arguments, errors and aliasing rules as qat_linear_fwd. */
#define QAT_NOALLOC_MAX_ELEMS 4194304
#define QAT_NOALLOC_MAX_ROWS 16384
int qat_linear_fwd_noalloc(const float* W, int32_t N, int32_t K, int32_t bits,
                           const qat_bf16* X, int64_t ldx, int64_t T,
                           const qat_bf16* residual, qat_bf16* Y, qat_stream_t stream);

/* ---------------------------------------------------------------------------
 * Export quantizer, [P5] "后训练量化导出".
 * Per row of W [rows, cols] fp32:
 *   clip   = linear-interpolated quantile of |w| at q = 0.9999984: sorted
 *            values v, pos = q*(cols-1) (double), lo = floor(pos), hi = lo+1,
 *            clip = fl32(v_lo + fl32(fl32(pos-lo) * fl32(v_hi - v_lo)))
 *   s32    = fl32(max(clip, 1e-12) / 127)   (/ 15 for bits = 5)
 *   codes  = the training grid (bits 5, 6 or 8) applied to clamp(w, -clip, clip) with s32
 *   scales = fp16_rne(s32)
 * Only the top (cols - lo) order statistics of |w| matter; rows longer than
 * 625,001 columns (where more than the top two would) return QAT_ERR_SHAPE.
 * Bit-exact with the CPU oracle.
 * ------------------------------------------------------------------------- */
int quantize_rows_export(const float* W, int64_t rows, int64_t cols, int32_t bits,
                         int8_t* codes, qat_fp16* scales, qat_stream_t stream);

/* One grouped launch over a whole state dict.  `descs` is a HOST array of n
 * descriptors (n <= QAT_EXPORT_MAX_DESCS); mode 5, 6 or 8 quantizes rows as
 * above into dst (int8 codes) and scales; mode QAT_EXPORT_FP16 converts src
 * to fp16 (rne) into dst (the passthrough of non-2D, small and tied-embedding
 * tensors; scales unused).  The caller applies the passthrough rules.
 * flags: 0, or QAT_EXPORT_PACK6 with mode 5 or 6 -- dst then receives the codes
 * 6-bit packed (see unpack_codes6), rows*cols*3/4 bytes, row r at byte
 * r*cols*3/4 (the bit-packing of [P1] Day 0; the format is this library's:
 * one 6-bit two's-complement field per code, c/4 for int6 and c for int5,
 * field i at bits 6i..6i+5 of a little-endian bit stream).
 * QAT_EXPORT_CLIP_SEARCH (modes 5, 6, 8; may be combined with PACK6): instead
 * of the fixed 99.99984 percentile, each row tries the clip quantiles
 * q = 1.0, 0.9999984, 0.99999, 0.9999, 0.9995, 0.999 (in this order; each
 * exported as above) and keeps the first whose stored row has the least
 * squared error sum_j (w_j - c_j * fp32(scale_fp16))^2, computed in fp32 (the
 * [P4] leaderboard's "GPTQ-lite" clip search, which the pages do not define;
 * this is the library's reading).  Rows of more than 2048 columns return
 * QAT_ERR_SHAPE.  Other flags, or PACK6 with another mode, return
 * QAT_ERR_ARG. */
#define QAT_EXPORT_FP16 16
#define QAT_EXPORT_MAX_DESCS 256
#define QAT_EXPORT_PACK6 1
#define QAT_EXPORT_CLIP_SEARCH 2
typedef struct qat_export_desc {
  const float* src;
  int64_t rows, cols;
  int32_t mode;
  int32_t flags;
  void* dst;
  qat_fp16* scales;
} qat_export_desc;
int quantize_export_batch(const qat_export_desc* descs, int32_t n, qat_stream_t stream);

/* Unpacks n 6-bit packed codes (QAT_EXPORT_PACK6 layout, 3n/4 bytes at
 * `packed`) into n int8 codes: the field sign-extended, times 4 for bits = 6.
 * n must be a multiple of 8 (QAT_ERR_SHAPE otherwise); bits 5 or 6.  Both
 * pointers are device pointers, 16-byte aligned.  Bit-exact with the oracle. */
int unpack_codes6(const uint8_t* packed, int64_t n, int32_t bits, int8_t* codes,
                  qat_stream_t stream);

/* Roundtrip dequantize ([P5] "后训练量化导出", roundtrip re-evaluation):
 *   out = fl32(c * fp32(scale_fp16))  as fp32 (out_dtype 0) or bf16_rne of it (1).
 * codes int8 [rows, cols] row-major, scales fp16 [rows] (one per row, as
 * quantize_rows_export writes them), out [rows, cols] row-major; all device
 * pointers, caller-owned.  cols a positive multiple of 8 (QAT_ERR_SHAPE), codes
 * and out 16-byte aligned (QAT_ERR_ALIGN), a null pointer, rows < 0 or another
 * out_dtype QAT_ERR_ARG; more than 2^41 groups of four codes (rows * cols / 4:
 * one thread block per 1,024 groups) QAT_ERR_SHAPE.  Bit-exact with the
 * oracle. */
enum { QAT_DTYPE_F32 = 0, QAT_DTYPE_BF16 = 1 };
int dequantize_rows(const int8_t* codes, const qat_fp16* scales, int64_t rows, int64_t cols,
                    int32_t out_dtype, void* out, qat_stream_t stream);

/* Grouped dequantize_rows: the rows of up to QAT_DEQUANT_MAX_DESCS tensors in
 * one launch (a state dict's roundtrip), each descriptor the arguments of one
 * dequantize_rows call.  Every descriptor is checked as dequantize_rows checks
 * its arguments before anything launches; the first failing one decides the
 * error.  n outside 1 .. QAT_DEQUANT_MAX_DESCS or a null array: QAT_ERR_ARG;
 * more than 2^31 - 1 thread blocks in all (one per 1,024 groups of four codes
 * of a tensor, each tensor rounded up to whole blocks): QAT_ERR_SHAPE. */
#define QAT_DEQUANT_MAX_DESCS 256
typedef struct qat_dequant_desc {
  const int8_t* codes;
  const qat_fp16* scales;
  int64_t rows, cols;
  int32_t out_dtype;
  int32_t reserved; /* 0 */
  void* out;
} qat_dequant_desc;
int dequantize_rows_batch(const qat_dequant_desc* descs, int32_t n, qat_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* QAT_B200_H */
