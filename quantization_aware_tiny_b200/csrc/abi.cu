// extern "C" entry points declared in include/qat.h: argument checks on the
// host, workspace carving, and the sequencing of quantizer and GEMM launches.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "gemm_sm100.cuh"
#include "quant.cuh"

namespace qat {

// The one device-side error flag (per device, zero-initialised at load).
__device__ int g_device_error = 0;

// Per-device caches below are filled on first use with the device current;
// concurrent first calls from several host threads store the same value.
int* device_error_ptr() {
  static std::atomic<int*> cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  int* p = cached[dev].load(std::memory_order_acquire);
  if (!p) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_device_error) != cudaSuccess) return nullptr;
    p = static_cast<int*>(a);
    cached[dev].store(p, std::memory_order_release);
  }
  return p;
}

static std::atomic<int64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int sm_count() {
  static std::atomic<int> cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

bool device_flag_once(std::atomic<uint64_t>& done, int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  if (dev_out) *dev_out = dev;
  if (dev < 0 || dev >= 64) return false;
  return (done.load(std::memory_order_acquire) >> dev) & 1u;
}

void device_flag_set(std::atomic<uint64_t>& done, int dev) {
  if (dev >= 0 && dev < 64) done.fetch_or(uint64_t{1} << dev, std::memory_order_acq_rel);
}

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Carves 256-byte aligned pieces from the caller's workspace.
struct Carver {
  uint8_t* base;
  size_t cap, used = 0;
  Carver(void* b, size_t c) : base(static_cast<uint8_t*>(b)), cap(c) {}
  void* take(size_t bytes) {
    const size_t at = used;
    used = align_up(used + bytes);
    return (base && used <= cap) ? base + at : nullptr;
  }
};

inline size_t operand_bytes(int64_t N, int64_t K) { return align_up(N * K * 2) + align_up(N * 4); }

bool bits_ok(int bits) { return bits == 5 || bits == 6 || bits == 8; }
bool act_ok(int act) { return act == QAT_ACT_RELU2 || act == QAT_ACT_LEAKY_RELU2; }
bool dim_ok(int64_t x) { return x > 0 && (x & 7) == 0 && x <= (1 << 20); }

// The bf16 operand of a weight: taken from `qw`, or produced from fp32 `W`
// into the workspace.  Exactly one of W / qw must be given.
int get_operand(const float* W, const qat_qweight* qw, int64_t N, int64_t K, int bits, Carver& ws,
                cudaStream_t s, const __nv_bfloat16** out) {
  if ((W == nullptr) == (qw == nullptr)) return QAT_ERR_ARG;
  if (qw) {
    if (!qw->operand || qw->N != N || qw->K != K) return QAT_ERR_ARG;
    if (!aligned16(qw->operand)) return QAT_ERR_ALIGN;
    *out = reinterpret_cast<const __nv_bfloat16*>(qw->operand);
    return QAT_OK;
  }
  if (!aligned16(W)) return QAT_ERR_ALIGN;
  void* op = ws.take(N * K * 2);
  void* sc = ws.take(N * 4);
  if (!op || !sc) return QAT_ERR_WORKSPACE;
  const int rc = launch_quantize_weights(W, static_cast<int>(N), static_cast<int>(K), bits, nullptr,
                                         static_cast<float*>(sc),
                                         static_cast<__nv_bfloat16*>(op), s);
  *out = static_cast<const __nv_bfloat16*>(op);
  return rc;
}

}  // namespace
}  // namespace qat

using namespace qat;

extern "C" {

const char* qat_strerror(int code) {
  switch (code) {
    case QAT_OK: return "ok";
    case QAT_ERR_ARG: return "invalid argument";
    case QAT_ERR_ALIGN: return "pointer not 16-byte aligned";
    case QAT_ERR_SHAPE: return "unsupported shape (feature dims must be multiples of 8)";
    case QAT_ERR_WORKSPACE: return "workspace missing or too small";
    case QAT_ERR_CUDA: return "CUDA runtime error";
    case QAT_ERR_TIMEOUT: return "a bounded device wait timed out";
    case QAT_ERR_UNSUPPORTED: return "unsupported device or driver";
    default: return "unknown error";
  }
}

int64_t qat_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int qat_device_error(qat_stream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return QAT_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return QAT_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess)
    return QAT_ERR_CUDA;
  return v;
}

int qat_noisy_operand(const float* W, int32_t N, int32_t K, int32_t bits, uint64_t seed,
                      uint64_t offset, float* scales, qat_bf16* operand, qat_stream_t stream) {
  if (!W || !operand || N <= 0 || !bits_ok(bits)) return QAT_ERR_ARG;
  if (!dim_ok(K)) return QAT_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(operand)) return QAT_ERR_ALIGN;
  return launch_noisy_operand(W, N, K, bits, seed, offset, scales,
                              reinterpret_cast<__nv_bfloat16*>(operand), stream);
}

size_t qat_workspace_size(int32_t op, int32_t N_or_d, int32_t K_or_H, int64_t T,
                          int32_t raw_weights) {
  const int64_t a = N_or_d, b = K_or_H;
  if (a <= 0 || b <= 0 || T < 0) return 0;
  switch (op) {
    case QAT_OP_LINEAR_FWD:
    case QAT_OP_LINEAR_BWD:
      return raw_weights ? operand_bytes(a, b) : 0;
    case QAT_OP_MLP_FWD:  // h [T,H] when not saved by the caller, + operands of fc [H,d], proj [d,H]
    case QAT_OP_MLP_BWD:  // dpre [T,H] + operands
      return align_up(static_cast<size_t>(T) * b * 2) +
             (raw_weights ? operand_bytes(b, a) + operand_bytes(a, b) : 0);
    default:
      return 0;
  }
}

int qat_quantize_weights(const float* W, int32_t N, int32_t K, int32_t bits, int8_t* codes,
                         float* scales, qat_bf16* operand, qat_stream_t stream) {
  if (!W || !scales || N <= 0 || !bits_ok(bits)) return QAT_ERR_ARG;
  if (!dim_ok(K)) return QAT_ERR_SHAPE;
  if (!aligned16(W) || (codes && !aligned16(codes)) || (operand && !aligned16(operand)))
    return QAT_ERR_ALIGN;
  return launch_quantize_weights(W, N, K, bits, codes, scales,
                                 reinterpret_cast<__nv_bfloat16*>(operand), stream);
}

int qat_quantize_weights_batch(const qat_quant_desc* descs, int32_t n, qat_stream_t stream) {
  if (!descs || n <= 0 || n > QAT_QUANT_MAX_DESCS) return QAT_ERR_ARG;
  QuantBatch b;
  b.n = n;
  b.tile_begin[0] = 0;
  for (int i = 0; i < n; ++i) {
    const qat_quant_desc& s = descs[i];
    if (!s.W || !s.scales || s.N <= 0 || !bits_ok(s.bits)) return QAT_ERR_ARG;
    if (!dim_ok(s.K)) return QAT_ERR_SHAPE;
    if (!aligned16(s.W) || (s.codes && !aligned16(s.codes)) || (s.operand && !aligned16(s.operand)))
      return QAT_ERR_ALIGN;
    b.d[i] = QuantDescDev{s.W, s.codes, s.scales, reinterpret_cast<__nv_bfloat16*>(s.operand),
                          s.N, s.K, s.bits, 0};
    b.tile_begin[i + 1] = b.tile_begin[i] + quant_tiles(s.N, s.K);
  }
  return launch_quantize_batch(b, stream);
}

int qat_linear_fwd(const float* W, const qat_qweight* qw, int32_t N, int32_t K, int32_t bits,
                   const qat_bf16* X, int64_t ldx, int64_t T, const qat_bf16* residual,
                   qat_bf16* Y, void* workspace, size_t ws_bytes, qat_stream_t stream) {
  if ((T > 0 && (!X || !Y)) || T < 0 || !bits_ok(bits)) return QAT_ERR_ARG;
  if (!dim_ok(N) || !dim_ok(K)) return QAT_ERR_SHAPE;
  if (ldx == 0) ldx = K;
  if (ldx < K || (ldx & 7)) return QAT_ERR_SHAPE;
  if (T == 0) return ((W == nullptr) != (qw == nullptr)) ? QAT_OK : QAT_ERR_ARG;
  GemmDesc g;
  g.A = X; g.lda = ldx;
  g.M = T; g.N = N; g.K = K;
  g.epi = residual ? EPI_BF16_RESID : EPI_BF16;
  g.D = Y; g.ldd = N;
  g.R = residual; g.ldr = N;
  if (W && !qw && workspace == nullptr && fused_b_supported(T, N, K, g.epi)) {
    // no workspace: the GEMM quantizes W itself, the operand never reaches global memory
    if (!aligned16(W)) return QAT_ERR_ALIGN;
    g.Wraw = W;
    g.bits = bits;
    return launch_gemm(g, stream);
  }
  Carver ws(workspace, ws_bytes);
  const __nv_bfloat16* op = nullptr;
  int rc = get_operand(W, qw, N, K, bits, ws, stream, &op);
  if (rc) return rc;
  g.B = op; g.ldb = K;
  return launch_gemm(g, stream);
}

int qat_linear_bwd(const float* W, const qat_qweight* qw, int32_t N, int32_t K, int32_t bits,
                   const qat_bf16* X, int64_t ldx, const qat_bf16* dY, int64_t T,
                   const qat_bf16* dX_residual, qat_bf16* dX, float* dW, int32_t accumulate_dW,
                   void* workspace, size_t ws_bytes, qat_stream_t stream) {
  if ((T > 0 && !dY) || T < 0 || !bits_ok(bits)) return QAT_ERR_ARG;
  if (!dim_ok(N) || !dim_ok(K)) return QAT_ERR_SHAPE;
  if (T > 0 && dW && !X) return QAT_ERR_ARG;
  if (dX_residual && !dX) return QAT_ERR_ARG;
  if (ldx == 0) ldx = K;
  if (ldx < K || (ldx & 7)) return QAT_ERR_SHAPE;
  Carver ws(workspace, ws_bytes);
  if (dX) {
    const __nv_bfloat16* op = nullptr;
    int rc = get_operand(W, qw, N, K, bits, ws, stream, &op);
    if (rc) return rc;
    if (T > 0) {
      GemmDesc g;  // dX[T,K] = dY[T,N] . Wq[N,K] (+ residual): B = Wq read N-major along K
      g.A = dY; g.lda = N;
      g.B = op; g.ldb = K; g.b_mn = true;
      g.M = T; g.N = K; g.K = N;
      g.epi = dX_residual ? EPI_BF16_RESID : EPI_BF16;
      g.D = dX; g.ldd = K;
      g.R = dX_residual; g.ldr = K;
      rc = launch_gemm(g, stream);
      if (rc) return rc;
    }
  }
  if (dW) {
    if (T == 0) {
      if (!accumulate_dW) return cuda_status(cudaMemsetAsync(dW, 0, static_cast<size_t>(N) * K * 4, stream));
      return QAT_OK;
    }
    GemmDesc g;  // dW[N,K] = dY^T . X : both operands read along T
    g.A = dY; g.lda = N; g.a_mn = true;
    g.B = X; g.ldb = ldx; g.b_mn = true;
    g.M = N; g.N = K; g.K = T;
    g.epi = EPI_F32;
    g.D = dW; g.ldd = K;
    g.accumulate = accumulate_dW != 0;
    return launch_gemm(g, stream);
  }
  return QAT_OK;
}

int qat_mlp_fwd(const float* Wfc, const float* Wproj, const qat_qweight* qfc,
                const qat_qweight* qproj, int32_t d, int32_t H, int32_t bits, int32_t act,
                const qat_bf16* X, int64_t T, const qat_bf16* residual, qat_bf16* Y,
                qat_bf16* pre_save, qat_bf16* h_save, void* workspace, size_t ws_bytes,
                qat_stream_t stream) {
  if ((T > 0 && (!X || !Y)) || T < 0 || !bits_ok(bits) || !act_ok(act)) return QAT_ERR_ARG;
  if (!dim_ok(d) || !dim_ok(H)) return QAT_ERR_SHAPE;
  if ((pre_save && !aligned16(pre_save)) || (h_save && !aligned16(h_save))) return QAT_ERR_ALIGN;
  Carver ws(workspace, ws_bytes);
  const __nv_bfloat16 *op_fc = nullptr, *op_proj = nullptr;
  const int fc_epi = act == QAT_ACT_RELU2 ? EPI_RELU2 : EPI_LRELU2;
  // fc from fp32 weights and no workspace: the fc GEMM quantizes Wfc itself
  const bool fc_fused = Wfc && !qfc && !workspace && T > 0 && fused_b_supported(T, H, d, fc_epi);
  int rc = QAT_OK;
  if (fc_fused) {
    if (!aligned16(Wfc)) return QAT_ERR_ALIGN;
  } else {
    rc = get_operand(Wfc, qfc, H, d, bits, ws, stream, &op_fc);
    if (rc) return rc;
  }
  rc = get_operand(Wproj, qproj, d, H, bits, ws, stream, &op_proj);
  if (rc) return rc;
  if (T == 0) return QAT_OK;
  void* h = h_save;
  if (!h) {
    h = ws.take(static_cast<size_t>(T) * H * 2);
    if (!h) return QAT_ERR_WORKSPACE;
  }
  GemmDesc g1;  // pre = X . Wfc^T ; h = act(pre)
  g1.A = X; g1.lda = d;
  g1.B = op_fc; g1.ldb = d;
  if (fc_fused) {
    g1.Wraw = Wfc;
    g1.bits = bits;
  }
  g1.M = T; g1.N = H; g1.K = d;
  g1.epi = fc_epi;
  g1.D = pre_save; g1.ldd = H;
  g1.D2 = h; g1.ldd2 = H;
  rc = launch_gemm(g1, stream);
  if (rc) return rc;
  GemmDesc g2;  // Y = h . Wproj^T (+ residual)
  g2.A = h; g2.lda = H;
  g2.B = op_proj; g2.ldb = H;
  g2.M = T; g2.N = d; g2.K = H;
  g2.epi = residual ? EPI_BF16_RESID : EPI_BF16;
  g2.D = Y; g2.ldd = d;
  g2.R = residual; g2.ldr = d;
  return launch_gemm(g2, stream);
}

int qat_mlp_bwd(const float* Wfc, const float* Wproj, const qat_qweight* qfc,
                const qat_qweight* qproj, int32_t d, int32_t H, int32_t bits, int32_t act,
                const qat_bf16* X, const qat_bf16* pre, const qat_bf16* h, const qat_bf16* dY,
                int64_t T, const qat_bf16* dX_residual, qat_bf16* dX, qat_bf16* dpre_save,
                float* dWfc, float* dWproj, int32_t accumulate_dW, void* workspace,
                size_t ws_bytes, qat_stream_t stream) {
  if ((T > 0 && (!X || !pre || !h || !dY)) || T < 0 || !bits_ok(bits) || !act_ok(act))
    return QAT_ERR_ARG;
  if (dX_residual && !dX) return QAT_ERR_ARG;
  if (!dim_ok(d) || !dim_ok(H)) return QAT_ERR_SHAPE;
  Carver ws(workspace, ws_bytes);
  const __nv_bfloat16 *op_fc = nullptr, *op_proj = nullptr;
  int rc = get_operand(Wfc, qfc, H, d, bits, ws, stream, &op_fc);
  if (rc) return rc;
  rc = get_operand(Wproj, qproj, d, H, bits, ws, stream, &op_proj);
  if (rc) return rc;
  if (T == 0) {
    if (!accumulate_dW) {
      if (dWfc && cudaMemsetAsync(dWfc, 0, static_cast<size_t>(H) * d * 4, stream) != cudaSuccess)
        return QAT_ERR_CUDA;
      if (dWproj && cudaMemsetAsync(dWproj, 0, static_cast<size_t>(d) * H * 4, stream) != cudaSuccess)
        return QAT_ERR_CUDA;
    }
    return QAT_OK;
  }
  if (dpre_save && !aligned16(dpre_save)) return QAT_ERR_ALIGN;
  void* dpre = dpre_save ? static_cast<void*>(dpre_save) : ws.take(static_cast<size_t>(T) * H * 2);
  if (!dpre) return QAT_ERR_WORKSPACE;
  if (dWproj) {  // dWproj[d,H] = dY^T . h
    GemmDesc g;
    g.A = dY; g.lda = d; g.a_mn = true;
    g.B = h; g.ldb = H; g.b_mn = true;
    g.M = d; g.N = H; g.K = T;
    g.epi = EPI_F32;
    g.D = dWproj; g.ldd = H;
    g.accumulate = accumulate_dW != 0;
    rc = launch_gemm(g, stream);
    if (rc) return rc;
  }
  {  // dpre[T,H] = (dY . Wproj_q) * act'(pre)
    GemmDesc g;
    g.A = dY; g.lda = d;
    g.B = op_proj; g.ldb = H; g.b_mn = true;
    g.M = T; g.N = H; g.K = d;
    g.epi = act == QAT_ACT_RELU2 ? EPI_DRELU2 : EPI_DLRELU2;
    g.D = dpre; g.ldd = H;
    g.R = pre; g.ldr = H;
    rc = launch_gemm(g, stream);
    if (rc) return rc;
  }
  if (dWfc) {  // dWfc[H,d] = dpre^T . X
    GemmDesc g;
    g.A = dpre; g.lda = H; g.a_mn = true;
    g.B = X; g.ldb = d; g.b_mn = true;
    g.M = H; g.N = d; g.K = T;
    g.epi = EPI_F32;
    g.D = dWfc; g.ldd = d;
    g.accumulate = accumulate_dW != 0;
    rc = launch_gemm(g, stream);
    if (rc) return rc;
  }
  if (dX) {  // dX[T,d] = dpre . Wfc_q (+ residual)
    GemmDesc g;
    g.A = dpre; g.lda = H;
    g.B = op_fc; g.ldb = d; g.b_mn = true;
    g.M = T; g.N = d; g.K = H;
    g.epi = dX_residual ? EPI_BF16_RESID : EPI_BF16;
    g.D = dX; g.ldd = d;
    g.R = dX_residual; g.ldr = d;
    rc = launch_gemm(g, stream);
    if (rc) return rc;
  }
  return QAT_OK;
}

int quantize_rows_export(const float* W, int64_t rows, int64_t cols, int32_t bits, int8_t* codes,
                         qat_fp16* scales, qat_stream_t stream) {
  qat_export_desc d;
  d.src = W;
  d.rows = rows;
  d.cols = cols;
  d.mode = bits;
  d.flags = 0;
  d.dst = codes;
  d.scales = scales;
  if (!bits_ok(bits)) return QAT_ERR_ARG;
  return quantize_export_batch(&d, 1, stream);
}

int quantize_export_batch(const qat_export_desc* descs, int32_t n, qat_stream_t stream) {
  if (!descs || n <= 0 || n > QAT_EXPORT_MAX_DESCS) return QAT_ERR_ARG;
  static thread_local ExportBatch b;  // ~20 KB: kept off the stack
  b.n = n;
  b.total_units = 0;
  for (int i = 0; i < n; ++i) {
    const qat_export_desc& s = descs[i];
    ExportDescDev& d = b.d[i];
    if (!s.src || !s.dst || s.rows < 0 || s.cols < 0) return QAT_ERR_ARG;
    if (!aligned16(s.src) || !aligned16(s.dst)) return QAT_ERR_ALIGN;
    d.src = s.src;
    d.dst = s.dst;
    d.scales = reinterpret_cast<__half*>(s.scales);
    d.mode = s.mode;
    d.m = 1;
    d.frac = 0.0f;
    if (s.flags & ~(QAT_EXPORT_PACK6 | QAT_EXPORT_CLIP_SEARCH)) return QAT_ERR_ARG;
    d.pack6 = (s.flags & QAT_EXPORT_PACK6) != 0;
    d.search = (s.flags & QAT_EXPORT_CLIP_SEARCH) != 0;
    d.pad = 0;
    if (d.pack6 && s.mode != 5 && s.mode != 6) return QAT_ERR_ARG;
    if (d.search && !bits_ok(s.mode)) return QAT_ERR_ARG;
    if (d.search && !clip_search_supported(s.cols)) return QAT_ERR_SHAPE;
    d.unit_begin = b.total_units;
    if (s.mode == QAT_EXPORT_FP16) {
      d.numel = s.rows * s.cols;
      d.cols = kFp16Chunk;
      d.rows = (d.numel + kFp16Chunk - 1) / kFp16Chunk;
      d.unit_rows = 1;
    } else if (bits_ok(s.mode)) {
      if (!s.scales) return QAT_ERR_ARG;
      if (!dim_ok(s.cols)) return QAT_ERR_SHAPE;
      d.rows = s.rows;
      d.cols = s.cols;
      d.numel = s.rows * s.cols;
      // staged rows travel in units of as many rows as fit kExportUnitBytes
      d.unit_rows = (s.cols <= kExportMaxStagedCols)
                        ? std::max<int64_t>(1, kExportUnitBytes / (s.cols * 4))
                        : 1;
      const int rc = export_quantile_params(s.cols, &d.m, &d.frac);
      if (rc) return rc;
    } else {
      return QAT_ERR_ARG;
    }
    b.total_units += (d.rows + d.unit_rows - 1) / d.unit_rows;
  }
  return launch_export_batch(b, stream);
}

int unpack_codes6(const uint8_t* packed, int64_t n, int32_t bits, int8_t* codes,
                  qat_stream_t stream) {
  if (!packed || !codes || n < 0 || (bits != 5 && bits != 6)) return QAT_ERR_ARG;
  if (n % 8 != 0) return QAT_ERR_SHAPE;
  if (!aligned16(packed) || !aligned16(codes)) return QAT_ERR_ALIGN;
  return launch_unpack6(packed, n, bits, codes, stream);
}

int dequantize_rows(const int8_t* codes, const qat_fp16* scales, int64_t rows, int64_t cols,
                    int32_t out_dtype, void* out, qat_stream_t stream) {
  if (!codes || !scales || !out || rows < 0) return QAT_ERR_ARG;
  if (out_dtype != QAT_DTYPE_F32 && out_dtype != QAT_DTYPE_BF16) return QAT_ERR_ARG;
  if (!dim_ok(cols)) return QAT_ERR_SHAPE;
  if (!aligned16(codes) || !aligned16(out)) return QAT_ERR_ALIGN;
  return launch_dequant(codes, reinterpret_cast<const __half*>(scales), rows, cols,
                        out_dtype == QAT_DTYPE_BF16, out, stream);
}

int dequantize_rows_batch(const qat_dequant_desc* descs, int32_t n, qat_stream_t stream) {
  if (!descs || n <= 0 || n > QAT_DEQUANT_MAX_DESCS) return QAT_ERR_ARG;
  static thread_local DequantBatch b;  // ~14 KB: kept off the stack
  b.n = n;
  b.tile_begin[0] = 0;
  for (int i = 0; i < n; ++i) {
    const qat_dequant_desc& s = descs[i];
    if (!s.codes || !s.scales || !s.out || s.rows < 0) return QAT_ERR_ARG;
    if (s.out_dtype != QAT_DTYPE_F32 && s.out_dtype != QAT_DTYPE_BF16) return QAT_ERR_ARG;
    if (!dim_ok(s.cols)) return QAT_ERR_SHAPE;
    if (!aligned16(s.codes) || !aligned16(s.out)) return QAT_ERR_ALIGN;
    DequantDescDev& d = b.d[i];
    d.codes = s.codes;
    d.scales = reinterpret_cast<const __half*>(s.scales);
    d.out = s.out;
    d.items = s.rows * (s.cols >> 2);
    d.row_magic = dequant_row_magic(s.cols >> 2);
    d.out_bf16 = s.out_dtype == QAT_DTYPE_BF16;
    d.pad = 0;
    b.tile_begin[i + 1] = b.tile_begin[i] + (d.items + kDequantTile - 1) / kDequantTile;
  }
  return launch_dequant_batch(b, stream);
}

}  // extern "C"
