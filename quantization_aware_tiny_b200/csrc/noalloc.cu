// qat_linear_fwd_noalloc: the QAT linear forward from fp32 weights for callers
// that cannot allocate device memory.
//
// Some callers cannot allocate device memory themselves: a plugin running
// inside a host framework that owns all device memory through its own pool,
// a real-time or fixed-budget service that allocates everything at start-up
// and nothing afterwards, or latency-critical code that cannot afford the
// device-wide synchronization cudaMalloc / cudaFree may cause.  They still
// need the one piece of scratch the raw-weight forward uses -- the bf16
// operand bf16(fl32(c*s)) and the per-row scales -- so this entry point keeps
// it in a fixed array compiled into the library instead of a workspace.
//
// The array lives in device memory of every GPU that loads the library, from
// load until process exit (8 MiB + 64 KiB each).  All calls share it: a call
// fully rewrites the part it uses before reading it (nothing has to start at
// zero), and calls whose kernels overlap on the GPU -- different streams, or
// different host threads, on the same device -- race on it.  Serialize them.
#include <mutex>

#include "gemm_sm100.cuh"
#include "quant.cuh"

namespace qat {
namespace {

constexpr size_t kOperandBytes = static_cast<size_t>(QAT_NOALLOC_MAX_ELEMS) * 2;
constexpr size_t kScaleBytes = static_cast<size_t>(QAT_NOALLOC_MAX_ROWS) * 4;

// The scratch itself.  In host code this name is only a stand-in for the
// symbol, never a device address: the address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kOperandBytes + kScaleBytes];

// Device address of the scratch on the current device, looked up on the
// first call made on each device (with that device current) and cached; that
// first call should therefore come before any stream capture.
int scratch_on_current_device(unsigned char** out) {
  static std::mutex mu;
  static unsigned char* cached[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return QAT_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!cached[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return QAT_ERR_CUDA;
    cached[dev] = static_cast<unsigned char*>(p);
  }
  *out = cached[dev];
  return QAT_OK;
}

}  // namespace
}  // namespace qat

extern "C" int qat_linear_fwd_noalloc(const float* W, int32_t N, int32_t K, int32_t bits,
                                      const qat_bf16* X, int64_t ldx, int64_t T,
                                      const qat_bf16* residual, qat_bf16* Y, qat_stream_t stream) {
  using namespace qat;
  if (!W || (T > 0 && (!X || !Y)) || T < 0 || (bits != 5 && bits != 6 && bits != 8)) return QAT_ERR_ARG;
  if (N <= 0 || K <= 0 || (N & 7) || (K & 7)) return QAT_ERR_SHAPE;
  if (static_cast<int64_t>(N) * K > QAT_NOALLOC_MAX_ELEMS || N > QAT_NOALLOC_MAX_ROWS)
    return QAT_ERR_SHAPE;
  if (ldx == 0) ldx = K;
  if (ldx < K || (ldx & 7)) return QAT_ERR_SHAPE;
  if (T == 0) return QAT_OK;  // as qat_linear_fwd: no tokens, nothing checked further
  if (!aligned16(W) || !aligned16(X) || !aligned16(Y) || (residual && !aligned16(residual)))
    return QAT_ERR_ALIGN;
  unsigned char* scratch = nullptr;
  int rc = scratch_on_current_device(&scratch);
  if (rc) return rc;
  __nv_bfloat16* operand = reinterpret_cast<__nv_bfloat16*>(scratch);
  float* scales = reinterpret_cast<float*>(scratch + kOperandBytes);
  rc = launch_quantize_weights(W, N, K, bits, nullptr, scales, operand, stream);
  if (rc) return rc;
  GemmDesc g;
  g.A = X;
  g.lda = ldx;
  g.B = operand;
  g.ldb = K;
  g.M = T;
  g.N = N;
  g.K = K;
  g.epi = residual ? EPI_BF16_RESID : EPI_BF16;
  g.D = Y;
  g.ldd = N;
  g.R = residual;
  g.ldr = N;
  return launch_gemm(g, stream);
}
