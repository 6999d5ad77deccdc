// Host interface of the tcgen05 GEMM used by every linear of the library.
#pragma once

#include "common.cuh"

namespace qat {

// Epilogue applied to the fp32 accumulator tile.
enum Epi : int {
  EPI_BF16 = 0,        // D = bf16(acc)
  EPI_BF16_RESID = 1,  // D = bf16(acc + R)
  EPI_RELU2 = 2,       // D = bf16(acc) (optional), D2 = bf16(relu(acc)^2)
  EPI_DRELU2 = 3,      // D = bf16(acc * 2*relu(R))     (R = saved pre-activation)
  EPI_F32 = 4,         // D = acc (+ D if accumulate), single writer per element
  EPI_F32_ATOMIC = 5,  // D += acc with atomics (split-K partial sums)
  EPI_LRELU2 = 6,      // D = bf16(acc) (optional), D2 = bf16(leaky_relu(acc, 0.5)^2)
  EPI_DLRELU2 = 7,     // D = bf16(acc * g(R)), g = 2R for R > 0 else R/2 (its derivative)
};

// Epilogues that read a bf16 tile R, and those that write the activation pair.
constexpr bool epi_reads_r(int e) {
  return e == EPI_BF16_RESID || e == EPI_DRELU2 || e == EPI_DLRELU2;
}
constexpr bool epi_act_fwd(int e) { return e == EPI_RELU2 || e == EPI_LRELU2; }

// D[M,N] = A[M,K] . B[N,K]^T with bf16 operands and fp32 accumulation.
// A is K-major (row m contiguous along K, row stride lda) unless a_mn, in which
// case it is stored [K][lda] with M contiguous (the transpose of a row-major
// [K,M] tensor).  Likewise B.  All strides are in elements.
struct GemmDesc {
  const void* A = nullptr;
  int64_t lda = 0;
  bool a_mn = false;
  const void* B = nullptr;
  int64_t ldb = 0;
  bool b_mn = false;
  int64_t M = 0, N = 0, K = 0;
  int epi = EPI_BF16;
  void* D = nullptr;
  int64_t ldd = 0;
  void* D2 = nullptr;
  int64_t ldd2 = 0;
  const void* R = nullptr;
  int64_t ldr = 0;
  bool accumulate = false;  // fp32 epilogues: add into D instead of overwriting
  // Fused quantizing B producer: when set, B / ldb are ignored and the kernel
  // builds the bf16 operand bf16(fl32(c * s)) of this fp32 weight [N,K]
  // (row-major, ld = K) on the grid `bits` in shared memory -- the quantized
  // weight never reaches global memory.  Forward epilogues, M >= 256 and
  // fused_b_supported() only.
  const float* Wraw = nullptr;
  int bits = 0;
};

// Whether launch_gemm can quantize B inside the GEMM for this shape / epilogue.
bool fused_b_supported(int64_t M, int64_t N, int64_t K, int epi);


// Validates, encodes the tensor maps and launches.  Returns a QAT_* code.
int launch_gemm(const GemmDesc& g, cudaStream_t stream);

}  // namespace qat
