// qat_selftest_wait_timeout: a diagnostic of the library's failure reporting.
//
// Every wait inside the library's kernels is bounded: after its limit it
// records QAT_ERR_TIMEOUT in the device error flag, and the kernel returns
// instead of hanging, so the CUDA context stays usable and the host learns of
// the failure from qat_device_error().  This entry point runs exactly that
// path on purpose, with a short limit: one thread waits on an mbarrier that
// nothing ever arrives on, through the same bounded wait the GEMMs use, gives
// up after limit_ns and records the timeout.  No fault, trap or unbounded loop
// is involved.
#include "common.cuh"
#include "sm100_ptx.cuh"

namespace qat {
namespace {

__global__ void wait_timeout_kernel(unsigned long long limit_ns, int* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // phase 0 of a fresh barrier with no arrivals never completes
  if (threadIdx.x == 0) mbar_wait_for(&bar, 0, &abort_flag, err, limit_ns);
}

}  // namespace
}  // namespace qat

using namespace qat;

extern "C" int qat_selftest_wait_timeout(int64_t limit_ns, qat_stream_t stream) {
  if (limit_ns < 1000 || limit_ns > 10000000000ll) return QAT_ERR_ARG;
  int* err = device_error_ptr();
  if (!err) return QAT_ERR_CUDA;
  wait_timeout_kernel<<<1, 32, 0, stream>>>(static_cast<unsigned long long>(limit_ns), err);
  count_launch();
  return cuda_status(cudaGetLastError());
}
