// qsa_selftest_wait_timeout: exercises the bounded wait that every pipelined kernel of libqsa uses.
//
// No counterpart in the article.  One CTA initialises an mbarrier in shared memory and waits, with
// the library's wait helper and a caller-given limit, on a phase that nothing completes.  When the
// limit runs out the helper sets QSA_DEVERR_TIMEOUT in the error flag and the kernel returns: the
// failure is reported on the host through the flag and the CUDA context stays usable.  The wait
// always ends (the limit is bounded on the host), nothing faults and nothing is left in flight.
#include "../../include/qsa.h"
#include "common.cuh"

namespace qsa {
namespace {

__global__ void wait_timeout_kernel(int32_t* err, long long limit) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, err, limit);  // phase 0 never completes
}

}  // namespace
}  // namespace qsa

extern "C" qsa_status_t qsa_selftest_wait_timeout(int32_t* err_flag, int64_t limit_cycles,
                                                 qsa_stream_t stream) {
  if (!err_flag || limit_cycles < 1000 || limit_cycles > 1000000000) return QSA_ERR_INVALID_ARG;
  qsa::wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(err_flag, (long long)limit_cycles);
  return cudaGetLastError() == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
}
