// Self-test of the bounded device waits that every pipelined kernel here uses:
// one CTA waits on an mbarrier that nothing ever arrives on, gives up after the
// requested limit, records QSA_ERR_TIMEOUT in the workspace status word and
// returns -- the same path a real kernel takes when a copy or a peer stalls. No
// trap, no fault, no hang: the context stays usable.
#include "qsa_internal.h"
#include "sm100_ptx.cuh"

namespace qsa {
namespace {

__global__ void k_wait_timeout(int *status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    sm100::fence_mbar_init();
  }
  __syncthreads();
  // phase 0 never completes: no thread arrives and no copy is pending
  const bool done = sm100::mbar_wait(&bar, 0, limit_ns);
  if (!done && threadIdx.x == 0) record_status(status, QSA_ERR_TIMEOUT);
}

}  // namespace
}  // namespace qsa

extern "C" qsa_status_t qsa_selftest_wait_timeout(void *workspace, int64_t limit_ns, qsa_stream_t stream) {
  if (!workspace || limit_ns < 1000000 || limit_ns > 5000000000LL) return QSA_ERR_INVALID_ARG;
  qsa::note_launch();
  qsa::k_wait_timeout<<<1, 32, 0, (cudaStream_t)stream>>>((int *)workspace, (unsigned long long)limit_ns);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    qsa::note_error("qsa_selftest_wait_timeout launch", e);
    return QSA_ERR_CUDA;
  }
  return QSA_OK;
}
