// lq_selftest.cu -- lq_check_wait_timeout: exercises the bounded mbarrier wait of the kernels
// on a barrier that never completes, so that the timeout path (status word, clean exit) can be
// tested without faulting or hanging the GPU.
#include "lq_internal.cuh"
#include "lq_sm100.cuh"

namespace lq {
namespace {

using namespace lq::sm100;

__global__ void wait_timeout_probe(uint32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);   // one arrival expected; none will come
    mbar_fence_init();
  }
  __syncwarp();
  uint64_t t0;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t0));
  for (;;) {
    if (mbar_try_wait(&bar, 0)) return;   // cannot happen: the phase never completes
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    if (t - t0 > limit_ns) break;
  }
  if (threadIdx.x == 0) atomicCAS(status, 0u, (uint32_t)LQ_ETIMEOUT);
}

}  // namespace
}  // namespace lq

extern "C" lq_status lq_check_wait_timeout(void* workspace, int32_t limit_ms, lq_stream stream) {
  lq::set_last_error("%s", "");
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256 != 0) {
    lq::set_last_error("lq_check_wait_timeout: workspace is null or not 256-byte aligned");
    return LQ_EINVAL;
  }
  if (limit_ms < 1 || limit_ms > 1000) {
    lq::set_last_error("lq_check_wait_timeout: limit_ms = %d outside 1..1000", limit_ms);
    return LQ_EINVAL;
  }
  lq::wait_timeout_probe<<<1, 32, 0, (cudaStream_t)stream>>>(static_cast<uint32_t*>(workspace),
                                                              (uint64_t)limit_ms * 1000000ull);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    lq::set_last_error("lq_check_wait_timeout: %s", cudaGetErrorString(e));
    return LQ_ECUDA;
  }
  return LQ_OK;
}
