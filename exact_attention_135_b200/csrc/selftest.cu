// Self-test of the bounded-wait failure path (no fault, no hang).
//
// One CTA waits on an mbarrier that nothing ever arrives on, with the same
// bounded wait the attention kernels use but a caller-chosen limit.  When
// the limit passes the wait gives up, records ATTN_ERR_TIMEOUT in the device
// status word and the kernel returns normally, so the context stays usable.
#include "host_common.h"
#include "sm100.cuh"

namespace ea {

__global__ void selftest_wait_kernel(int* status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar_storage;
  __shared__ int abort_flag_storage;
  const uint32_t bar = smem_addr(&bar_storage);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);   // one arrival expected; none will come
    abort_flag_storage = 0;
    fence_barrier_init();
  }
  __syncthreads();
  volatile int* abort_flag = &abort_flag_storage;
  if (threadIdx.x < 32) {
    const bool ok = mbar_wait(bar, 0, abort_flag, status, limit_ns);
    (void)ok;
  }
  __syncthreads();
}

}  // namespace ea

extern "C" int attn_selftest_wait_timeout(unsigned int limit_us, void* stream) {
  if (limit_us == 0 || limit_us > 10u * 1000u * 1000u) return ATTN_ERR_INVALID_ARG;
  int* status = ea::device_status_ptr();
  if (!status) return ATTN_ERR_CUDA;
  ea::selftest_wait_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(
      status, static_cast<unsigned long long>(limit_us) * 1000ull);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}
