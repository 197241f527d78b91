// Self-test of the kernels' bounded waits.
//
// Every mbarrier wait in the library's kernels gives up after
// OOMB_WAIT_LIMIT_CYCLES of polling, records OOMB_DEV_WAIT_LIMIT in the pool's
// device status word and unwinds, so a lost arrival can never hang the GPU.
// This entry point runs that path on purpose: one thread waits on an mbarrier
// that nothing arrives at, gives up after the limit (about a second) and
// records the bit; the context stays usable.
#include "internal.h"
#include "ptx.cuh"

namespace {

__global__ void wait_limit_probe(uint32_t* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    oomb::mbar_init(&bar, 1);
    oomb::fence_mbar_init();
    if (!oomb::mbar_wait(&bar, 0, &abort_flag)) atomicOr(status, OOMB_DEV_WAIT_LIMIT);
  }
}

}  // namespace

extern "C" oomb_status oomb_selftest_wait_limit(oomb_pool* pool, void* stream) {
  if (!pool || pool->desc.location == OOMB_LOC_HOST || !pool->d_status)
    return OOMB_ERR_INVALID_ARG;
  oomb::DeviceGuard guard(pool->desc.device);
  wait_limit_probe<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(pool->d_status);
  return oomb::check_launch();
}
