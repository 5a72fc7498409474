// Test harness for the device-timeout path (compiled by tests/test_timeout_gpu.py with a
// wait limit of a few milliseconds).  One CTA waits, through the library's bounded wait,
// on an mbarrier that nothing ever arrives on: the wait must give up, the kernel must
// record the timeout in the workspace header exactly as the library's kernels do, and
// return.  Nothing is in flight toward the waiting CTA, nothing traps or faults.
#include <cstdint>

#include "internal.cuh"
#include "ptx.cuh"

using namespace dspark;

// waited: 1 when the wait gave up, 2 when it (wrongly) completed; ns: how long it waited
__global__ void never_armed_wait_kernel(WsHeader* hdr, uint32_t* waited, uint64_t* ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = global_timer_ns();
    const bool ok = mbar_wait_bounded(smem_u32(&bar), 0);
    *ns = global_timer_ns() - t0;
    if (!ok) atomicOr(&hdr->status, kFlagTimeout);
    *waited = ok ? 2u : 1u;
  }
}

extern "C" int timeout_harness_run(void* ws, uint32_t* waited, uint64_t* ns, cudaStream_t s) {
  never_armed_wait_kernel<<<1, 32, 0, s>>>(static_cast<WsHeader*>(ws), waited, ns);
  return int(cudaGetLastError());
}

extern "C" uint64_t timeout_harness_limit_ns() { return kWaitLimitNs; }
