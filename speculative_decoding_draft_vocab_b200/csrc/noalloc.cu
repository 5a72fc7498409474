// dspark_loss_fwd_noalloc: the fused forward (+ backward) of dspark_loss_fwd with its
// workspace in a fixed device array of this library instead of caller memory.
//
// Some callers cannot hand the library a workspace: an operator plugin running inside
// a host framework that owns all device memory and gives its operators no allocator,
// or a runtime that forbids cudaMalloc/cudaFree once it is serving, because those calls
// synchronise the device and fragment its memory.  For them this entry point needs no
// allocation at all: the scratch is a file-scope __device__ array that every GPU
// loading the library holds until the process exits.
#include <cuda.h>

#include <mutex>

#include "internal.cuh"

using namespace dspark;

namespace {

// Largest micro-batch (rows B*N*K) the fixed scratch serves.
constexpr int64_t kNoAllocMaxRows = DSPARK_NOALLOC_MAX_ROWS;
constexpr size_t kNoAllocBytes = ws_offsets(kNoAllocMaxRows).bytes;
static_assert(kNoAllocBytes == DSPARK_NOALLOC_BYTES, "the header states the scratch size");

__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocBytes];

// The array's device address, looked up once per (device, context): a context that was
// torn down (cudaDeviceReset) and created again maps the array at a new address, so the
// context handle is part of the key.
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of the scratch array in the current device's current context.
cudaError_t scratch_address(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  CtxGetCurrentFn get_ctx = ctx_get_current();
  if (get_ctx == nullptr) return cudaErrorDeviceUninitialized;
  std::lock_guard<std::mutex> lk(g_mu);
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  if (ctx == nullptr || g_scratch_ptr[dev] == nullptr || g_scratch_ctx[dev] != ctx) {
    // the lookup also brings up the device's primary context when none is current yet
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorDeviceUninitialized;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *ptr = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" dspark_status_t dspark_loss_fwd_noalloc(const dspark_problem_t* prob,
                                                   const dspark_params_t* params,
                                                   const dspark_fwd_out_t* out,
                                                   const dspark_grads_t* grads,
                                                   dspark_stream_t stream) {
  if (prob == nullptr) return DSPARK_ERR_INVALID_ARG;
  if (prob->B <= 0 || prob->N <= 0 || prob->K <= 0) return DSPARK_ERR_INVALID_ARG;
  if (prob->B * prob->N * prob->K > kNoAllocMaxRows) return DSPARK_ERR_WORKSPACE;
  // a problem whose workspace is larger than the array (the Markov head, the teacher
  // from hidden states, a confidence head on a few hundred rows or more) is refused by
  // dspark_loss_fwd's workspace check before anything is enqueued
  void* ws = nullptr;
  if (scratch_address(&ws) != cudaSuccess) return DSPARK_ERR_CUDA;
  // the prologue kernel clears the scratch header (status, counters) on every call
  return dspark_loss_fwd(prob, params, out, grads, ws, kNoAllocBytes, stream);
}
