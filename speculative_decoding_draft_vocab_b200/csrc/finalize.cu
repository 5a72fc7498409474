// Standalone acceptance report and dL/dc after a separate forward.  The fused
// per-row epilogue and report live in finalize.cuh (run at the end of the sweep).
//
// Megatron-Bridge API doc, bridge.training.post_training.dspark.loss,
// _acceptance_report: accept = 1 - 0.5*L1 per supervised position and
// tau = 1 + sum_k prod_{j<=k} accept_j per block, reported as [numerator,
// denominator] pairs that are never divided here.
#include "finalize.cuh"

namespace dspark {

constexpr int kFinThreads = 1024;

// -------------------------------------------------------- standalone acceptance
__global__ void __launch_bounds__(kFinThreads)
acceptance_kernel(int64_t B, int64_t N, int64_t K, const float* l1_rows, const uint8_t* eval_mask,
                  const uint8_t* block_keep, float* accept_pair, float* tau_pair,
                  float* accept_rows) {
  double acc[kNAcc] = {0, 0, 0, 0, 0, 0, 0};
  const int64_t nblk = B * N;
  for (int64_t blk = threadIdx.x; blk < nblk; blk += kFinThreads) {
    const bool kept = block_keep == nullptr || block_keep[blk] != 0;
    bool run_m = kept;
    double run = 1.0, tau = 1.0;
    for (int64_t k = 0; k < K; ++k) {
      const int64_t r = blk * K + k;
      run_m = run_m && eval_mask[r] != 0;
      const double a = run_m ? clamp01(1.0 - 0.5 * double(l1_rows[r])) : 0.0;
      if (accept_rows) accept_rows[r] = float(a);
      acc[4] += a;
      acc[3] += run_m ? 1.0 : 0.0;
      run *= a;
      tau += run;
    }
    acc[5] += kept ? tau : 0.0;
    acc[6] += kept ? 1.0 : 0.0;
  }
  __shared__ double scratch[(kFinThreads / 32) * kNAcc];
  block_reduce_acc(acc, scratch);
  if (threadIdx.x == 0) {
    accept_pair[0] = float(acc[4]);
    accept_pair[1] = float(acc[3]);
    tau_pair[0] = float(acc[5]);
    tau_pair[1] = float(acc[6]);
  }
}

cudaError_t launch_acceptance(int64_t B, int64_t N, int64_t K, const float* l1_rows,
                              const uint8_t* eval_mask, const uint8_t* block_keep,
                              float* accept_pair, float* tau_pair, float* accept_rows,
                              cudaStream_t s) {
  acceptance_kernel<<<1, kFinThreads, 0, s>>>(B, N, K, l1_rows, eval_mask, block_keep,
                                              accept_pair, tau_pair, accept_rows);
  return cudaGetLastError();
}

// ---------------------------------------------------------- dL/dc after a forward
__global__ void conf_grad_kernel(int64_t R, const float* confidence_logits, float conf_alpha,
                                 const float* grad_scale, WsView ws, float* dconf) {
  const double g = grad_scale ? double(*grad_scale) : 1.0;
  for (int64_t r = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; r < R;
       r += int64_t(gridDim.x) * blockDim.x) {
    float dc = 0.f;
    if (ws.m[r] != 0) {
      const float* st = ws.stats + r * kStride;
      const double c = confidence_logits ? confidence_logits[r] : st[kStConf];
      const double y = clamp01(1.0 - 0.5 * double(st[kStL1]));
      dc = float(g * double(ws.w[r]) * double(conf_alpha) * (1.0 / (1.0 + exp(-c)) - y));
    }
    ws.stats[r * kStride + kStDC] = dc;  // the confidence head's backward reads it
    if (dconf) dconf[r] = dc;
  }
}

cudaError_t launch_conf_grad(int64_t R, const float* confidence_logits, float conf_alpha,
                             const float* grad_scale, const WsView& ws, float* dconf,
                             cudaStream_t s) {
  const int blocks = int((R + 255) / 256);
  conf_grad_kernel<<<blocks > 0 ? blocks : 1, 256, 0, s>>>(R, confidence_logits, conf_alpha,
                                                           grad_scale, ws, dconf);
  return cudaGetLastError();
}

}  // namespace dspark
