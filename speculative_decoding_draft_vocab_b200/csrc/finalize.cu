// Per-row epilogue and report: confidence BCE against the detached acceptance
// label, dL/dc, the unnormalised loss numerator and the [numerator, denominator]
// report pairs, plus the standalone acceptance report.
//
// Megatron-Bridge API doc, bridge.training.post_training.dspark.loss:
//   module docstring (three position-weighted terms; accept = 1 - 0.5*L1;
//   tau = sum_k cumprod(accept)_k + 1), Return contract (nothing is divided),
//   _acceptance_report.  The clamp of accept to [0, 1] and the scrub of masked
//   slots follow the merge note of Megatron-Bridge pull request #5241.
// Sums are accumulated in FP64 by a fixed thread-to-row map and a fixed reduction
// tree, so repeated calls give bitwise the same report.
#include "internal.cuh"

namespace dspark {

constexpr int kFinThreads = 1024;
constexpr int kNAcc = 7;  // loss, ce, l1, conf, accept, tau, keep

__device__ __forceinline__ double softplus_d(double x) {
  return fmax(x, 0.0) + log1p(exp(-fabs(x)));
}

__device__ __forceinline__ double clamp01(double x) { return fmin(fmax(x, 0.0), 1.0); }

// Reduce kNAcc doubles over the CTA in a fixed order; thread 0 gets the totals.
__device__ void block_reduce_acc(double* acc) {
  __shared__ double part[kFinThreads / 32][kNAcc];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int i = 0; i < kNAcc; ++i) {
    double v = acc[i];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) part[warp][i] = v;
  }
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x / 32;
#pragma unroll
    for (int i = 0; i < kNAcc; ++i) {
      double v = lane < nw ? part[lane][i] : 0.0;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      acc[i] = v;
    }
  }
}

__global__ void __launch_bounds__(kFinThreads) finalize_kernel(const FinalizeArgs a) {
  const int64_t R = a.B * a.N * a.K;
  const float* st = a.ws.stats;
  const double g = a.grad_scale ? double(*a.grad_scale) : 1.0;
  double acc[kNAcc] = {0, 0, 0, 0, 0, 0, 0};
  for (int64_t r = threadIdx.x; r < R; r += kFinThreads) {
    const bool m = a.ws.m[r] != 0;
    const float cgiven = a.confidence_logits ? a.confidence_logits[r] : st[r * kStride + kStConf];
    const double c = a.has_conf ? double(cgiven) : 0.0;
    if (m) {
      const double ce = st[r * kStride + kStCE];
      const double l1 = st[r * kStride + kStL1];
      const double w = a.ws.w[r];
      const double y = clamp01(1.0 - 0.5 * l1);
      const double bce = a.has_conf ? y * softplus_d(-c) + (1.0 - y) * softplus_d(c) : 0.0;
      acc[0] += w * (double(a.ce_alpha) * ce + double(a.l1_alpha) * l1 +
                     (a.has_conf ? double(a.conf_alpha) * bce : 0.0));
      acc[1] += w * ce;
      acc[2] += w * l1;
      acc[3] += w * bce;
      acc[4] += y;
      if (a.ce_rows) a.ce_rows[r] = float(ce);
      if (a.l1_rows) a.l1_rows[r] = float(l1);
      if (a.accept_rows) a.accept_rows[r] = float(y);
      if (a.dconf) a.dconf[r] = a.has_conf ? float(g * w * double(a.conf_alpha) * (1.0 / (1.0 + exp(-c)) - y)) : 0.f;
    } else {
      if (a.ce_rows) a.ce_rows[r] = 0.f;
      if (a.l1_rows) a.l1_rows[r] = 0.f;
      if (a.accept_rows) a.accept_rows[r] = 0.f;
      if (a.dconf) a.dconf[r] = 0.f;
    }
    if (a.conf_rows) a.conf_rows[r] = float(c);
  }
  // the tau loop reads L1 through the stats of supervised rows only
  for (int64_t blk = threadIdx.x; blk < a.B * a.N; blk += kFinThreads) {
    const double keep = (a.block_keep == nullptr || a.block_keep[blk] != 0) ? 1.0 : 0.0;
    double run = 1.0, tau = 1.0;
    for (int64_t k = 0; k < a.K; ++k) {
      const int64_t r = blk * a.K + k;
      const double acc_k = a.ws.m[r] ? clamp01(1.0 - 0.5 * double(st[r * kStride + kStL1])) : 0.0;
      run *= acc_k;
      tau += run;
    }
    acc[5] += keep * tau;
    acc[6] += keep;
  }
  block_reduce_acc(acc);
  if (threadIdx.x == 0) {
    const int64_t n = a.ws.hdr->num_tokens;
    if (a.loss_num) *a.loss_num = float(acc[0]);
    if (a.num_tokens) *a.num_tokens = n;
    if (a.report) {
      const float nf = float(n);
      a.report[2 * DSPARK_REP_LOSS] = float(acc[0]);
      a.report[2 * DSPARK_REP_LOSS + 1] = nf;
      a.report[2 * DSPARK_REP_CE] = float(acc[1]);
      a.report[2 * DSPARK_REP_CE + 1] = nf;
      a.report[2 * DSPARK_REP_L1] = float(acc[2]);
      a.report[2 * DSPARK_REP_L1 + 1] = nf;
      a.report[2 * DSPARK_REP_CONF] = float(acc[3]);
      a.report[2 * DSPARK_REP_CONF + 1] = nf;
      a.report[2 * DSPARK_REP_ACCEPT] = float(acc[4]);
      a.report[2 * DSPARK_REP_ACCEPT + 1] = nf;
      a.report[2 * DSPARK_REP_TAU] = float(acc[5]);
      a.report[2 * DSPARK_REP_TAU + 1] = float(acc[6]);
    }
  }
}

cudaError_t launch_finalize(const FinalizeArgs& a, cudaStream_t s) {
  finalize_kernel<<<1, kFinThreads, 0, s>>>(a);
  return cudaGetLastError();
}

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
  block_reduce_acc(acc);
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
    if (ws.m[r] == 0) {
      dconf[r] = 0.f;
      continue;
    }
    const float* st = ws.stats + r * kStride;
    const double c = confidence_logits ? confidence_logits[r] : st[kStConf];
    const double y = clamp01(1.0 - 0.5 * double(st[kStL1]));
    dconf[r] = float(g * double(ws.w[r]) * double(conf_alpha) * (1.0 / (1.0 + exp(-c)) - y));
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
