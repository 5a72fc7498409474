// Per-row epilogue and report, run by one CTA once every row's statistics exist:
// confidence BCE against the detached acceptance label, dL/dc, the unnormalised
// loss numerator and the [numerator, denominator] report pairs.
//
// Megatron-Bridge API doc, bridge.training.post_training.dspark.loss: module
// docstring (three position-weighted terms; accept = 1 - 0.5*L1; tau = sum_k
// cumprod(accept)_k + 1), Return contract (nothing is divided), _acceptance_report.
// The clamp of accept to [0, 1] and the scrub of masked slots follow the merge note
// of Megatron-Bridge pull request #5241.  Sums are accumulated in FP64 by a fixed
// thread-to-row map and a fixed reduction tree, so repeated calls give bitwise the
// same report.
#pragma once
#include "internal.cuh"

namespace dspark {

constexpr int kNAcc = 7;  // loss, ce, l1, conf, accept, tau, keep

__device__ __forceinline__ double softplus_d(double x) { return fmax(x, 0.0) + log1p(exp(-fabs(x))); }

__device__ __forceinline__ double clamp01(double x) { return fmin(fmax(x, 0.0), 1.0); }

// Reduce kNAcc doubles over the CTA in a fixed order; thread 0 gets the totals.
// `scratch` holds (blockDim.x / 32) * kNAcc doubles of shared memory.
__device__ inline void block_reduce_acc(double* acc, double* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int i = 0; i < kNAcc; ++i) {
    double v = acc[i];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) scratch[warp * kNAcc + i] = v;
  }
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x / 32;
#pragma unroll
    for (int i = 0; i < kNAcc; ++i) {
      double v = lane < nw ? scratch[lane * kNAcc + i] : 0.0;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      acc[i] = v;
    }
  }
  __syncthreads();
}

__device__ inline void finalize_rows(const FinalizeArgs& a, double* scratch) {
  const int64_t R = a.B * a.N * a.K;
  const float* st = a.ws.stats;
  const double g = a.grad_scale ? double(*a.grad_scale) : 1.0;
  double acc[kNAcc] = {0, 0, 0, 0, 0, 0, 0};
  for (int64_t r = threadIdx.x; r < R; r += blockDim.x) {
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
      const float dc = a.has_conf ? float(g * w * double(a.conf_alpha) * (1.0 / (1.0 + exp(-c)) - y)) : 0.f;
      if (a.dconf) a.dconf[r] = dc;
      a.ws.stats[r * kStride + kStDC] = dc;
    } else {
      if (a.ce_rows) a.ce_rows[r] = 0.f;
      if (a.l1_rows) a.l1_rows[r] = 0.f;
      if (a.accept_rows) a.accept_rows[r] = 0.f;
      if (a.dconf) a.dconf[r] = 0.f;
      a.ws.stats[r * kStride + kStDC] = 0.f;
    }
    if (a.conf_rows) a.conf_rows[r] = float(c);
  }
  // tau per block: 1 + sum_k prod_{j<=k} m_j * accept_j
  for (int64_t blk = threadIdx.x; blk < a.B * a.N; blk += blockDim.x) {
    const double keep = (a.block_keep == nullptr || a.block_keep[blk] != 0) ? 1.0 : 0.0;
    double run = 1.0, tau = 1.0;
    for (int64_t k = 0; k < a.K; ++k) {
      const int64_t r = blk * a.K + k;
      const double ak = a.ws.m[r] ? clamp01(1.0 - 0.5 * double(st[r * kStride + kStL1])) : 0.0;
      run *= ak;
      tau += run;
    }
    acc[5] += keep * tau;
    acc[6] += keep;
  }
  block_reduce_acc(acc, scratch);
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

// The sweep's report: the same terms as finalize_rows, laid out for one CTA of blockDim.x
// threads with (kNAcc + 1) * blockDim.x + kNAcc doubles of shared memory at `sm`.
//  - The rows are taken a chunk of whole blocks at a time (blockDim.x / K blocks; K up to
//    blockDim.x): each row's acceptance goes to shared memory, and each block's tau is
//    formed from there, so no global load waits on another.
//  - The per-row transcendental terms (softplus, sigmoid) are taken in FP32, the precision
//    of their inputs (CE, L1 and c are FP32); every sum is FP64.
//  - The report is summed through shared memory: thread partials, then warp i adds the
//    partials of accumulator i in a fixed order.
__device__ __forceinline__ float softplus_f(float x) { return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))); }

__device__ inline void finalize_rows_smem(const FinalizeArgs& a, double* sm) {
  const int nt = blockDim.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t nblk = a.B * a.N;
  double* part = sm;               // [kNAcc][nt] thread partials
  double* yrow = sm + kNAcc * nt;  // [nt] acceptances of a chunk's rows
  double* tot = yrow + nt;         // [kNAcc] totals
  const float* st = a.ws.stats;
  const double g = a.grad_scale ? double(*a.grad_scale) : 1.0;
  double acc[kNAcc] = {0, 0, 0, 0, 0, 0, 0};
  const int64_t bpc = a.K <= nt ? nt / a.K : 0;  // whole blocks per chunk
  for (int64_t b0 = 0; b0 < nblk; b0 += bpc) {
    const int64_t nb = nblk - b0 < bpc ? nblk - b0 : bpc;
    const int64_t r = b0 * a.K + tid;
    // the block's keep flag, loaded here so that its latency hides behind the row terms
    const bool kept = tid >= nb || a.block_keep == nullptr || a.block_keep[b0 + tid] != 0;
    if (tid < nb * a.K) {
      // every load first (an unsupervised row's statistics are read and not used)
      const bool m = a.ws.m[r] != 0;
      const float cf = a.confidence_logits ? a.confidence_logits[r] : st[r * kStride + kStConf];
      const float ce_f = st[r * kStride + kStCE], l1_f = st[r * kStride + kStL1], w_f = a.ws.w[r];
      const float c = a.has_conf ? cf : 0.f;
      double y = 0.0;
      float dc = 0.f;
      if (m) {
        const double ce = ce_f, l1 = l1_f, w = w_f;
        y = clamp01(1.0 - 0.5 * l1);
        const double bce =
            a.has_conf ? y * double(softplus_f(-c)) + (1.0 - y) * double(softplus_f(c)) : 0.0;
        acc[0] += w * (double(a.ce_alpha) * ce + double(a.l1_alpha) * l1 +
                       (a.has_conf ? double(a.conf_alpha) * bce : 0.0));
        acc[1] += w * ce;
        acc[2] += w * l1;
        acc[3] += w * bce;
        acc[4] += y;
        if (a.has_conf) dc = float(g * w * double(a.conf_alpha) * (double(1.f / (1.f + expf(-c))) - y));
      }
      if (a.ce_rows) a.ce_rows[r] = m ? ce_f : 0.f;
      if (a.l1_rows) a.l1_rows[r] = m ? l1_f : 0.f;
      if (a.accept_rows) a.accept_rows[r] = float(y);
      if (a.dconf) a.dconf[r] = dc;
      a.ws.stats[r * kStride + kStDC] = dc;
      if (a.conf_rows) a.conf_rows[r] = c;
      yrow[tid] = y;
    }
    __syncthreads();
    if (tid < nb) {  // tau of block b0 + tid: 1 + sum_k prod_{j<=k} m_j * accept_j
      const double keep = kept ? 1.0 : 0.0;
      double run = 1.0, tau = 1.0;
      for (int64_t k = 0; k < a.K; ++k) {
        run *= yrow[tid * a.K + k];
        tau += run;
      }
      acc[5] += keep * tau;
      acc[6] += keep;
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < kNAcc; ++i) part[i * nt + tid] = acc[i];
  __syncthreads();
  if (warp < kNAcc) {
    double v = 0.0;
    for (int k = lane; k < nt; k += 32) v += part[warp * nt + k];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) tot[warp] = v;
  }
  __syncthreads();
  if (tid == 0) {
    const int64_t n = a.ws.hdr->num_tokens;
    if (a.loss_num) *a.loss_num = float(tot[0]);
    if (a.num_tokens) *a.num_tokens = n;
    if (a.report) {
      const float nf = float(n);
      a.report[2 * DSPARK_REP_LOSS] = float(tot[0]);
      a.report[2 * DSPARK_REP_LOSS + 1] = nf;
      a.report[2 * DSPARK_REP_CE] = float(tot[1]);
      a.report[2 * DSPARK_REP_CE + 1] = nf;
      a.report[2 * DSPARK_REP_L1] = float(tot[2]);
      a.report[2 * DSPARK_REP_L1 + 1] = nf;
      a.report[2 * DSPARK_REP_CONF] = float(tot[3]);
      a.report[2 * DSPARK_REP_CONF + 1] = nf;
      a.report[2 * DSPARK_REP_ACCEPT] = float(tot[4]);
      a.report[2 * DSPARK_REP_ACCEPT + 1] = nf;
      a.report[2 * DSPARK_REP_TAU] = float(tot[5]);
      a.report[2 * DSPARK_REP_TAU + 1] = float(tot[6]);
    }
  }
}

}  // namespace dspark
