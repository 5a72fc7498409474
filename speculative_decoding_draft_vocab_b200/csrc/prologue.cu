// Mask prologue: the contiguous-prefix supervision mask, the per-position loss
// weights, the supervised-token count and the two ordered row lists the sweep
// walks (supervised rows, then rows whose dlogits are only zero-filled).
//
// m[b,n,k] = prod_{j<=k} eval[b,n,j] * keep[b,n]  (TorchSpec pull request #132,
// scope list: cumprod prefix mask; Megatron-Bridge API doc, DSparkForwardOutput)
// w[b,n,k] = m * exp(-k/gamma)                     (Megatron-Bridge API doc,
// _loss_weight_mask; k is the 0-based block position)
// Integer work is exact; one CTA does it all (R is a few thousand rows).
#include "internal.cuh"

namespace dspark {

constexpr int kPrologueThreads = 1024;
constexpr int kRowsPerThread = 8;     // R <= 8192 keeps every row's mask in registers

__global__ void __launch_bounds__(kPrologueThreads) prologue_kernel(const PrologueArgs a) {
  // the sweep may be scheduled now; it waits for this grid before reading anything
  asm volatile("griddepcontrol.launch_dependents;");
  const int tid = threadIdx.x;
  const int64_t nblk = a.B * a.N;
  const int64_t R = nblk * a.K;
  WsHeader* hdr = a.ws.hdr;
  if (tid == 0) {
    hdr->status = 0;
    hdr->done = 0;
  }

  // ---- masks and weights, one thread per row (the prefix is re-scanned per row); every
  // load of a row is issued before any is used
  uint32_t flags = 0;
  uint32_t mbits = 0;  // mask of this thread's rows tid, tid + 1024, ... (R <= 8192)
  for (int64_t r = tid, i = 0; r < R; r += kPrologueThreads, ++i) {
    const int64_t blk = r / a.K, k = r - blk * a.K;
    const int64_t t = a.target_ids[r];
    const bool vld = a.valid != nullptr && a.valid[r] != 0;
    const int64_t pv = (a.prev_ids != nullptr) ? a.prev_ids[r] : 0;
    bool run = a.block_keep == nullptr || a.block_keep[blk] != 0;
    for (int64_t j = 0; j <= k; ++j) run &= a.eval_mask[blk * a.K + j] != 0;
    bool mm = run;
    if (mm) {
      if (t < 0 || t >= a.V) { flags |= kFlagIdOutOfRange; mm = false; }
      if (a.prev_ids != nullptr && vld && (pv < 0 || pv >= a.Vt)) { flags |= kFlagIdOutOfRange; mm = false; }
    }
    a.ws.m[r] = mm ? 1 : 0;
    a.ws.w[r] = !mm ? 0.f : (a.gamma_enabled ? expf(-float(k) / a.gamma) : 1.f);
    if (i < 32) mbits |= uint32_t(mm) << i;
  }
  __syncthreads();  // status cleared before any flag is raised
  if (flags) atomicOr(&hdr->status, flags);

  // ---- ordered compaction of the two row lists, with the supervised rows' target id
  // (bit 31: an invalid Markov slot whose corrected row is all zero) and weight
  __shared__ int warp_sup[kPrologueThreads / 32];
  __shared__ int base_sup;
  const int lane = tid & 31, warp = tid >> 5;
  if (tid == 0) base_sup = 0;
  __syncthreads();
  for (int64_t r0 = 0, i = 0; r0 < R; r0 += kPrologueThreads, ++i) {
    const int64_t r = r0 + tid;
    const bool s = r < R && (i < 32 ? ((mbits >> i) & 1u) != 0 : a.ws.m[r] != 0);
    const unsigned bal = __ballot_sync(0xffffffffu, s);
    if (lane == 0) warp_sup[warp] = __popc(bal);
    __syncthreads();
    int before = base_sup;
    for (int w = 0; w < warp; ++w) before += warp_sup[w];
    before += __popc(bal & ((1u << lane) - 1u));
    if (r < R) {
      if (s) {
        a.ws.sup_list[before] = int32_t(r);
        int32_t tk = int32_t(a.target_ids[r]);
        if (a.invalid_zero && a.valid != nullptr && a.valid[r] == 0) tk |= int32_t(0x80000000u);
        a.ws.sup_tok[before] = tk;
        a.ws.sup_w[before] = a.ws.w[r];
      } else {
        a.ws.zero_list[r - before] = int32_t(r);
      }
      a.ws.sup_index[r] = s ? int32_t(before) : -1;
    }
    __syncthreads();
    if (tid == 0) {
      int tot = 0;
      for (int w = 0; w < kPrologueThreads / 32; ++w) tot += warp_sup[w];
      base_sup += tot;
    }
    __syncthreads();
  }
  if (tid == 0) {
    hdr->n_sup = base_sup;
    hdr->n_zero = int32_t(R - base_sup);
    hdr->num_tokens = base_sup;
  }
}

cudaError_t launch_prologue(const PrologueArgs& a, cudaStream_t s) {
  prologue_kernel<<<1, kPrologueThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace dspark
