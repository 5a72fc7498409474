// Mask prologue: the contiguous-prefix supervision mask, the per-position loss
// weights, the supervised-token count and the two ordered row lists the sweep
// walks (supervised rows, then rows whose dlogits are only zero-filled).
//
// m[b,n,k] = prod_{j<=k} eval[b,n,j] * keep[b,n]  (TorchSpec pull request #132,
// scope list: cumprod prefix mask; Megatron-Bridge API doc, DSparkForwardOutput)
// w[b,n,k] = m * exp(-k/gamma)                     (Megatron-Bridge API doc,
// _loss_weight_mask; k is the 0-based block position)
// Integer work is exact; one CTA does it all (R is a few thousand rows).  The kernel is
// latency-bound (the sweep waits for it), so each row's inputs are loaded once and its
// mask, target record and weight stay in registers through the compaction (rows beyond
// kRegRows per thread, R > 8192, are re-read from the workspace instead).
#include "internal.cuh"

namespace dspark {

constexpr int kPrologueThreads = 1024;
constexpr int kRegRows = 8;  // rows per thread held in registers: R <= 8192

namespace {

struct RowRec {
  bool m;
  int32_t tok;  // target id; bit 31: an invalid Markov slot whose corrected row is all zero
  float w;
};

// Mask, weight and id checks of row r (its loads issued together).
__device__ __forceinline__ RowRec row_record(const PrologueArgs& a, int64_t r, uint32_t& flags) {
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
  RowRec rec;
  rec.m = mm;
  rec.w = !mm ? 0.f : (a.gamma_enabled ? expf(-float(k) / a.gamma) : 1.f);
  int32_t tk = int32_t(t);
  if (a.invalid_zero && a.valid != nullptr && !vld) tk |= int32_t(0x80000000u);
  rec.tok = tk;
  a.ws.m[r] = mm ? 1 : 0;
  a.ws.w[r] = rec.w;
  return rec;
}

}  // namespace

__global__ void __launch_bounds__(kPrologueThreads) prologue_kernel(const PrologueArgs a) {
  // the sweep may be scheduled now; it waits for this grid before reading anything
  asm volatile("griddepcontrol.launch_dependents;");
  const int tid = threadIdx.x;
  const int64_t R = a.B * a.N * a.K;
  WsHeader* hdr = a.ws.hdr;
  if (tid == 0) {
    hdr->status = 0;
    hdr->done = 0;
  }

  // ---- masks and weights, one thread per row
  uint32_t flags = 0;
  RowRec reg[kRegRows];
#pragma unroll
  for (int i = 0; i < kRegRows; ++i) {
    const int64_t r = tid + int64_t(i) * kPrologueThreads;
    reg[i] = RowRec{false, 0, 0.f};
    if (r < R) reg[i] = row_record(a, r, flags);
  }
  for (int64_t r = tid + int64_t(kRegRows) * kPrologueThreads; r < R; r += kPrologueThreads)
    row_record(a, r, flags);
  __syncthreads();  // status cleared before any flag is raised; masks of every row written
  if (flags) atomicOr(&hdr->status, flags);

  // ---- ordered compaction of the two row lists, with the supervised rows' target id
  // record and weight
  __shared__ int warp_sup[kPrologueThreads / 32];
  __shared__ int base_sup;
  const int lane = tid & 31, warp = tid >> 5;
  if (tid == 0) base_sup = 0;
  __syncthreads();
  auto chunk = [&](int64_t r, bool s, int32_t tok, float w) {
    const unsigned bal = __ballot_sync(0xffffffffu, s);
    if (lane == 0) warp_sup[warp] = __popc(bal);
    __syncthreads();
    int before = base_sup;
    for (int x = 0; x < warp; ++x) before += warp_sup[x];
    before += __popc(bal & ((1u << lane) - 1u));
    if (r < R) {
      if (s) {
        a.ws.sup_list[before] = int32_t(r);
        a.ws.sup_tok[before] = tok;
        a.ws.sup_w[before] = w;
      } else {
        a.ws.zero_list[r - before] = int32_t(r);
      }
      a.ws.sup_index[r] = s ? int32_t(before) : -1;
    }
    __syncthreads();
    if (tid == 0) {
      int tot = 0;
      for (int x = 0; x < kPrologueThreads / 32; ++x) tot += warp_sup[x];
      base_sup += tot;
    }
    __syncthreads();
  };
#pragma unroll
  for (int i = 0; i < kRegRows; ++i) {
    const int64_t r0 = int64_t(i) * kPrologueThreads;
    if (r0 >= R) break;  // the same in every thread
    const int64_t r = r0 + tid;
    chunk(r, r < R && reg[i].m, reg[i].tok, reg[i].w);
  }
  for (int64_t r0 = int64_t(kRegRows) * kPrologueThreads; r0 < R; r0 += kPrologueThreads) {
    const int64_t r = r0 + tid;
    const bool s = r < R && a.ws.m[r] != 0;
    int32_t tok = 0;
    float w = 0.f;
    if (s) {
      tok = int32_t(a.target_ids[r]);
      if (a.invalid_zero && a.valid != nullptr && a.valid[r] == 0) tok |= int32_t(0x80000000u);
      w = a.ws.w[r];
    }
    chunk(r, s, tok, w);
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
