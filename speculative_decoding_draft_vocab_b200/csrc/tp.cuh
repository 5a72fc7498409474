// Vocabulary-parallel steps: kernel arguments and launchers (csrc/tp.cu).
#pragma once
#include "internal.cuh"

namespace dspark {

// One rank's shard of a micro-batch and the exchange records of the three steps.
struct TpArgs {
  const void* draft;         // shard columns of the base draft rows
  int64_t ld_d;
  const void* target;        // shard columns of the teacher rows, or null (CE only)
  int64_t ld_t;
  void* dlogits;             // shard columns of dL/dz, or null (forward only)
  int64_t ld_g;
  const int64_t* tids;       // global target ids
  const float* grad_scale;   // null: 1
  int64_t R;
  int64_t V;                 // shard width
  int64_t vocab_begin;       // global id of the shard's first column
  int32_t tp_size;
  float* rec1;               // [R][8] this shard's logsumexp partials
  const float* rec1_all;     // [tp_size][R][8] every rank's, rank order
  float* rec2;               // [R][4] this shard's (L1, S) partials
  const float* rec2_all;     // [tp_size][R][4]
  const float* bias;         // Markov bias rows of the shard (compact by supervised position), or null
  int32_t t_compact;         // teacher rows: FP32, compact by supervised position, ld_t columns
                             // (the teacher computed from hidden states on the shard)
  // Step 1 straight behind the mask prologue (no heads): it takes every row and decides
  // by the prologue's own rule whether the row is supervised, so it need not wait for
  // the prologue's lists
  int32_t own_rows;
  const uint8_t* eval_mask;
  const uint8_t* block_keep;
  int64_t K;
  int64_t vocab_size;        // global vocabulary (the target ids' range)
  float ce_alpha, l1_alpha;
  WsView ws;
  FinalizeArgs fin;          // the per-row epilogue and report the last CTA of step 3 runs
};

constexpr int kTpRec1 = 8;
constexpr int kTpRec2 = 4;

cudaError_t launch_tp_partials(bool f32, const TpArgs& a, cudaStream_t s);
cudaError_t launch_tp_l1(bool f32, const TpArgs& a, cudaStream_t s);
// the rows' L1 and S, dlogits of the shard, then (last CTA) the per-row epilogue and the report
cudaError_t launch_tp_finish(bool f32, const TpArgs& a, cudaStream_t s);

// Markov head on a vocabulary shard (csrc/heads.cu): the dE GEMM against this shard's
// W2 rows, its K splits summed into de_part [R][rank], and dW2 for this shard's rows
cudaError_t launch_markov_bwd_shard(const HeadsArgs& a, float* de_part, cudaStream_t s);
// dE from the ranks' parts de_all [nranks][R][rank] (+ dc proj_e), dW1, and the
// confidence head's gradients
cudaError_t launch_heads_bwd_merge(const HeadsArgs& a, const float* de_all, int nranks, cudaStream_t s);

}  // namespace dspark
