/*
 * dspark.h: C ABI of the fused DSpark draft-training loss for NVIDIA B200 (sm_100a).
 *
 * What it computes.  For draft logits laid out [B, N, K, V] (batch, sampled anchor
 * blocks, block positions, vocabulary) and the frozen target's next-token
 * distribution, the three position-weighted terms of the DSpark objective
 * (Megatron-Bridge API doc, bridge.training.post_training.dspark.loss, module
 * docstring and dspark_loss):
 *   loss = sum_r w_r * (ce_alpha*CE_r + l1_alpha*L1_r + conf_alpha*BCE_r)
 *   CE_r  = logsumexp(z_r) - z_r[target_id]
 *   L1_r  = sum_j |softmax(z_r)_j - softmax(t_r)_j|    (raw L1, no 1/2)
 *   BCE_r = binary cross-entropy of the confidence logit c_r against the detached
 *           label clamp(1 - 0.5*L1_r, 0, 1)
 *   w_r   = m_r * exp(-k/gamma), m = cumulative product of eval_mask along the block
 *           (TorchSpec pull request #132, scope list) times block_keep
 * plus the acceptance report (accept = 1 - 0.5*L1, tau = 1 + sum_k prod_{j<=k}
 * accept_j per block; Megatron-Bridge API doc, _acceptance_report), the gradient of
 * grad_scale*loss with respect to the base draft logits, and, when the optional heads
 * are given, the low-rank Markov correction z = base + markov_w2 . markov_w1[prev_id]
 * (zero row on invalid slots) and the linear confidence head c = proj . [h ; e] + b
 * (NeMo RL design doc "DSpark Auxiliary Heads", Inputs and Outputs, Checkpoint
 * Contract) with their weight gradients.
 *
 * Return contract (Megatron-Bridge API doc, module docstring, Return contract): the
 * library returns the UNNORMALISED weighted numerator, the supervised-token count and
 * [numerator, denominator] report pairs.  It never divides by a local denominator;
 * the caller sums numerators and denominators over micro-batches and data-parallel
 * ranks and divides once (that is the calculate_per_token_loss=True convention).
 *
 * Conventions for every entry point:
 *  - Pointers are DEVICE pointers unless stated otherwise.  The caller owns every
 *    buffer; the library allocates nothing and keeps no state between calls except
 *    what it writes into the caller's workspace.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream) and
 *    the call returns without synchronising.  dspark_check_status() synchronises.
 *  - Errors the host can see (bad sizes, NULL buffers, misalignment, short workspace,
 *    a teacher-dependent term without a teacher) are returned before anything is
 *    enqueued.  Errors only the device can see (an id out of range, a bounded wait
 *    that ran out) set a flag in the workspace; the offending row is skipped (it
 *    contributes nothing and its dlogits row is zero) and dspark_check_status()
 *    reports the flag.
 *  - Row r = (b*N + n)*K + k.  Logit rows have a leading dimension `*_ld` in
 *    elements; ld*sizeof(element) must be a multiple of 16 bytes, V*sizeof(element)
 *    must be a multiple of 16 bytes, and row pointers must be 16-byte aligned.
 *  - Calls that share a workspace must not overlap on the GPU.
 */
#ifndef DSPARK_H
#define DSPARK_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DSPARK_API __attribute__((visibility("default")))
#else
#define DSPARK_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t. */
typedef struct CUstream_st* dspark_stream_t;

typedef enum {
  DSPARK_OK = 0,
  DSPARK_ERR_INVALID_ARG = 1,     /* a size, pointer or parameter is not acceptable   */
  DSPARK_ERR_MISSING_TARGET = 2,  /* L1 or confidence term requested with no teacher
                                     (the ValueError of dspark_loss in the API doc)    */
  DSPARK_ERR_ID_OUT_OF_RANGE = 3, /* device: a target/prev id outside its vocabulary  */
  DSPARK_ERR_ALIGNMENT = 4,       /* a pointer or row stride breaks the 16-byte rule   */
  DSPARK_ERR_WORKSPACE = 5,       /* workspace NULL or smaller than required          */
  DSPARK_ERR_UNSUPPORTED = 6,     /* a shape/dtype combination this build does not run */
  DSPARK_ERR_DEVICE_TIMEOUT = 7,  /* device: a bounded wait gave up                   */
  DSPARK_ERR_CUDA = 8             /* the CUDA runtime reported an error               */
} dspark_status_t;

typedef enum { DSPARK_F32 = 0, DSPARK_BF16 = 1 } dspark_dtype_t;

/* Report pair order: report[2*i] = numerator, report[2*i + 1] = denominator. */
enum {
  DSPARK_REP_LOSS = 0,   /* [sum w*(a_ce CE + a_l1 L1 + a_c BCE), num_tokens]          */
  DSPARK_REP_CE = 1,     /* [sum w*CE, num_tokens]                                      */
  DSPARK_REP_L1 = 2,     /* [sum w*L1, num_tokens]  (raw L1)                            */
  DSPARK_REP_CONF = 3,   /* [sum w*BCE, num_tokens]  (0 numerator without confidence)   */
  DSPARK_REP_ACCEPT = 4, /* [sum m*accept, num_tokens]      "dspark accept rate"        */
  DSPARK_REP_TAU = 5,    /* [sum keep*tau_block, sum keep]  "dspark tau"                */
  DSPARK_REP_COUNT = 6
};

/*
 * One micro-batch: DSparkForwardOutput of the Megatron-Bridge API doc plus the head
 * inputs of the NeMo RL design doc.  Unused optional pointers are NULL.
 */
typedef struct {
  int64_t B, N, K, V;          /* R = B*N*K rows of V logits                            */
  int64_t logits_dtype;        /* dspark_dtype_t of draft, target and dlogits            */
  const void* draft_logits;    /* [R, V] base draft logits, row stride draft_ld          */
  int64_t draft_ld;
  const void* target_logits;   /* [R, V] teacher logits (row stride target_ld) or NULL   */
  int64_t target_ld;
  const int64_t* target_ids;   /* [R] teacher-forced next token, in [0, V)               */
  const uint8_t* eval_mask;    /* [R] nonzero = position enabled; cut to its prefix      */
  const uint8_t* block_keep;   /* [B*N] kept-anchor mask, or NULL = all kept             */
  const float* confidence_logits; /* [R] given confidence logits, or NULL                */
  /* teacher from the target's final hidden states (used when target_logits is NULL) */
  const void* target_hidden;   /* bf16 [R, target_hidden_size], already final-normed    */
  const void* lm_head;         /* bf16 [V, target_hidden_size]                          */
  int64_t target_hidden_size;
  /* Markov head (all NULL / 0 when absent).  Needs bf16 logits (the backward
   * contracts the bf16 dlogits on the tensor cores), markov_rank a multiple of 8 and
   * 16-byte aligned weights; otherwise DSPARK_ERR_UNSUPPORTED / DSPARK_ERR_ALIGNMENT. */
  const int64_t* prev_ids;     /* [R] previous token, in [0, target_vocab)              */
  const uint8_t* valid;        /* [R] nonzero = valid slot (also used by the conf head) */
  int64_t target_vocab;
  const void* markov_w1;       /* bf16 [target_vocab, markov_rank]                      */
  const void* markov_w2;       /* bf16 [V, markov_rank]                                 */
  int64_t markov_rank;
  /* confidence head (NULL when absent; exclusive with confidence_logits).  Needs
   * `valid`, hidden_size a multiple of 8 and 16-byte aligned draft_hidden / conf_w;
   * conf_with_markov needs the Markov head. */
  const void* draft_hidden;    /* bf16 [R, hidden_size]                                 */
  int64_t hidden_size;
  const void* conf_w;          /* bf16 [hidden_size (+ markov_rank)]: proj.weight       */
  const float* conf_b;         /* [1] proj.bias                                         */
  int64_t conf_with_markov;    /* 1: proj input is [hidden ; markov embedding]          */
  /* pre-norm teacher hidden states (NULL when target_hidden is already normed): the
   * target's final RMS norm, y = w * x / sqrt(mean(x^2) + eps) per row, rounded to bf16,
   * is applied to target_hidden before lm_head (TorchSpec pull request #132, review of
   * the vLLM path, whose stored last hidden states precede the final norm) */
  const void* target_norm_weight; /* bf16 [target_hidden_size], 16-byte aligned        */
  float target_norm_eps;       /* e.g. 1e-6                                             */
} dspark_problem_t;

typedef struct {
  float ce_alpha;              /* 0.1 in the API doc's signature                        */
  float l1_alpha;              /* 0.9                                                   */
  float conf_alpha;            /* 1.0 (used only with a confidence source)              */
  float gamma;                 /* 4.0                                                   */
  int32_t gamma_enabled;       /* 0 = no positional decay (loss_decay_gamma=None)       */
  int32_t invalid_row_mode;    /* 0: invalid Markov slot -> all-zero corrected row;
                                  1: invalid slot keeps its base row (bias removed)     */
} dspark_params_t;

/* Forward outputs.  Scalars are device buffers; per-row outputs are optional. */
typedef struct {
  float* loss_num;             /* [1] unnormalised weighted numerator                   */
  int64_t* num_tokens;         /* [1] supervised-token count (exact)                    */
  float* report;               /* [2*DSPARK_REP_COUNT] pairs, or NULL                   */
  float* ce_rows;              /* [R] CE per row (0 where unsupervised), or NULL        */
  float* l1_rows;              /* [R] raw L1 per row, or NULL                           */
  float* accept_rows;          /* [R] m*accept per row, or NULL                         */
  float* conf_rows;            /* [R] confidence logit used per row, or NULL            */
} dspark_fwd_out_t;

/* Backward outputs.  dlogits is written for EVERY row (zeros where unsupervised).  The
 * head gradients (dW1, dW2, dconf_w, dhidden) must be 16-byte aligned. */
typedef struct {
  const float* grad_scale;     /* device scalar g = d(objective)/d(loss_num); NULL = 1  */
  void* dlogits;               /* [R, V] dL/d(base draft logits), logits dtype          */
  int64_t dlogits_ld;
  float* dconf;                /* [R] dL/dc, or NULL                                    */
  float* dW1;                  /* fp32 [target_vocab, rank]: ALWAYS accumulated (+=)    */
  float* dW2;                  /* fp32 [V, rank]                                        */
  float* dconf_w;              /* fp32 [hidden_size (+ rank)]                           */
  float* dconf_b;              /* fp32 [1]                                              */
  void* dhidden;               /* bf16 [R, hidden_size], written for every row, or NULL */
  int64_t accumulate;          /* 1: dW2, dconf_w, dconf_b += ; 0: overwritten          */
} dspark_grads_t;

/* Bytes of device workspace dspark_loss_fwd / dspark_loss_bwd need for `prob`
 * (0 on an invalid problem).  Depends on the sizes and on which optional parts are
 * present (non-NULL), not on the addresses.  With the Markov head it includes the
 * corrected rows, 4*V bytes per row (the Markov head's corrected logits are kept in
 * FP32 between the forward and the backward). */
DSPARK_API size_t dspark_workspace_size(const dspark_problem_t* prob);

/*
 * Forward, and with `grads` != NULL the fused backward in the same sweep (the
 * gradient scale g must then be known before the call, e.g. 1 under per-token
 * loss).  Writes every field of `out` that is non-NULL; leaves in `ws` the per-row
 * statistics dspark_loss_bwd recomputes from.  `ws` must hold
 * dspark_workspace_size(prob) bytes, 256-byte aligned.
 */
DSPARK_API dspark_status_t dspark_loss_fwd(const dspark_problem_t* prob, const dspark_params_t* params,
                                const dspark_fwd_out_t* out, const dspark_grads_t* grads,
                                void* ws, size_t ws_bytes, dspark_stream_t stream);

/*
 * Backward alone, after a dspark_loss_fwd(..., grads = NULL) on the same problem,
 * params and workspace: one more pass over the logits (the corrected rows the forward
 * left in `ws` when the Markov head is on), recomputing the probabilities from the
 * per-row statistics saved in `ws`.  The statistics are kept; the backward writes its
 * own scratch (dL/dc per row, the split partials of dL/de) into `ws`.
 */
DSPARK_API dspark_status_t dspark_loss_bwd(const dspark_problem_t* prob, const dspark_params_t* params,
                                const dspark_grads_t* grads, void* ws, size_t ws_bytes,
                                dspark_stream_t stream);

/*
 * Acceptance report alone (Megatron-Bridge API doc, _acceptance_report) from per-row
 * raw L1 values: accept_r = clamp(1 - 0.5*l1_r, 0, 1) on supervised rows (m from
 * eval_mask and block_keep as above), tau_block = 1 + sum_k prod_{j<=k} m_j*accept_j.
 * Writes accept_pair[2] = [sum m*accept, sum m], tau_pair[2] = [sum keep*tau, sum keep]
 * and, if non-NULL, accept_rows[R] = m*accept.
 */
DSPARK_API dspark_status_t dspark_acceptance(int64_t B, int64_t N, int64_t K, const float* l1_rows,
                                  const uint8_t* eval_mask, const uint8_t* block_keep,
                                  float* accept_pair, float* tau_pair, float* accept_rows,
                                  dspark_stream_t stream);

/*
 * dspark_loss_fwd without a caller workspace (no counterpart on the source pages; it is
 * a service of this library).  For callers that cannot allocate device memory or pass
 * a workspace, e.g. an operator plugin whose host framework owns all device memory, or
 * a runtime that forbids cudaMalloc/cudaFree while serving because they synchronise the
 * device: the workspace is a fixed __device__ array inside this library,
 * DSPARK_NOALLOC_BYTES bytes, held on every GPU that loads the library until the process
 * exits.  Same problem, params, outputs and gradients as dspark_loss_fwd; nothing is
 * allocated.
 *  - Serves exactly the problems with at most DSPARK_NOALLOC_MAX_ROWS rows (B*N*K) and
 *    dspark_workspace_size(prob) <= DSPARK_NOALLOC_BYTES; every other problem returns
 *    DSPARK_ERR_WORKSPACE before anything is enqueued.  Without heads that is every
 *    micro-batch of at most 8192 rows.  The Markov head (its FP32 bias rows take 4*V
 *    bytes per supervised row) and the teacher from hidden states (its FP32 teacher chunk
 *    takes 4*V bytes per chunk row) never fit at a real vocabulary.  A confidence head
 *    adds ceil(R/16)*(hidden_size [+ markov_rank])*4 bytes of partial sums, so with
 *    hidden_size 4096 it fits only up to about 430 rows (the 448-row recipe micro-batch
 *    with a confidence head is refused).
 *  - The first call on a device (and the first after that device's context was torn down
 *    and created again) looks the array's device address up, with that device current;
 *    make that first call before any stream capture.
 *  - Every call on a device shares the one array and leaves its contents behind; the
 *    next call clears what must start at zero.  Calls that overlap on the GPU (other
 *    streams, other threads) race on the array: serialise them.
 *  - Device-side error flags land in the shared array and are not reported back (there
 *    is no workspace pointer to pass to dspark_check_status); rows with out-of-range ids
 *    are still skipped.
 */
enum { DSPARK_NOALLOC_MAX_ROWS = 8192, DSPARK_NOALLOC_BYTES = 467200 };

DSPARK_API dspark_status_t dspark_loss_fwd_noalloc(const dspark_problem_t* prob,
                                                   const dspark_params_t* params,
                                                   const dspark_fwd_out_t* out,
                                                   const dspark_grads_t* grads,
                                                   dspark_stream_t stream);

/*
 * Vocabulary-parallel (tensor-parallel) loss.  NeMo RL design doc "DSpark Auxiliary
 * Heads", Tensor Parallelism: each tensor-parallel rank receives the base logits of
 * its own shard of the draft vocabulary.  The row terms are full-vocabulary sums, so
 * each rank reduces its columns to per-row partials, the ranks exchange them, and
 * every rank merges all ranks' partials in rank order: every rank then holds bitwise
 * the same row statistics and writes the same forward outputs.  One micro-batch is
 * three calls per rank, with an all-gather over the tensor-parallel group (done by
 * the caller, e.g. NCCL all_gather) after each of the first two:
 *
 *   dspark_tp_partials(prob, params, tp, rec1, ws, ...)        rec1:     [R][8] floats
 *   all-gather rec1 in rank order                               rec1_all: [tp_size][R][8]
 *   dspark_tp_l1(prob, params, tp, rec1_all, rec2, ws, ...)     rec2:     [R][4] floats
 *   all-gather rec2 in rank order                               rec2_all: [tp_size][R][4]
 *   dspark_tp_finish(prob, params, tp, rec2_all, out, grads, de_part, ws, ...)
 * and with a head and gradients a fourth call after one more all-gather:
 *   all-gather de_part in rank order (Markov head only)         de_all: [tp_size][R][rank]
 *   dspark_tp_heads_bwd(prob, params, tp, de_all, grads, ws, ...)
 *
 * `prob` describes this rank's shard: V is the shard's width; draft_logits,
 * target_logits and dlogits point at the shard's first column, with the full rows'
 * strides as their leading dimensions; target_ids are GLOBAL ids in [0, vocab_size).
 * The ranks' shards must tile [0, vocab_size) without overlap.  Shard widths obey the
 * 16-byte rule above (multiples of 8 bf16 or 4 fp32 columns).  Heads follow the same
 * design doc section: markov_w2 points at this shard's rows [V, markov_rank] (its rows
 * split over the ranks) while markov_w1 and the confidence head are replicated; dW2 is
 * written for this shard's rows, and the embedding gradient dL/de is the sum of the
 * ranks' parts (the reduce across tensor parallelism) before dW1 is scattered and the
 * confidence head's own term dc*proj_e is added once.  dW1, dconf_w, dconf_b and dhidden
 * come out the same on every rank.  The teacher from hidden states is taken on this path
 * with lm_head split like the logits: lm_head points at this shard's rows [V,
 * target_hidden_size] and target_hidden (with target_norm_weight) is replicated;
 * dspark_tp_partials computes the shard's FP32 teacher rows of every supervised row into
 * the workspace, where the next two calls read them, so a micro-batch may hold at most 512
 * rows (DSPARK_ERR_UNSUPPORTED above that).  Sum the forward outputs and the replicated gradients
 * over data-parallel ranks only: every tensor-parallel rank holds the same values.  The
 * calls of a micro-batch take the same problem, params, tp and workspace
 * (dspark_workspace_size(prob) bytes), in stream order.
 *
 * Record 1 of row r (rec1 + 8r): [m_d, s_d, m_t, s_t, zt, 0, 0, 0] where, over this
 * shard's columns, m = max_j x_j*log2(e) (-inf for no column) and s = sum_j
 * 2^(x_j*log2(e) - m) for the draft (d) and the teacher (t; -inf, 0 without one), and
 * zt is the draft logit at the target id if this shard holds that id, else 0.
 * Record 2 of row r (rec2 + 4r): [L1 part, S part, 0, 0], this shard's sums of
 * |p_j - q_j| and p_j*sign(p_j - q_j) (an exact tie counts as +p_j).  Only supervised
 * rows' records are written; the others are left as they were.  Records are
 * 16-byte aligned device buffers owned by the caller.
 */
typedef struct {
  int64_t tp_size;      /* ranks sharing the vocabulary, in [1, 1024]                  */
  int64_t vocab_begin;  /* global id of this shard's first column                      */
  int64_t vocab_size;   /* the whole vocabulary: vocab_begin + V <= vocab_size <= 2^30 */
} dspark_tp_t;

enum { DSPARK_TP_REC1_FLOATS = 8, DSPARK_TP_REC2_FLOATS = 4 };

/* Step 1: the mask prologue (ids checked against vocab_size) and this shard's
 * logsumexp partials and target logit -> rec1. */
DSPARK_API dspark_status_t dspark_tp_partials(const dspark_problem_t* prob, const dspark_params_t* params,
                                              const dspark_tp_t* tp, float* rec1, void* ws,
                                              size_t ws_bytes, dspark_stream_t stream);

/* Step 2: merges rec1_all (every rank's rec1, rank order) into the row logsumexps and
 * the target logit, saved in `ws`, then this shard's (L1, S) partials -> rec2. */
DSPARK_API dspark_status_t dspark_tp_l1(const dspark_problem_t* prob, const dspark_params_t* params,
                                        const dspark_tp_t* tp, const float* rec1_all, float* rec2,
                                        void* ws, size_t ws_bytes, dspark_stream_t stream);

/* Step 3: sums rec2_all (rank order) into L1 and S, writes the forward outputs (as
 * dspark_loss_fwd) and, with `grads`, dlogits of this shard's columns for every row
 * (zeros where unsupervised) and dconf.  With the Markov head and `grads` it also writes
 * dW2 for this shard's rows and this shard's part of dL/de, W2_shard^T dz_r for every
 * row r (0 where no gradient flows), into de_part ([R][markov_rank] floats, 16-byte
 * aligned, owned by the caller); de_part may be NULL otherwise. */
DSPARK_API dspark_status_t dspark_tp_finish(const dspark_problem_t* prob, const dspark_params_t* params,
                                            const dspark_tp_t* tp, const float* rec2_all,
                                            const dspark_fwd_out_t* out, const dspark_grads_t* grads,
                                            float* de_part, void* ws, size_t ws_bytes, dspark_stream_t stream);

/* Step 4, with a head and gradients: dL/de_r = the ranks' de_part rows summed (de_all,
 * [tp_size][R][markov_rank], rank order; NULL without the Markov head) + dc_r*proj_e,
 * dW1[prev_r] += dL/de_r, and the confidence head's dconf_w, dconf_b and dhidden.  The
 * same on every rank.  Returns DSPARK_OK without work when the problem has no head. */
DSPARK_API dspark_status_t dspark_tp_heads_bwd(const dspark_problem_t* prob, const dspark_params_t* params,
                                               const dspark_tp_t* tp, const float* de_all,
                                               const dspark_grads_t* grads, void* ws, size_t ws_bytes,
                                               dspark_stream_t stream);

/* Synchronises `stream` and returns the first device-side error recorded in `ws`
 * by the last call that used it (DSPARK_OK if none). */
DSPARK_API dspark_status_t dspark_check_status(const void* ws, dspark_stream_t stream);

/* Static English text for a status code. */
DSPARK_API const char* dspark_status_string(dspark_status_t status);

/* Name of the CUDA runtime error behind the most recent DSPARK_ERR_CUDA returned by any
 * call of this library in the process ("cudaSuccess" if there was none).  A library
 * service with no counterpart on the source pages: it tells the caller which CUDA call
 * failed without a debugger.  Static storage; never NULL. */
DSPARK_API const char* dspark_last_cuda_error(void);

#ifdef __cplusplus
}
#endif
#endif /* DSPARK_H */
