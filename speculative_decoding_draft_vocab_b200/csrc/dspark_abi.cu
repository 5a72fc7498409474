// The C ABI of include/dspark.h: host-side validation, workspace carving and the
// launch sequence of each entry point.  No allocation, no synchronisation (except
// dspark_check_status, whose job it is).
#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>

#include "internal.cuh"
#include "tp.cuh"

using namespace dspark;

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t elem_size(int64_t dtype) { return dtype == DSPARK_BF16 ? 2 : 4; }

// Which optional parts a problem uses.
struct Shape {
  int64_t R;
  bool has_target_rows;  // teacher given as logits
  bool has_lm_head;      // teacher from hidden states
  bool has_teacher;
  bool has_markov;
  bool has_conf_given;
  bool has_conf_head;
};

inline bool markov_present(const dspark_problem_t* p) {
  return p->markov_w2 != nullptr || p->markov_w1 != nullptr || p->prev_ids != nullptr;
}

inline bool lm_present(const dspark_problem_t* p) { return p->lm_head != nullptr || p->target_hidden != nullptr; }

inline WsDims ws_dims(const dspark_problem_t* p) {
  WsDims d{};
  d.R = p->B * p->N * p->K;
  d.V = p->V;
  d.markov = markov_present(p);
  if (d.markov) {
    d.rank = p->markov_rank;
    d.splits = heads_splits(d.R, p->V);
  }
  if (p->conf_w != nullptr || p->draft_hidden != nullptr)
    d.conf_cols = p->hidden_size + (p->conf_with_markov && d.markov ? p->markov_rank : 0);
  d.lm = lm_present(p) && p->target_logits == nullptr;
  if (d.lm) {
    d.Ht = p->target_hidden_size;
    d.chunk = teacher_chunk_rows(d.R);
  }
  return d;
}

// Row types the sweep reads and writes.
inline int sweep_kind(const dspark_problem_t* p) {
  if (p->logits_dtype == DSPARK_F32) return kSweepF32;
  const bool z32 = markov_present(p), t32 = lm_present(p);
  return z32 ? (t32 ? kSweepZT32 : kSweepZ32) : (t32 ? kSweepT32 : kSweepBf16);
}

// `sweep`: the fused row sweep will run this problem (its builds bound V).
dspark_status_t check_problem(const dspark_problem_t* p, const dspark_params_t* prm, Shape* sh,
                              bool sweep = true) {
  if (p == nullptr) return DSPARK_ERR_INVALID_ARG;
  if (p->B <= 0 || p->N <= 0 || p->K <= 0 || p->V <= 0) return DSPARK_ERR_INVALID_ARG;
  if (p->logits_dtype != DSPARK_F32 && p->logits_dtype != DSPARK_BF16) return DSPARK_ERR_INVALID_ARG;
  if (p->B * p->N * p->K > (int64_t(1) << 31) - 1) return DSPARK_ERR_UNSUPPORTED;
  if (p->V > (int64_t(1) << 30)) return DSPARK_ERR_UNSUPPORTED;
  if (!p->draft_logits || !p->target_ids || !p->eval_mask) return DSPARK_ERR_INVALID_ARG;
  const size_t es = elem_size(p->logits_dtype);
  if (p->draft_ld < p->V) return DSPARK_ERR_INVALID_ARG;
  if (!aligned16(p->draft_logits) || (p->draft_ld * es) % 16 || (p->V * es) % 16)
    return DSPARK_ERR_ALIGNMENT;
  Shape s{};
  s.R = p->B * p->N * p->K;
  s.has_target_rows = p->target_logits != nullptr;
  s.has_lm_head = lm_present(p);
  s.has_teacher = s.has_target_rows || s.has_lm_head;
  s.has_markov = markov_present(p);
  s.has_conf_given = p->confidence_logits != nullptr;
  s.has_conf_head = p->conf_w != nullptr || p->draft_hidden != nullptr;
  if (s.has_target_rows) {
    if (p->target_ld < p->V) return DSPARK_ERR_INVALID_ARG;
    if (!aligned16(p->target_logits) || (p->target_ld * es) % 16) return DSPARK_ERR_ALIGNMENT;
  }
  if (s.has_target_rows && s.has_lm_head) return DSPARK_ERR_INVALID_ARG;
  if (s.has_conf_given && s.has_conf_head) return DSPARK_ERR_INVALID_ARG;
  if (prm != nullptr) {
    if (!s.has_teacher && (prm->l1_alpha != 0.f || s.has_conf_given || s.has_conf_head))
      return DSPARK_ERR_MISSING_TARGET;
    if (prm->gamma_enabled && !(prm->gamma > 0.f)) return DSPARK_ERR_INVALID_ARG;
    if (prm->invalid_row_mode != 0 && prm->invalid_row_mode != 1) return DSPARK_ERR_INVALID_ARG;
  }
  if (p->target_norm_weight && !s.has_lm_head) return DSPARK_ERR_INVALID_ARG;
  if (s.has_lm_head) {
    if (!p->lm_head || !p->target_hidden || p->target_hidden_size <= 0) return DSPARK_ERR_INVALID_ARG;
    // the teacher rows come from the tensor cores in FP32; the sweep pairs them with
    // bf16 logits
    if (p->logits_dtype != DSPARK_BF16) return DSPARK_ERR_UNSUPPORTED;
    if (p->target_hidden_size % 8 || !aligned16(p->lm_head) || !aligned16(p->target_hidden) ||
        (p->target_norm_weight && !aligned16(p->target_norm_weight)))
      return DSPARK_ERR_ALIGNMENT;
    if (p->target_norm_weight && !(p->target_norm_eps >= 0.f)) return DSPARK_ERR_INVALID_ARG;
  }
  if (s.has_markov) {
    if (!p->markov_w1 || !p->markov_w2 || !p->prev_ids || !p->valid) return DSPARK_ERR_INVALID_ARG;
    if (p->markov_rank <= 0 || p->target_vocab <= 0) return DSPARK_ERR_INVALID_ARG;
    // the backward contracts the bf16 dlogits on the tensor cores
    if (p->logits_dtype != DSPARK_BF16) return DSPARK_ERR_UNSUPPORTED;
    if (p->markov_rank % 8 || !aligned16(p->markov_w1) || !aligned16(p->markov_w2)) return DSPARK_ERR_ALIGNMENT;
  }
  if (s.has_conf_head) {
    if (!p->conf_w || !p->conf_b || !p->draft_hidden || !p->valid) return DSPARK_ERR_INVALID_ARG;
    if (p->hidden_size <= 0) return DSPARK_ERR_INVALID_ARG;
    if (p->conf_with_markov && !s.has_markov) return DSPARK_ERR_INVALID_ARG;
    if (p->hidden_size % 8 || !aligned16(p->conf_w) || !aligned16(p->draft_hidden)) return DSPARK_ERR_ALIGNMENT;
  }
  if (sweep && !sweep_supported(sweep_kind(p), p->V, s.has_teacher)) return DSPARK_ERR_UNSUPPORTED;
  *sh = s;
  return DSPARK_OK;
}

// The CUDA error behind the most recent DSPARK_ERR_CUDA of any call in this process.
std::atomic<int> g_last_cuda_error{0};

inline dspark_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return DSPARK_OK;
  g_last_cuda_error.store(int(e), std::memory_order_relaxed);
  return DSPARK_ERR_CUDA;
}

dspark_status_t check_ws(const dspark_problem_t* p, const void* ws, size_t ws_bytes) {
  if (ws == nullptr) return DSPARK_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return DSPARK_ERR_ALIGNMENT;
  if (ws_bytes < ws_offsets(ws_dims(p)).bytes) return DSPARK_ERR_WORKSPACE;
  return DSPARK_OK;
}

dspark_status_t check_grads(const dspark_problem_t* p, const dspark_grads_t* g) {
  if (g == nullptr || g->dlogits == nullptr) return DSPARK_ERR_INVALID_ARG;
  const size_t es = elem_size(p->logits_dtype);
  if (g->dlogits_ld < p->V) return DSPARK_ERR_INVALID_ARG;
  if (!aligned16(g->dlogits) || (g->dlogits_ld * es) % 16) return DSPARK_ERR_ALIGNMENT;
  // head gradients are written in 16-byte vectors or by tensor stores
  if ((g->dW1 && !aligned16(g->dW1)) || (g->dW2 && !aligned16(g->dW2)) || (g->dhidden && !aligned16(g->dhidden)) ||
      (g->dconf_w && !aligned16(g->dconf_w)))
    return DSPARK_ERR_ALIGNMENT;
  return DSPARK_OK;
}

SweepArgs sweep_args(const dspark_problem_t* p, const dspark_params_t* prm, const WsView& ws,
                     const dspark_grads_t* g) {
  SweepArgs a{};
  a.draft = p->draft_logits;
  a.ld_d = p->draft_ld;
  a.target = p->target_logits;
  a.ld_t = p->target_ld;
  a.dlogits = g ? g->dlogits : nullptr;
  a.ld_g = g ? g->dlogits_ld : 0;
  a.tids = p->target_ids;
  a.grad_scale = g ? g->grad_scale : nullptr;
  a.ws = ws;
  a.V = p->V;
  a.ce_alpha = prm->ce_alpha;
  a.l1_alpha = (p->target_logits || lm_present(p)) ? prm->l1_alpha : 0.f;
  a.row0 = 0;
  a.row1 = int32_t(p->B * p->N * p->K);
  a.do_zero = 1;
  a.do_final = 1;
  if (lm_present(p)) {  // the teacher rows of the current chunk
    a.target = ws.tchunk;
    a.ld_t = p->V;
    a.target_compact = 1;
  }
  if (markov_present(p)) {  // the sweep adds the head's bias rows (compact by supervised position)
    a.bias = ws.bias;
    a.ld_b = p->V;
    a.valid = p->valid;
    a.invalid_zero = prm->invalid_row_mode == 0;
  }
  return a;
}

TeacherArgs teacher_args(const dspark_problem_t* p, const WsView& ws) {
  TeacherArgs t{};
  t.R = p->B * p->N * p->K;
  t.V = p->V;
  t.Ht = p->target_hidden_size;
  t.hidden = static_cast<const uint16_t*>(p->target_hidden);
  t.lm_head = static_cast<const uint16_t*>(p->lm_head);
  t.norm_w = static_cast<const uint16_t*>(p->target_norm_weight);
  t.norm_eps = p->target_norm_eps;
  t.ws = ws;
  return t;
}

HeadsArgs heads_args(const dspark_problem_t* p, const dspark_params_t* prm, const WsView& ws,
                     const dspark_grads_t* g) {
  HeadsArgs h{};
  h.R = p->B * p->N * p->K;
  h.V = p->V;
  h.Vt = p->target_vocab;
  h.rank = markov_present(p) ? p->markov_rank : 0;
  h.H = p->conf_w ? p->hidden_size : 0;
  h.prev_ids = p->prev_ids;
  h.valid = p->valid;
  h.w1 = markov_present(p) ? static_cast<const uint16_t*>(p->markov_w1) : nullptr;
  h.w2 = static_cast<const uint16_t*>(p->markov_w2);
  h.hidden = static_cast<const uint16_t*>(p->draft_hidden);
  h.conf_w = static_cast<const uint16_t*>(p->conf_w);
  h.conf_b = p->conf_b;
  h.conf_with_markov = p->conf_w && p->conf_with_markov ? 1 : 0;
  h.invalid_row_mode = prm->invalid_row_mode;
  if (g) {
    h.dlogits = static_cast<const uint16_t*>(g->dlogits);
    h.ld_g = g->dlogits_ld;
    h.dw1 = g->dW1;
    h.dw2 = g->dW2;
    h.dconf_w = g->dconf_w;
    h.dconf_b = g->dconf_b;
    h.dhidden = static_cast<uint16_t*>(g->dhidden);
    h.accumulate = g->accumulate ? 1 : 0;
  }
  h.ws = ws;
  return h;
}

// A vocabulary-parallel shard: the plain problem's rules, no teacher from hidden states,
// and a shard that lies inside the vocabulary.
dspark_status_t check_tp(const dspark_problem_t* p, const dspark_params_t* prm, const dspark_tp_t* tp,
                         Shape* sh) {
  if (prm == nullptr || tp == nullptr) return DSPARK_ERR_INVALID_ARG;
  dspark_status_t st = check_problem(p, prm, sh, false);
  if (st != DSPARK_OK) return st;
  // the teacher from hidden states: the shard's teacher rows of every supervised row are
  // kept in the workspace's teacher chunk through the three calls, so all rows must fit
  // one chunk
  if (sh->has_lm_head && sh->R > kTeacherChunk) return DSPARK_ERR_UNSUPPORTED;
  if (tp->tp_size < 1 || tp->tp_size > 1024) return DSPARK_ERR_INVALID_ARG;
  if (tp->vocab_size <= 0 || tp->vocab_size > (int64_t(1) << 30) || tp->vocab_begin < 0 ||
      tp->vocab_begin > tp->vocab_size - p->V)
    return DSPARK_ERR_INVALID_ARG;
  return DSPARK_OK;
}

dspark_status_t check_rec(const float* r) {
  if (r == nullptr) return DSPARK_ERR_INVALID_ARG;
  return aligned16(r) ? DSPARK_OK : DSPARK_ERR_ALIGNMENT;
}

TpArgs tp_args(const dspark_problem_t* p, const dspark_params_t* prm, const dspark_tp_t* tp,
               const WsView& ws) {
  TpArgs a{};
  a.draft = p->draft_logits;
  a.ld_d = p->draft_ld;
  a.target = p->target_logits;
  a.ld_t = p->target_ld;
  a.tids = p->target_ids;
  a.R = p->B * p->N * p->K;
  a.V = p->V;
  a.vocab_begin = tp->vocab_begin;
  a.tp_size = int32_t(tp->tp_size);
  a.ce_alpha = prm->ce_alpha;
  a.l1_alpha = (p->target_logits || lm_present(p)) ? prm->l1_alpha : 0.f;
  a.bias = markov_present(p) ? ws.bias : nullptr;
  if (lm_present(p)) {  // the shard's teacher rows, computed by dspark_tp_partials
    a.target = ws.tchunk;
    a.ld_t = p->V;
    a.t_compact = 1;
  }
  a.ws = ws;
  return a;
}

}  // namespace

extern "C" {

const char* dspark_status_string(dspark_status_t s) {
  switch (s) {
    case DSPARK_OK: return "ok";
    case DSPARK_ERR_INVALID_ARG: return "invalid argument";
    case DSPARK_ERR_MISSING_TARGET: return "L1 or confidence term requested without target logits";
    case DSPARK_ERR_ID_OUT_OF_RANGE: return "a target or previous-token id is outside its vocabulary";
    case DSPARK_ERR_ALIGNMENT: return "pointer or row stride is not 16-byte aligned";
    case DSPARK_ERR_WORKSPACE: return "workspace missing or too small";
    case DSPARK_ERR_UNSUPPORTED: return "shape or option not supported by this build";
    case DSPARK_ERR_DEVICE_TIMEOUT: return "a bounded device wait ran out";
    case DSPARK_ERR_CUDA: return "CUDA runtime error";
  }
  return "unknown status";
}

const char* dspark_last_cuda_error(void) {
  return cudaGetErrorName(static_cast<cudaError_t>(g_last_cuda_error.load(std::memory_order_relaxed)));
}

size_t dspark_workspace_size(const dspark_problem_t* prob) {
  if (prob == nullptr || prob->B <= 0 || prob->N <= 0 || prob->K <= 0) return 0;
  if (markov_present(prob) && (prob->V <= 0 || prob->markov_rank <= 0)) return 0;
  return ws_offsets(ws_dims(prob)).bytes;
}

dspark_status_t dspark_loss_fwd(const dspark_problem_t* prob, const dspark_params_t* params,
                                const dspark_fwd_out_t* out, const dspark_grads_t* grads,
                                void* ws, size_t ws_bytes, dspark_stream_t stream) {
  if (params == nullptr || out == nullptr) return DSPARK_ERR_INVALID_ARG;
  Shape sh{};
  dspark_status_t st = check_problem(prob, params, &sh);
  if (st != DSPARK_OK) return st;
  if ((st = check_ws(prob, ws, ws_bytes)) != DSPARK_OK) return st;
  if (grads && (st = check_grads(prob, grads)) != DSPARK_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const WsView v = ws_layout(ws, ws_dims(prob));

  PrologueArgs pa{};
  pa.B = prob->B; pa.N = prob->N; pa.K = prob->K; pa.V = prob->V; pa.Vt = prob->target_vocab;
  pa.eval_mask = prob->eval_mask;
  pa.block_keep = prob->block_keep;
  pa.target_ids = prob->target_ids;
  pa.prev_ids = sh.has_markov ? prob->prev_ids : nullptr;
  pa.valid = prob->valid;
  pa.invalid_zero = sh.has_markov && params->invalid_row_mode == 0;
  pa.gamma = params->gamma;
  pa.gamma_enabled = params->gamma_enabled;
  pa.ws = v;
  cudaError_t e = launch_prologue(pa, s);
  if (e != cudaSuccess) return cuda_status(e);

  const HeadsArgs ha = heads_args(prob, params, v, grads);
  if (sh.has_markov || sh.has_conf_head) {
    if ((e = launch_heads_prep(ha, s)) != cudaSuccess) return cuda_status(e);
  }
  if (sh.has_markov) {
    if ((e = launch_markov_bias(ha, s)) != cudaSuccess) return cuda_status(e);
  }

  SweepArgs sa = sweep_args(prob, params, v, grads);
  FinalizeArgs& fa = sa.fin;
  fa.B = prob->B; fa.N = prob->N; fa.K = prob->K;
  fa.block_keep = prob->block_keep;
  fa.confidence_logits = prob->confidence_logits;
  fa.has_conf = sh.has_conf_given || sh.has_conf_head;
  fa.ce_alpha = params->ce_alpha;
  fa.l1_alpha = params->l1_alpha;
  fa.conf_alpha = params->conf_alpha;
  fa.grad_scale = grads ? grads->grad_scale : nullptr;
  fa.ws = v;
  fa.loss_num = out->loss_num;
  fa.num_tokens = out->num_tokens;
  fa.report = out->report;
  fa.ce_rows = out->ce_rows;
  fa.l1_rows = out->l1_rows;
  fa.accept_rows = out->accept_rows;
  fa.conf_rows = out->conf_rows;
  fa.dconf = grads ? grads->dconf : nullptr;
  const int kind = sweep_kind(prob);
  if (!sh.has_lm_head) {
    // the zero rows are filled on the SMs the sweep leaves idle, by its dependent grid
    const bool side_zero = sa.dlogits != nullptr;
    sa.do_zero = side_zero ? 0 : 1;
    int ctas = 0;
    e = launch_sweep(kind, sh.has_teacher, sa, s, &ctas);
    if (e == cudaSuccess && side_zero) e = launch_zero_rows(kind, sa, ctas, s);
    if (e != cudaSuccess) return cuda_status(e);
  } else {
    // teacher rows a chunk of supervised rows at a time, each chunk swept right after
    const TeacherArgs ta = teacher_args(prob, v);
    if ((e = launch_gather_hidden(ta, s)) != cudaSuccess) return cuda_status(e);
    const int64_t C = teacher_chunk_rows(sh.R);
    for (int64_t r0 = 0; r0 < sh.R; r0 += C) {
      if ((e = launch_teacher_chunk(ta, r0, s)) != cudaSuccess) return cuda_status(e);
      sa.row0 = int32_t(r0);
      sa.row1 = int32_t(std::min<int64_t>(r0 + C, sh.R));
      sa.do_zero = r0 == 0;
      sa.do_final = r0 + C >= sh.R;
      if ((e = launch_sweep(kind, true, sa, s)) != cudaSuccess) return cuda_status(e);
    }
  }
  if (grads && (sh.has_markov || sh.has_conf_head)) e = launch_heads_bwd(ha, s);
  return cuda_status(e);
}

dspark_status_t dspark_loss_bwd(const dspark_problem_t* prob, const dspark_params_t* params,
                                const dspark_grads_t* grads, void* ws, size_t ws_bytes,
                                dspark_stream_t stream) {
  if (params == nullptr) return DSPARK_ERR_INVALID_ARG;
  Shape sh{};
  dspark_status_t st = check_problem(prob, params, &sh);
  if (st != DSPARK_OK) return st;
  if ((st = check_ws(prob, ws, ws_bytes)) != DSPARK_OK) return st;
  if ((st = check_grads(prob, grads)) != DSPARK_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const WsView v = ws_layout(ws, ws_dims(prob));
  SweepArgs sa = sweep_args(prob, params, v, grads);
  const int kind = sweep_kind(prob);
  cudaError_t e = cudaSuccess;
  if (!sh.has_lm_head) {
    e = launch_bwd_stream(kind, sh.has_teacher, sa, sh.R, s);
    if (e != cudaSuccess) return cuda_status(e);
  } else {
    // a single chunk is still in the workspace from the forward; more are recomputed
    const TeacherArgs ta = teacher_args(prob, v);
    const int64_t C = teacher_chunk_rows(sh.R);
    for (int64_t r0 = 0; r0 < sh.R; r0 += C) {
      if (C < sh.R && (e = launch_teacher_chunk(ta, r0, s)) != cudaSuccess) return cuda_status(e);
      sa.row0 = int32_t(r0);
      sa.row1 = int32_t(std::min<int64_t>(r0 + C, sh.R));
      sa.do_zero = r0 == 0;
      if ((e = launch_bwd_stream(kind, true, sa, sh.R, s)) != cudaSuccess) return cuda_status(e);
    }
  }
  if (sh.has_conf_given || sh.has_conf_head) {
    // dL/dc for this call's grad_scale, also saved for the confidence head's backward
    e = launch_conf_grad(sh.R, prob->confidence_logits, params->conf_alpha, grads->grad_scale, v,
                         grads->dconf, s);
  } else if (grads->dconf) {
    e = cudaMemsetAsync(grads->dconf, 0, sizeof(float) * sh.R, s);
  }
  if (e != cudaSuccess) return cuda_status(e);
  if (sh.has_markov || sh.has_conf_head) e = launch_heads_bwd(heads_args(prob, params, v, grads), s);
  return cuda_status(e);
}

dspark_status_t dspark_acceptance(int64_t B, int64_t N, int64_t K, const float* l1_rows,
                                  const uint8_t* eval_mask, const uint8_t* block_keep,
                                  float* accept_pair, float* tau_pair, float* accept_rows,
                                  dspark_stream_t stream) {
  if (B <= 0 || N <= 0 || K <= 0) return DSPARK_ERR_INVALID_ARG;
  if (!l1_rows || !eval_mask || !accept_pair || !tau_pair) return DSPARK_ERR_INVALID_ARG;
  return cuda_status(launch_acceptance(B, N, K, l1_rows, eval_mask, block_keep, accept_pair,
                                       tau_pair, accept_rows, reinterpret_cast<cudaStream_t>(stream)));
}

dspark_status_t dspark_tp_partials(const dspark_problem_t* prob, const dspark_params_t* params,
                                   const dspark_tp_t* tp, float* rec1, void* ws, size_t ws_bytes,
                                   dspark_stream_t stream) {
  Shape sh{};
  dspark_status_t st = check_tp(prob, params, tp, &sh);
  if (st != DSPARK_OK) return st;
  if ((st = check_ws(prob, ws, ws_bytes)) != DSPARK_OK) return st;
  if ((st = check_rec(rec1)) != DSPARK_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const WsView v = ws_layout(ws, ws_dims(prob));
  PrologueArgs pa{};
  pa.B = prob->B; pa.N = prob->N; pa.K = prob->K;
  pa.V = tp->vocab_size;  // target ids are global
  pa.Vt = prob->target_vocab;
  pa.eval_mask = prob->eval_mask;
  pa.block_keep = prob->block_keep;
  pa.target_ids = prob->target_ids;
  pa.prev_ids = sh.has_markov ? prob->prev_ids : nullptr;
  pa.valid = prob->valid;
  pa.invalid_zero = sh.has_markov && params->invalid_row_mode == 0;
  pa.gamma = params->gamma;
  pa.gamma_enabled = params->gamma_enabled;
  pa.ws = v;
  cudaError_t e = launch_prologue(pa, s);
  if (e != cudaSuccess) return cuda_status(e);
  if (sh.has_markov || sh.has_conf_head) {
    // embeddings and confidence logits (replicated), the bias rows of this shard
    const HeadsArgs ha = heads_args(prob, params, v, nullptr);
    if ((e = launch_heads_prep(ha, s)) != cudaSuccess) return cuda_status(e);
    if (sh.has_markov && (e = launch_markov_bias(ha, s)) != cudaSuccess) return cuda_status(e);
  }
  if (sh.has_lm_head) {
    // the supervised rows' hidden states (with the final norm if pre-norm), then the
    // shard's teacher rows: hidden x lm_head rows of the shard, FP32, on the tensor cores
    const TeacherArgs ta = teacher_args(prob, v);
    if ((e = launch_gather_hidden(ta, s)) != cudaSuccess) return cuda_status(e);
    if ((e = launch_teacher_chunk(ta, 0, s)) != cudaSuccess) return cuda_status(e);
  }
  TpArgs a = tp_args(prob, params, tp, v);
  a.rec1 = rec1;
  if (!sh.has_markov && !sh.has_conf_head && !sh.has_lm_head) {  // nothing between the prologue and step 1
    a.own_rows = 1;
    a.eval_mask = prob->eval_mask;
    a.block_keep = prob->block_keep;
    a.K = prob->K;
    a.vocab_size = tp->vocab_size;
  }
  return cuda_status(launch_tp_partials(prob->logits_dtype == DSPARK_F32, a, s));
}

dspark_status_t dspark_tp_l1(const dspark_problem_t* prob, const dspark_params_t* params,
                             const dspark_tp_t* tp, const float* rec1_all, float* rec2, void* ws,
                             size_t ws_bytes, dspark_stream_t stream) {
  Shape sh{};
  dspark_status_t st = check_tp(prob, params, tp, &sh);
  if (st != DSPARK_OK) return st;
  if ((st = check_ws(prob, ws, ws_bytes)) != DSPARK_OK) return st;
  if ((st = check_rec(rec1_all)) != DSPARK_OK || (st = check_rec(rec2)) != DSPARK_OK) return st;
  const WsView v = ws_layout(ws, ws_dims(prob));
  TpArgs a = tp_args(prob, params, tp, v);
  a.rec1_all = rec1_all;
  a.rec2 = rec2;
  return cuda_status(launch_tp_l1(prob->logits_dtype == DSPARK_F32, a, reinterpret_cast<cudaStream_t>(stream)));
}

dspark_status_t dspark_tp_finish(const dspark_problem_t* prob, const dspark_params_t* params,
                                 const dspark_tp_t* tp, const float* rec2_all,
                                 const dspark_fwd_out_t* out, const dspark_grads_t* grads, float* de_part,
                                 void* ws, size_t ws_bytes, dspark_stream_t stream) {
  if (out == nullptr) return DSPARK_ERR_INVALID_ARG;
  Shape sh{};
  dspark_status_t st = check_tp(prob, params, tp, &sh);
  if (st != DSPARK_OK) return st;
  if ((st = check_ws(prob, ws, ws_bytes)) != DSPARK_OK) return st;
  if ((st = check_rec(rec2_all)) != DSPARK_OK) return st;
  if (grads) {
    if ((st = check_grads(prob, grads)) != DSPARK_OK) return st;
    // this shard's part of dL/de goes to de_part
    if (sh.has_markov && (st = check_rec(de_part)) != DSPARK_OK) return st;
  }
  const WsView v = ws_layout(ws, ws_dims(prob));
  TpArgs a = tp_args(prob, params, tp, v);
  a.rec2_all = rec2_all;
  if (grads) {
    a.dlogits = grads->dlogits;
    a.ld_g = grads->dlogits_ld;
    a.grad_scale = grads->grad_scale;
  }
  FinalizeArgs& f = a.fin;
  f.B = prob->B; f.N = prob->N; f.K = prob->K;
  f.block_keep = prob->block_keep;
  f.confidence_logits = prob->confidence_logits;
  f.has_conf = sh.has_conf_given || sh.has_conf_head;
  f.ce_alpha = params->ce_alpha;
  f.l1_alpha = params->l1_alpha;
  f.conf_alpha = params->conf_alpha;
  f.grad_scale = grads ? grads->grad_scale : nullptr;
  f.ws = v;
  f.loss_num = out->loss_num;
  f.num_tokens = out->num_tokens;
  f.report = out->report;
  f.ce_rows = out->ce_rows;
  f.l1_rows = out->l1_rows;
  f.accept_rows = out->accept_rows;
  f.conf_rows = out->conf_rows;
  f.dconf = grads ? grads->dconf : nullptr;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_tp_finish(prob->logits_dtype == DSPARK_F32, a, s);
  if (e == cudaSuccess && grads && sh.has_markov)
    e = launch_markov_bwd_shard(heads_args(prob, params, v, grads), de_part, s);
  return cuda_status(e);
}

dspark_status_t dspark_tp_heads_bwd(const dspark_problem_t* prob, const dspark_params_t* params,
                                    const dspark_tp_t* tp, const float* de_all, const dspark_grads_t* grads,
                                    void* ws, size_t ws_bytes, dspark_stream_t stream) {
  Shape sh{};
  dspark_status_t st = check_tp(prob, params, tp, &sh);
  if (st != DSPARK_OK) return st;
  if ((st = check_ws(prob, ws, ws_bytes)) != DSPARK_OK) return st;
  if ((st = check_grads(prob, grads)) != DSPARK_OK) return st;
  if (sh.has_markov && (st = check_rec(de_all)) != DSPARK_OK) return st;
  if (!sh.has_markov && !sh.has_conf_head) return DSPARK_OK;  // no head: nothing to do
  const WsView v = ws_layout(ws, ws_dims(prob));
  return cuda_status(launch_heads_bwd_merge(heads_args(prob, params, v, grads), de_all, int(tp->tp_size),
                                            reinterpret_cast<cudaStream_t>(stream)));
}

dspark_status_t dspark_check_status(const void* ws, dspark_stream_t stream) {
  if (ws == nullptr) return DSPARK_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_status(e);
  uint32_t flags = 0;
  e = cudaMemcpy(&flags, ws, sizeof(flags), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_status(e);
  if (flags & kFlagIdOutOfRange) return DSPARK_ERR_ID_OUT_OF_RANGE;
  if (flags & kFlagTimeout) return DSPARK_ERR_DEVICE_TIMEOUT;
  return DSPARK_OK;
}

}  // extern "C"
