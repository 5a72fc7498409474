// Internal layout shared by the kernels and the C-ABI layer: workspace map, status
// bits, per-row statistic slots and the host-side launchers of each kernel family.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "dspark.h"

namespace dspark {

// Device-side error bits, OR-ed into the workspace status word.
enum : uint32_t {
  kFlagIdOutOfRange = 1u << 0,
  kFlagTimeout = 1u << 1,
};

// Per-row statistics saved by the forward (float slots of an 8-float record).
enum : int {
  kStLseD = 0,   // logsumexp of the (corrected) draft row
  kStLseT = 1,   // logsumexp of the teacher row
  kStCE = 2,     // cross-entropy
  kStL1 = 3,     // raw probability L1
  kStS = 4,      // sum_j p_j * sign(p_j - q_j)
  kStConf = 5,   // confidence logit c
  kStZT = 6,     // corrected draft logit at the target id
  kStDC = 7,     // dL/dc of the confidence logit
  kStride = 8,
};

// Header at the start of the workspace (256 bytes).
struct WsHeader {
  uint32_t status;      // device error bits
  int32_t n_sup;        // supervised rows
  int32_t n_zero;       // unsupervised rows
  int32_t pad0;
  int64_t num_tokens;   // == n_sup
  uint32_t done;        // cluster completion counter (reset by the last finisher)
  uint32_t pad1[57];
};
static_assert(sizeof(WsHeader) == 256, "header is one 256-byte line");

// Device pointers into the caller's workspace, carved by ws_layout().
struct WsView {
  WsHeader* hdr;
  uint8_t* m;          // [R] supervision mask (prefix * keep, id-checked)
  float* w;            // [R] loss weight m * exp(-k/gamma)
  int32_t* sup_list;   // [R] supervised rows in row order
  int32_t* zero_list;  // [R] unsupervised rows in row order
  int32_t* sup_index;  // [R] position of a row in sup_list, -1 if unsupervised
  int32_t* sup_tok;    // [R] target id of the i-th supervised row (bit 31: all-zero corrected row)
  float* sup_w;        // [R] loss weight of the i-th supervised row
  float* stats;        // [R][kStride]
  // Markov head (present when the problem has it)
  float* bias;         // [R][V] Markov bias rows W2.e (0 on invalid slots), compact by supervised position
  uint16_t* esup;      // [R][rank] bf16 Markov embeddings, compact (0 on invalid slots)
  uint16_t* eall;      // [R][rank] bf16 Markov embeddings by row (0 unless supervised+valid)
  float* dep;          // [splits][R][rank] split-K partials of dE
  float* de;           // [R][rank] dL/de
  // teacher from hidden states (present when the problem has it)
  uint16_t* hsup;      // [R][Ht] bf16 target hidden rows, compact by supervised position
  float* tchunk;       // [chunk][V] FP32 teacher rows of one chunk of supervised rows
  // confidence head (present when the problem has it)
  float* dpp;          // [ceil(R / kDprojRows)][conf_cols] partial sums of dL/dproj
  size_t bytes;        // total bytes used
};

constexpr size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// What a problem needs besides the per-row arrays.
struct WsDims {
  int64_t R = 0, V = 0, rank = 0, splits = 0;
  bool markov = false;
  int64_t Ht = 0, chunk = 0;  // teacher from hidden states: hidden size, rows per chunk
  bool lm = false;
  int64_t conf_cols = 0;      // confidence head: length of proj (0 without the head)
};

// Rows per partial sum of the confidence head's weight gradient.
constexpr int64_t kDprojRows = 16;

// Supervised rows per teacher chunk (the FP32 teacher rows of a chunk are the only
// vocabulary-wide teacher buffer; a multiple of the GEMM's 128-row tile).
constexpr int64_t kTeacherChunk = 512;
constexpr int64_t teacher_chunk_rows(int64_t R) { return R < kTeacherChunk ? R : kTeacherChunk; }

struct WsOffsets {
  size_t hdr, m, w, sup, zero, sidx, stok, sw, stats, z, esup, eall, dep, de, hsup, tchunk, dpp, bytes;
};

constexpr WsOffsets ws_offsets(const WsDims& d) {
  WsOffsets o{};
  size_t off = 0;
  const size_t R = size_t(d.R);
  o.hdr = off;
  off = align256(off + sizeof(WsHeader));
  o.m = off;
  off = align256(off + R);
  o.w = off;
  off = align256(off + sizeof(float) * R);
  o.sup = off;
  off = align256(off + sizeof(int32_t) * R);
  o.zero = off;
  off = align256(off + sizeof(int32_t) * R);
  o.sidx = off;
  off = align256(off + sizeof(int32_t) * R);
  o.stok = off;
  off = align256(off + sizeof(int32_t) * R);
  o.sw = off;
  off = align256(off + sizeof(float) * R);
  o.stats = off;
  off = align256(off + sizeof(float) * kStride * R);
  const size_t zr = d.markov ? R : 0, er = d.markov ? R * size_t(d.rank) : 0;
  o.z = off;
  off = align256(off + sizeof(float) * zr * size_t(d.V));
  o.esup = off;
  off = align256(off + 2 * er);
  o.eall = off;
  off = align256(off + 2 * er);
  o.dep = off;
  off = align256(off + sizeof(float) * er * size_t(d.markov ? d.splits : 0));
  o.de = off;
  off = align256(off + sizeof(float) * er);
  o.hsup = off;
  off = align256(off + (d.lm ? 2 * R * size_t(d.Ht) : 0));
  o.tchunk = off;
  off = align256(off + (d.lm ? sizeof(float) * size_t(d.chunk) * size_t(d.V) : 0));
  o.dpp = off;
  off = align256(off + sizeof(float) * size_t((d.R + kDprojRows - 1) / kDprojRows) * size_t(d.conf_cols));
  o.bytes = off;
  return o;
}

constexpr WsOffsets ws_offsets(int64_t R) {
  WsDims d{};
  d.R = R;
  return ws_offsets(d);
}

inline WsView ws_layout(void* base, const WsDims& d) {
  const WsOffsets o = ws_offsets(d);
  uint8_t* b = static_cast<uint8_t*>(base);
  WsView v{};
  v.hdr = reinterpret_cast<WsHeader*>(b + o.hdr);
  v.m = b + o.m;
  v.w = reinterpret_cast<float*>(b + o.w);
  v.sup_list = reinterpret_cast<int32_t*>(b + o.sup);
  v.zero_list = reinterpret_cast<int32_t*>(b + o.zero);
  v.sup_index = reinterpret_cast<int32_t*>(b + o.sidx);
  v.sup_tok = reinterpret_cast<int32_t*>(b + o.stok);
  v.sup_w = reinterpret_cast<float*>(b + o.sw);
  v.stats = reinterpret_cast<float*>(b + o.stats);
  v.bias = d.markov ? reinterpret_cast<float*>(b + o.z) : nullptr;
  v.esup = d.markov ? reinterpret_cast<uint16_t*>(b + o.esup) : nullptr;
  v.eall = d.markov ? reinterpret_cast<uint16_t*>(b + o.eall) : nullptr;
  v.dep = d.markov ? reinterpret_cast<float*>(b + o.dep) : nullptr;
  v.de = d.markov ? reinterpret_cast<float*>(b + o.de) : nullptr;
  v.hsup = d.lm ? reinterpret_cast<uint16_t*>(b + o.hsup) : nullptr;
  v.tchunk = d.lm ? reinterpret_cast<float*>(b + o.tchunk) : nullptr;
  v.dpp = d.conf_cols ? reinterpret_cast<float*>(b + o.dpp) : nullptr;
  v.bytes = o.bytes;
  return v;
}

inline WsView ws_layout(void* base, int64_t R) {
  WsDims d{};
  d.R = R;
  return ws_layout(base, d);
}

// ------------------------------------------------------------- kernel arguments
struct PrologueArgs {
  int64_t B, N, K, V, Vt;
  const uint8_t* eval_mask;
  const uint8_t* block_keep;
  const int64_t* target_ids;
  const int64_t* prev_ids;   // checked on valid rows when non-null
  const uint8_t* valid;
  int32_t invalid_zero;      // Markov head: an invalid slot's corrected row is all zero
  float gamma;
  int32_t gamma_enabled;
  WsView ws;
};

struct FinalizeArgs {
  int64_t B, N, K;
  const uint8_t* block_keep;
  const float* confidence_logits;  // given logits or null
  int32_t has_conf;                // a confidence source exists
  float ce_alpha, l1_alpha, conf_alpha;
  const float* grad_scale;
  WsView ws;
  // outputs
  float* loss_num;
  int64_t* num_tokens;
  float* report;
  float* ce_rows;
  float* l1_rows;
  float* accept_rows;
  float* conf_rows;
  float* dconf;
};

struct SweepArgs {
  const void* draft;
  int64_t ld_d;
  const void* target;        // null: CE only
  int64_t ld_t;
  void* dlogits;             // null: forward only
  int64_t ld_g;
  const int64_t* tids;
  const float* grad_scale;   // null: 1
  WsView ws;
  int64_t V;
  int32_t vvec;              // V / elements per 16-byte vector
  int32_t seg_vec;           // vectors per CTA segment
  int32_t nbuf;              // prefetch depth (1 or 2)
  const float* bias;         // Markov bias rows (compact by supervised position), or null
  int64_t ld_b;
  const uint8_t* valid;      // Markov valid-slot mask (with invalid_zero)
  int32_t invalid_zero;      // invalid slots get zero dlogits (all-zero corrected row)
  int32_t target_compact;    // teacher row of list position i is i - row0 (teacher chunk)
  int32_t row0, row1;        // supervised-list positions this launch covers
  int32_t do_zero;           // this launch also zero-fills the unsupervised rows' dlogits
  int32_t do_final;          // this launch ends with the per-row epilogue and report
  float ce_alpha, l1_alpha;
  FinalizeArgs fin;          // the per-row epilogue the last CTA runs
};



// Markov head and confidence head (inputs, weight gradients and workspace).
struct HeadsArgs {
  int64_t R, V, Vt, rank, H;
  const int64_t* prev_ids;
  const uint8_t* valid;
  const uint16_t* w1;        // bf16 [Vt][rank], null without the Markov head
  const uint16_t* w2;        // bf16 [V][rank]
  const uint16_t* hidden;    // bf16 [R][H], null without the confidence head
  const uint16_t* conf_w;    // bf16 [H (+ rank)]
  const float* conf_b;
  int32_t conf_with_markov;
  int32_t invalid_row_mode;
  const uint16_t* dlogits;   // bf16 [R][ld_g] (backward)
  int64_t ld_g;
  float* dw1;
  float* dw2;
  float* dconf_w;
  float* dconf_b;
  uint16_t* dhidden;         // bf16 [R][H]
  int32_t accumulate;
  WsView ws;
};

// K splits of the dE contraction (a fixed count for a given shape, so the workspace
// size does not depend on the device).
constexpr int kHeadsSlots = 148;
constexpr int heads_splits(int64_t R, int64_t V) {
  const int64_t m_tiles = (R + 127) / 128, kchunks = (V + 63) / 64;
  const int64_t s = kHeadsSlots / m_tiles;
  return int(s < 1 ? 1 : (s > kchunks ? kchunks : s));
}

// ------------------------------------------------------------------ launchers
cudaError_t launch_prologue(const PrologueArgs& a, cudaStream_t s);
// Row types of a sweep: draft / teacher / dlogits.
enum : int {
  kSweepBf16 = 0,  // bf16 / bf16 / bf16
  kSweepF32 = 1,   // f32 / f32 / f32
  kSweepZ32 = 2,   // bf16 + FP32 Markov bias rows / bf16 / bf16
  kSweepT32 = 3,   // bf16 / f32 teacher chunk (teacher from hidden states) / bf16
  kSweepZT32 = 4,  // bf16 + FP32 Markov bias rows / f32 teacher chunk / bf16
};
// False if V exceeds every build of that kind.
bool sweep_supported(int kind, int64_t V, bool has_target);

// `ctas` (if non-null) receives the number of CTAs the sweep launched.
cudaError_t launch_sweep(int kind, bool has_target, const SweepArgs& a, cudaStream_t s, int* ctas = nullptr);
// The unsupervised rows' zero dlogits, launched right behind a sweep that leaves them out
// (do_zero = 0) as its programmatic dependent: it runs on the SMs the sweep leaves idle
// (`sweep_ctas` of them taken) and finishes only after the sweep has.
cudaError_t launch_zero_rows(int kind, const SweepArgs& a, int sweep_ctas, cudaStream_t s);
cudaError_t launch_acceptance(int64_t B, int64_t N, int64_t K, const float* l1_rows,
                              const uint8_t* eval_mask, const uint8_t* block_keep,
                              float* accept_pair, float* tau_pair, float* accept_rows,
                              cudaStream_t s);
// dconf (if non-null) and the saved dL/dc of every row, for the given grad_scale
cudaError_t launch_conf_grad(int64_t R, const float* confidence_logits, float conf_alpha,
                             const float* grad_scale, const WsView& ws, float* dconf,
                             cudaStream_t s);
cudaError_t launch_bwd_stream(int kind, bool has_target, const SweepArgs& a, int64_t R, cudaStream_t s);
// Markov embeddings (both copies) and confidence logits
cudaError_t launch_heads_prep(const HeadsArgs& a, cudaStream_t s);
// Markov bias rows ws.bias = E.W2^T (compact, FP32; 0 on invalid slots) on the tensor cores
cudaError_t launch_markov_bias(const HeadsArgs& a, cudaStream_t s);
// dE, dW1, dW2, dconf_w, dconf_b, dhidden from dlogits and the saved dL/dc
cudaError_t launch_heads_bwd(const HeadsArgs& a, cudaStream_t s);
// Teacher from hidden states: gather of the supervised rows' hidden states, then the
// FP32 teacher rows of supervised-list positions [row0, row0 + chunk rows).
struct TeacherArgs {
  int64_t R, V, Ht;
  const uint16_t* hidden;    // bf16 [R][Ht]
  const uint16_t* lm_head;   // bf16 [V][Ht]
  const uint16_t* norm_w;    // bf16 [Ht] final RMS-norm weight, or null (already normed)
  float norm_eps;
  WsView ws;
};
cudaError_t launch_gather_hidden(const TeacherArgs& a, cudaStream_t s);
cudaError_t launch_teacher_chunk(const TeacherArgs& a, int64_t row0, cudaStream_t s);

}  // namespace dspark
