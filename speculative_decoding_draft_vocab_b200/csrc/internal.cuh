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
  float* stats;        // [R][kStride]
  size_t bytes;        // total bytes used
};

constexpr size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct WsOffsets {
  size_t hdr, m, w, sup, zero, stats, bytes;
};

constexpr WsOffsets ws_offsets(int64_t R) {
  WsOffsets o{};
  size_t off = 0;
  o.hdr = off;
  off = align256(off + sizeof(WsHeader));
  o.m = off;
  off = align256(off + size_t(R));
  o.w = off;
  off = align256(off + sizeof(float) * size_t(R));
  o.sup = off;
  off = align256(off + sizeof(int32_t) * size_t(R));
  o.zero = off;
  off = align256(off + sizeof(int32_t) * size_t(R));
  o.stats = off;
  off = align256(off + sizeof(float) * kStride * size_t(R));
  o.bytes = off;
  return o;
}

inline WsView ws_layout(void* base, int64_t R) {
  const WsOffsets o = ws_offsets(R);
  uint8_t* b = static_cast<uint8_t*>(base);
  WsView v{};
  v.hdr = reinterpret_cast<WsHeader*>(b + o.hdr);
  v.m = b + o.m;
  v.w = reinterpret_cast<float*>(b + o.w);
  v.sup_list = reinterpret_cast<int32_t*>(b + o.sup);
  v.zero_list = reinterpret_cast<int32_t*>(b + o.zero);
  v.stats = reinterpret_cast<float*>(b + o.stats);
  v.bytes = o.bytes;
  return v;
}

// ------------------------------------------------------------- kernel arguments
struct PrologueArgs {
  int64_t B, N, K, V, Vt;
  const uint8_t* eval_mask;
  const uint8_t* block_keep;
  const int64_t* target_ids;
  const int64_t* prev_ids;   // checked on valid rows when non-null
  const uint8_t* valid;
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
  float ce_alpha, l1_alpha;
  FinalizeArgs fin;          // the per-row epilogue the last CTA runs
};



// ------------------------------------------------------------------ launchers
cudaError_t launch_prologue(const PrologueArgs& a, cudaStream_t s);
// Sweep config chosen for (dtype, V); returns false if V exceeds every build.
bool sweep_supported(int dtype, int64_t V, bool has_target);
cudaError_t launch_sweep(int dtype, bool has_target, const SweepArgs& a, cudaStream_t s);
cudaError_t launch_acceptance(int64_t B, int64_t N, int64_t K, const float* l1_rows,
                              const uint8_t* eval_mask, const uint8_t* block_keep,
                              float* accept_pair, float* tau_pair, float* accept_rows,
                              cudaStream_t s);
cudaError_t launch_conf_grad(int64_t R, const float* confidence_logits, float conf_alpha,
                             const float* grad_scale, const WsView& ws, float* dconf,
                             cudaStream_t s);
cudaError_t launch_bwd_stream(int dtype, bool has_target, const SweepArgs& a, int64_t R,
                              cudaStream_t s);

}  // namespace dspark
