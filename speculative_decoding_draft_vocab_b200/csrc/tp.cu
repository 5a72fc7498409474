// Vocabulary-parallel DSpark loss: the row sweep split into three steps around two
// exchanges of per-row partials between tensor-parallel ranks.
//
// NeMo RL design doc "DSpark Auxiliary Heads", Tensor Parallelism: each rank holds the
// base logits of its own shard of the draft vocabulary.  Per row with draft z and
// teacher t (Megatron-Bridge API doc, bridge.training.post_training.dspark.loss,
// _chunk_terms and dspark_loss), in base 2 (x' = x log2 e):
//   step 1  (m, s) = (max_j x'_j, sum_j 2^(x'_j - m)) over the shard, for z and t;
//           the draft logit at the target id if the shard holds it
//   step 2  lse' = M + log2 sum_k s_k 2^(m_k - M) over the ranks' partials in rank
//           order (M = max_k m_k); over the shard L1 part = sum_j |p_j - q_j| and
//           S part = sum_j p_j sign(p_j - q_j), p = 2^(z' - lse'_z), q = 2^(t' - lse'_t)
//   step 3  L1, S = the parts summed in rank order; over the shard
//           dL/dz_j = g w [ce_alpha (p_j - [j = id]) + l1_alpha p_j (sign(p_j - q_j) - S)]
// With the Markov head the shard's corrected logits z = keep * base + bias are formed on
// chip from the base rows and the head's FP32 bias rows of the shard (keep = 0 only on an
// invalid slot whose corrected row is all zero; no gradient flows to its base row).
// An exact tie p_j == q_j counts as sign +1 in S and in dL/dz alike.  Each step is one
// pass over the shard's columns with one CTA per supervised row (the last CTA of step 3
// also writes the per-row epilogue and the report); a rank's shard of a
// micro-batch (rows x V / tp_size) is small enough to stay in L2 from one step to the
// next.  Every rank merges the same records in the same order, so all ranks hold
// bitwise the same row statistics.
#include <cuda_bf16.h>

#include "finalize.cuh"
#include "ptx.cuh"
#include "tp.cuh"

namespace dspark {
namespace {

constexpr int kTpThreads = 512;
constexpr int kTpWarps = kTpThreads / 32;

// One 16-byte vector of logits as floats (8 bf16 or 4 fp32).
template <typename T> struct Vec;
template <> struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  static __device__ __forceinline__ void load(const uint8_t* p, float* o) {
    const uint4 q = *reinterpret_cast<const uint4*>(p);
    o[0] = bf16lo(q.x); o[1] = bf16hi(q.x); o[2] = bf16lo(q.y); o[3] = bf16hi(q.y);
    o[4] = bf16lo(q.z); o[5] = bf16hi(q.z); o[6] = bf16lo(q.w); o[7] = bf16hi(q.w);
  }
  static __device__ __forceinline__ uint4 pack(const float* o) {
    return make_uint4(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]), pack_bf16(o[4], o[5]),
                      pack_bf16(o[6], o[7]));
  }
  static __device__ __forceinline__ float elem(const uint8_t* p) {
    return __uint_as_float(uint32_t(*reinterpret_cast<const uint16_t*>(p)) << 16);
  }
};
template <> struct Vec<float> {
  static constexpr int N = 4;
  static __device__ __forceinline__ void load(const uint8_t* p, float* o) {
    const float4 q = *reinterpret_cast<const float4*>(p);
    o[0] = q.x; o[1] = q.y; o[2] = q.z; o[3] = q.w;
  }
  static __device__ __forceinline__ uint4 pack(const float* o) {
    return make_uint4(__float_as_uint(o[0]), __float_as_uint(o[1]), __float_as_uint(o[2]),
                      __float_as_uint(o[3]));
  }
  static __device__ __forceinline__ float elem(const uint8_t* p) { return *reinterpret_cast<const float*>(p); }
};

// Adds one vector to a running base-2 logsumexp partial (m, s): the vector's maximum
// first (one rescale of s when it raises m), then its terms.
template <int N>
__device__ __forceinline__ void lse_add(float& m, float& s, const float* x) {
  float lm = x[0];
#pragma unroll
  for (int e = 1; e < N; ++e) lm = fmaxf(lm, x[e]);
  const float my = lm * kLog2e;
  if (my > m) {
    s = (m == -INFINITY) ? 0.f : s * ex2(m - my);
    m = my;
  }
  if (m != -INFINITY) {
#pragma unroll
    for (int e = 0; e < N; ++e) s += ex2(fmaf(x[e], kLog2e, -m));
  }
}

// (m, s) of a warp from its lanes' partials, in every lane.
__device__ __forceinline__ void warp_lse(float& m, float& s) {
  float M = m;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float t = (m == -INFINITY) ? 0.f : s * ex2(m - M);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
  m = M;
  s = t;
}

// Two (m, s) partials of the CTA (draft, teacher) merged in a fixed order; thread 0
// holds the result.  `sh` is 2 * kTpWarps float2 of shared memory.
__device__ __forceinline__ void block_lse2(float& m1, float& s1, float& m2, float& s2, float2* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  warp_lse(m1, s1);
  warp_lse(m2, s2);
  if (lane == 0) {
    sh[warp] = make_float2(m1, s1);
    sh[kTpWarps + warp] = make_float2(m2, s2);
  }
  __syncthreads();
  if (warp == 0) {
    const float2 a = lane < kTpWarps ? sh[lane] : make_float2(-INFINITY, 0.f);
    const float2 b = lane < kTpWarps ? sh[kTpWarps + lane] : make_float2(-INFINITY, 0.f);
    m1 = a.x, s1 = a.y, m2 = b.x, s2 = b.y;
    warp_lse(m1, s1);
    warp_lse(m2, s2);
  }
  __syncthreads();
}

// Two sums of the CTA in a fixed order; thread 0 holds them.
__device__ __forceinline__ void block_sum2(float& x, float& y, float2* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    x += __shfl_xor_sync(0xffffffffu, x, off);
    y += __shfl_xor_sync(0xffffffffu, y, off);
  }
  if (lane == 0) sh[warp] = make_float2(x, y);
  __syncthreads();
  if (warp == 0) {
    const float2 a = lane < kTpWarps ? sh[lane] : make_float2(0.f, 0.f);
    x = a.x, y = a.y;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      x += __shfl_xor_sync(0xffffffffu, x, off);
      y += __shfl_xor_sync(0xffffffffu, y, off);
    }
  }
  __syncthreads();
}

// z = keep * base + bias for one vector of the shard (bias rows are FP32, N per vector)
template <int N>
__device__ __forceinline__ void add_bias(float* x, const float* brow, int v, float keep) {
  const float4* b4 = reinterpret_cast<const float4*>(brow + size_t(v) * N);
#pragma unroll
  for (int q = 0; q < N / 4; ++q) {
    const float4 b = b4[q];
    x[4 * q + 0] = fmaf(x[4 * q + 0], keep, b.x);
    x[4 * q + 1] = fmaf(x[4 * q + 1], keep, b.y);
    x[4 * q + 2] = fmaf(x[4 * q + 2], keep, b.z);
    x[4 * q + 3] = fmaf(x[4 * q + 3], keep, b.w);
  }
}

template <typename T>
__device__ __forceinline__ const uint8_t* row_ptr(const void* base, int64_t row, int64_t ld) {
  return static_cast<const uint8_t*>(base) + size_t(row) * size_t(ld) * sizeof(T);
}

// The teacher row of a supervised row: the logits' own rows (type T, by row), or with TF
// the FP32 teacher rows computed from hidden states (compact by list position idx).
template <typename T, bool TF>
__device__ __forceinline__ const uint8_t* teacher_row(const TpArgs& a, int64_t row, int64_t idx) {
  if constexpr (TF) return row_ptr<float>(a.target, idx, a.ld_t);
  else return row_ptr<T>(a.target, row, a.ld_t);
}
// Vector v of a teacher row, as floats: the same columns as vector v of the draft row.
template <typename T, bool TF>
__device__ __forceinline__ void load_teacher(const uint8_t* tr, int v, float* y) {
  if constexpr (TF) {
    constexpr int N = Vec<T>::N;
#pragma unroll
    for (int q = 0; q < N / 4; ++q) Vec<float>::load(tr + (size_t(v) * N + 4 * q) * 4, y + 4 * q);
  } else {
    Vec<T>::load(tr + size_t(v) * 16, y);
  }
}

// ---------------------------------------------------------------- step 1
template <typename T, bool HAS_T, bool HAS_B, bool TF>
__global__ void __launch_bounds__(kTpThreads) tp_partials_kernel(const TpArgs a) {
  using VT = Vec<T>;
  __shared__ float2 sh[2 * kTpWarps];
  __shared__ int row_sup;
  const int nvec = int(a.V / VT::N);
  // own_rows: every row, supervised or not by the prologue's rule (prefix of eval_mask
  // within the block, block_keep, target id in range), decided here; otherwise the
  // prologue's list of supervised rows, complete past the dependency wait
  if (!a.own_rows) asm volatile("griddepcontrol.wait;" ::: "memory");
  // the next step may be scheduled now; it waits for this grid before reading anything
  asm volatile("griddepcontrol.launch_dependents;");
  const int n_rows = a.own_rows ? int(a.R) : a.ws.hdr->n_sup;
  for (int idx = blockIdx.x; idx < n_rows; idx += gridDim.x) {
    int64_t row;
    if (a.own_rows) {
      row = idx;
      if (threadIdx.x == 0) {
        const int64_t blk = row / a.K, k = row - blk * a.K;
        bool run = a.block_keep == nullptr || a.block_keep[blk] != 0;
        for (int64_t j = 0; j <= k; ++j) run &= a.eval_mask[blk * a.K + j] != 0;
        const int64_t t = a.tids[row];
        row_sup = run && t >= 0 && t < a.vocab_size;
      }
      __syncthreads();
      const bool sup = row_sup != 0;
      __syncthreads();  // read by every thread before thread 0 rewrites it
      if (!sup) continue;
    } else {
      row = a.ws.sup_list[idx];
    }
    const uint8_t* zr = row_ptr<T>(a.draft, row, a.ld_d);
    const uint8_t* tr = HAS_T ? teacher_row<T, TF>(a, row, idx) : nullptr;
    const float* br = HAS_B ? a.bias + size_t(idx) * size_t(a.V) : nullptr;
    const float keep = (HAS_B && a.ws.sup_tok[idx] < 0) ? 0.f : 1.f;
    float mz = -INFINITY, sz = 0.f, mt = -INFINITY, st = 0.f;
#pragma unroll 4
    for (int v = threadIdx.x; v < nvec; v += kTpThreads) {
      float x[VT::N];
      VT::load(zr + size_t(v) * 16, x);
      if constexpr (HAS_B) add_bias<VT::N>(x, br, v, keep);
      if constexpr (HAS_T) {
        float y[VT::N];
        load_teacher<T, TF>(tr, v, y);
        lse_add<VT::N>(mt, st, y);
      }
      lse_add<VT::N>(mz, sz, x);
    }
    block_lse2(mz, sz, mt, st, sh);
    if (threadIdx.x == 0) {
      const int64_t col = a.tids[row] - a.vocab_begin;
      float zt = 0.f;
      if (col >= 0 && col < a.V) {
        zt = VT::elem(zr + size_t(col) * sizeof(T));
        if constexpr (HAS_B) zt = fmaf(zt, keep, br[col]);
      }
      float4* rec = reinterpret_cast<float4*>(a.rec1 + size_t(row) * kTpRec1);
      rec[0] = make_float4(mz, sz, HAS_T ? mt : -INFINITY, HAS_T ? st : 0.f);
      rec[1] = make_float4(zt, 0.f, 0.f, 0.f);
    }
  }
  // what follows on the stream reads the prologue's lists: it must find the prologue
  // finished too
  if (a.own_rows) asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---------------------------------------------------------------- step 2
template <typename T, bool HAS_T, bool HAS_B, bool TF>
__global__ void __launch_bounds__(kTpThreads) tp_l1_kernel(const TpArgs a) {
  using VT = Vec<T>;
  __shared__ float2 sh[kTpWarps];
  __shared__ float2 lse2;  // the row's base-2 logsumexps, as every step uses them
  // launched behind the previous step (or the exchange): its results are visible past here
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  const int nvec = int(a.V / VT::N);
  const int n_sup = a.ws.hdr->n_sup;
  for (int idx = blockIdx.x; idx < n_sup; idx += gridDim.x) {
    const int64_t row = a.ws.sup_list[idx];
    if (threadIdx.x == 0) {
      float Mz = -INFINITY, Mt = -INFINITY;
      for (int k = 0; k < a.tp_size; ++k) {
        const float4 r = *reinterpret_cast<const float4*>(a.rec1_all + (size_t(k) * a.R + row) * kTpRec1);
        Mz = fmaxf(Mz, r.x);
        Mt = fmaxf(Mt, r.z);
      }
      float Sz = 0.f, St = 0.f, zt = 0.f;
      for (int k = 0; k < a.tp_size; ++k) {
        const float* r = a.rec1_all + (size_t(k) * a.R + row) * kTpRec1;
        if (r[0] != -INFINITY) Sz += r[1] * ex2(r[0] - Mz);
        if (HAS_T && r[2] != -INFINITY) St += r[3] * ex2(r[2] - Mt);
        zt += r[4];
      }
      // natural-log statistics as saved; steps 2 and 3 both work from these values
      const float lse_d = (Mz + log2f(Sz)) * kLn2;
      const float lse_t = HAS_T ? (Mt + log2f(St)) * kLn2 : 0.f;
      float* st = a.ws.stats + size_t(row) * kStride;
      st[kStLseD] = lse_d;
      st[kStLseT] = lse_t;
      st[kStZT] = zt;
      st[kStCE] = lse_d - zt;
      lse2 = make_float2(lse_d * kLog2e, lse_t * kLog2e);
    }
    __syncthreads();
    float l1 = 0.f, S = 0.f;
    if constexpr (HAS_T) {
      const float lz = lse2.x, lt = lse2.y;
      const uint8_t* zr = row_ptr<T>(a.draft, row, a.ld_d);
      const uint8_t* tr = teacher_row<T, TF>(a, row, idx);
      const float* br = HAS_B ? a.bias + size_t(idx) * size_t(a.V) : nullptr;
      const float keep = (HAS_B && a.ws.sup_tok[idx] < 0) ? 0.f : 1.f;
#pragma unroll 4
      for (int v = threadIdx.x; v < nvec; v += kTpThreads) {
        float x[VT::N], y[VT::N];
        VT::load(zr + size_t(v) * 16, x);
        if constexpr (HAS_B) add_bias<VT::N>(x, br, v, keep);
        load_teacher<T, TF>(tr, v, y);
#pragma unroll
        for (int e = 0; e < VT::N; ++e) {
          const float p = ex2(fmaf(x[e], kLog2e, -lz));
          const float d = p - ex2(fmaf(y[e], kLog2e, -lt));
          l1 += fabsf(d);
          S += copysignf(p, d);
        }
      }
      block_sum2(l1, S, sh);
    }
    if (threadIdx.x == 0)
      *reinterpret_cast<float4*>(a.rec2 + size_t(row) * kTpRec2) = make_float4(l1, S, 0.f, 0.f);
    __syncthreads();  // lse2 is rewritten for the next row
  }
}

// ---------------------------------------------------------------- step 3
template <typename T, bool HAS_T, bool HAS_B, bool TF>
__global__ void __launch_bounds__(kTpThreads) tp_finish_kernel(const TpArgs a) {
  using VT = Vec<T>;
  __shared__ float rowS;
  __shared__ int last;
  // the report's scratch: per-thread partials, one acceptance per thread, the totals
  __shared__ double scratch[(kNAcc + 1) * kTpThreads + kNAcc];
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int nvec = int(a.V / VT::N);
  const int n_sup = a.ws.hdr->n_sup;
  const int total = n_sup + (a.dlogits ? a.ws.hdr->n_zero : 0);
  for (int idx = blockIdx.x; idx < total; idx += gridDim.x) {
    if (idx >= n_sup) {  // unsupervised row: zero dlogits on the shard
      const int64_t row = a.ws.zero_list[idx - n_sup];
      uint8_t* out = static_cast<uint8_t*>(a.dlogits) + size_t(row) * size_t(a.ld_g) * sizeof(T);
      for (int v = threadIdx.x; v < nvec; v += kTpThreads)
        *reinterpret_cast<uint4*>(out + size_t(v) * 16) = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const int64_t row = a.ws.sup_list[idx];
    float* st = a.ws.stats + size_t(row) * kStride;
    if (threadIdx.x == 0) {
      float L1 = 0.f, S = 0.f;
      for (int k = 0; k < a.tp_size; ++k) {
        const float2 r = *reinterpret_cast<const float2*>(a.rec2_all + (size_t(k) * a.R + row) * kTpRec2);
        L1 += r.x;
        S += r.y;
      }
      st[kStL1] = L1;
      st[kStS] = S;
      rowS = S;
    }
    __syncthreads();
    if (a.dlogits) {
      const float S = rowS;
      const float g = a.grad_scale ? *a.grad_scale : 1.f;
      // an all-zero corrected row is a constant: nothing flows to its base row
      const bool zero_row = HAS_B && a.ws.sup_tok[idx] < 0;
      const float gw = zero_row ? 0.f : g * a.ws.w[row];
      const float cce = gw * a.ce_alpha, cl1 = gw * a.l1_alpha;
      const float kpos = cce + cl1 * (1.f - S), kneg = cce + cl1 * (-1.f - S);
      const float lz = st[kStLseD] * kLog2e, lt = st[kStLseT] * kLog2e;
      const int64_t col = a.tids[row] - a.vocab_begin;
      const uint8_t* zr = row_ptr<T>(a.draft, row, a.ld_d);
      const uint8_t* tr = HAS_T ? teacher_row<T, TF>(a, row, idx) : nullptr;
      const float* br = HAS_B ? a.bias + size_t(idx) * size_t(a.V) : nullptr;
      const float keep = zero_row ? 0.f : 1.f;
      uint8_t* out = static_cast<uint8_t*>(a.dlogits) + size_t(row) * size_t(a.ld_g) * sizeof(T);
#pragma unroll 4
      for (int v = threadIdx.x; v < nvec; v += kTpThreads) {
        float x[VT::N], o[VT::N];
        VT::load(zr + size_t(v) * 16, x);
        if constexpr (HAS_B) add_bias<VT::N>(x, br, v, keep);
        if constexpr (HAS_T) {
          float y[VT::N];
          load_teacher<T, TF>(tr, v, y);
#pragma unroll
          for (int e = 0; e < VT::N; ++e) {
            const float p = ex2(fmaf(x[e], kLog2e, -lz));
            const float d = p - ex2(fmaf(y[e], kLog2e, -lt));
            o[e] = p * (d >= 0.f ? kpos : kneg);
          }
        } else {
#pragma unroll
          for (int e = 0; e < VT::N; ++e) o[e] = ex2(fmaf(x[e], kLog2e, -lz)) * cce;
        }
        const int64_t c0 = int64_t(v) * VT::N;
        if (col >= c0 && col < c0 + VT::N) {
#pragma unroll
          for (int e = 0; e < VT::N; ++e)
            if (c0 + e == col) o[e] -= cce;
        }
        *reinterpret_cast<uint4*>(out + size_t(v) * 16) = VT::pack(o);
      }
    }
    __syncthreads();  // rowS is rewritten for the next row
  }
  // the last CTA to finish writes the per-row epilogue and the report
  if (threadIdx.x == 0) {
    __threadfence();
    last = atomicAdd(&a.ws.hdr->done, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (last) {
    __threadfence();
    if (a.fin.K <= kTpThreads) finalize_rows_smem(a.fin, scratch);
    else finalize_rows(a.fin, scratch);
    if (threadIdx.x == 0) a.ws.hdr->done = 0;
  }
}

unsigned tp_grid(int64_t rows) {
  return unsigned(rows < 1 ? 1 : (rows > 1184 ? 1184 : rows));  // 8 CTAs per SM at most
}

}  // namespace

cudaError_t launch_tp_partials(bool f32, const TpArgs& a, cudaStream_t s) {
  // programmatic dependent launch: scheduled while the mask prologue runs, waiting for
  // it (griddepcontrol.wait) before reading its lists
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tp_grid(a.R), 1, 1);
  cfg.blockDim = dim3(kTpThreads, 1, 1);
  cfg.stream = s;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  using bf16 = __nv_bfloat16;
  if (f32) {
    return a.target ? cudaLaunchKernelEx(&cfg, tp_partials_kernel<float, true, false, false>, a)
                    : cudaLaunchKernelEx(&cfg, tp_partials_kernel<float, false, false, false>, a);
  }
  if (a.t_compact) {  // the teacher from hidden states (bf16 logits)
    return a.bias ? cudaLaunchKernelEx(&cfg, tp_partials_kernel<bf16, true, true, true>, a)
                  : cudaLaunchKernelEx(&cfg, tp_partials_kernel<bf16, true, false, true>, a);
  }
  if (a.bias) {  // the Markov head needs bf16 logits
    return a.target ? cudaLaunchKernelEx(&cfg, tp_partials_kernel<bf16, true, true, false>, a)
                    : cudaLaunchKernelEx(&cfg, tp_partials_kernel<bf16, false, true, false>, a);
  }
  return a.target ? cudaLaunchKernelEx(&cfg, tp_partials_kernel<bf16, true, false, false>, a)
                  : cudaLaunchKernelEx(&cfg, tp_partials_kernel<bf16, false, false, false>, a);
}

// steps 2 and 3: programmatic dependent launches (scheduled early, waiting for the work
// before them on the stream before reading anything)
template <typename K>
cudaError_t launch_pdl(K kern, const TpArgs& a, cudaStream_t s) {
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tp_grid(a.R), 1, 1);
  cfg.blockDim = dim3(kTpThreads, 1, 1);
  cfg.stream = s;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  const cudaError_t err = cudaLaunchKernelEx(&cfg, kern, a);
  if (err != cudaSuccess) cudaGetLastError();
  return err;
}

cudaError_t launch_tp_l1(bool f32, const TpArgs& a, cudaStream_t s) {
  using bf16 = __nv_bfloat16;
  if (f32) return a.target ? launch_pdl(tp_l1_kernel<float, true, false, false>, a, s)
                           : launch_pdl(tp_l1_kernel<float, false, false, false>, a, s);
  if (a.t_compact) return a.bias ? launch_pdl(tp_l1_kernel<bf16, true, true, true>, a, s)
                                 : launch_pdl(tp_l1_kernel<bf16, true, false, true>, a, s);
  if (a.bias) return a.target ? launch_pdl(tp_l1_kernel<bf16, true, true, false>, a, s)
                              : launch_pdl(tp_l1_kernel<bf16, false, true, false>, a, s);
  return a.target ? launch_pdl(tp_l1_kernel<bf16, true, false, false>, a, s)
                  : launch_pdl(tp_l1_kernel<bf16, false, false, false>, a, s);
}

cudaError_t launch_tp_finish(bool f32, const TpArgs& a, cudaStream_t s) {
  using bf16 = __nv_bfloat16;
  if (f32) return a.target ? launch_pdl(tp_finish_kernel<float, true, false, false>, a, s)
                           : launch_pdl(tp_finish_kernel<float, false, false, false>, a, s);
  if (a.t_compact) return a.bias ? launch_pdl(tp_finish_kernel<bf16, true, true, true>, a, s)
                                 : launch_pdl(tp_finish_kernel<bf16, true, false, true>, a, s);
  if (a.bias) return a.target ? launch_pdl(tp_finish_kernel<bf16, true, true, false>, a, s)
                              : launch_pdl(tp_finish_kernel<bf16, false, true, false>, a, s);
  return a.target ? launch_pdl(tp_finish_kernel<bf16, true, false, false>, a, s)
                  : launch_pdl(tp_finish_kernel<bf16, false, false, false>, a, s);
}

}  // namespace dspark
