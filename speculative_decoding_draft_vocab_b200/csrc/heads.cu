// The two DSpark auxiliary heads (NeMo RL design doc "DSpark Auxiliary Heads"):
//   Markov head:      z = base + markov_w2 . e,  e = markov_w1[prev]   (valid slots;
//                     the bias rows are written here, the sweep adds the base rows)
//                     an invalid slot's corrected row is all zero (mode 0) or its base
//                     row (mode 1); prev ids are in the target vocabulary
//   confidence head:  c = proj . [h ; e] + bias on valid slots, 0 on invalid ones
// and their backward:
//   dE_r  = W2^T dz_r + dc_r proj_e,  dW2 = sum_r dz_r (x) e_r,  dW1[prev_r] += dE_r
//   dproj = sum_r dc_r [h_r ; e_r],  dbias = sum_r dc_r,  dh_r = dc_r proj_h
// (TorchSpec pull request #132, test list: the Markov bias is W2 applied to the W1 row
// of the previous token), and the teacher computed from the target's final hidden
// states, t = lm_head . h (TorchSpec pull request #132, scope list), one chunk of
// supervised rows at a time.  The contractions against the vocabulary (bias, teacher,
// dE, dW2) run on the tcgen05 GEMM; the rest are small row kernels.
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.cuh"
#include "tc_host.cuh"

namespace dspark {

namespace {

__device__ __forceinline__ float bf(uint16_t v) { return __uint_as_float(uint32_t(v) << 16); }

// ---- gather of the Markov embeddings and the confidence logits (one warp per row)
__global__ void __launch_bounds__(256) heads_prep_kernel(const HeadsArgs a) {
  const int warps = blockDim.x / 32;
  const int lane = threadIdx.x & 31;
  for (int64_t r = int64_t(blockIdx.x) * warps + threadIdx.x / 32; r < a.R; r += int64_t(gridDim.x) * warps) {
    const bool sup = a.ws.m[r] != 0;
    const bool valid = a.valid[r] != 0;
    const int64_t pv = a.prev_ids ? a.prev_ids[r] : -1;
    const bool has_e = a.w1 != nullptr && valid && pv >= 0 && pv < a.Vt;
    float edot = 0.f;
    if (a.w1 != nullptr) {
      const uint16_t* src = a.w1 + size_t(has_e ? pv : 0) * a.rank;
      uint16_t* dall = a.ws.eall + size_t(r) * a.rank;
      const int si = a.ws.sup_index[r];
      uint16_t* dsup = sup ? a.ws.esup + size_t(si) * a.rank : nullptr;
      for (int j = lane * 8; j < a.rank; j += 256) {  // 16-byte pieces
        uint4 q = has_e ? *reinterpret_cast<const uint4*>(src + j) : make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(dall + j) = (sup && has_e) ? q : make_uint4(0u, 0u, 0u, 0u);
        if (dsup) *reinterpret_cast<uint4*>(dsup + j) = q;
        if (a.conf_w != nullptr && a.conf_with_markov && has_e) {
          const uint16_t* e = reinterpret_cast<const uint16_t*>(&q);
          const uint16_t* pw = a.conf_w + a.H + j;
#pragma unroll
          for (int t = 0; t < 8; ++t) edot = fmaf(bf(e[t]), bf(pw[t]), edot);
        }
      }
    }
    if (a.conf_w != nullptr) {
      float hdot = 0.f;
      if (valid) {
        const uint16_t* h = a.hidden + size_t(r) * a.H;
#pragma unroll 4
        for (int j = lane * 8; j < a.H; j += 256) {
          const uint4 q = *reinterpret_cast<const uint4*>(h + j);
          const uint4 w = *reinterpret_cast<const uint4*>(a.conf_w + j);
          const uint16_t* hv = reinterpret_cast<const uint16_t*>(&q);
          const uint16_t* wv = reinterpret_cast<const uint16_t*>(&w);
#pragma unroll
          for (int t = 0; t < 8; ++t) hdot = fmaf(bf(hv[t]), bf(wv[t]), hdot);
        }
      }
      float c = hdot + edot;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
      if (lane == 0) a.ws.stats[r * kStride + kStConf] = valid ? c + *a.conf_b : 0.f;
    }
  }
}

// ---- epilogues (tensor stores of 32 x 32 blocks through the GEMM's TMA epilogue)
// bias GEMM: the Markov bias rows W2.e, compact by supervised position, 0 on invalid
// slots and past the last supervised row; the sweep adds them to the base rows.
struct BiasEpi {
  static constexpr bool kTma = true;
  const int32_t* sup_list;
  const WsHeader* hdr;
  const uint8_t* valid;
  __device__ float row_scale(int m) const {
    if (m >= hdr->n_sup) return 0.f;
    return valid[sup_list[m]] != 0 ? 1.f : 0.f;
  }
  __device__ int tma_mode() const { return 1; }
  __device__ void coords(int m0, int n0, int, int& x, int& y, int& z) const { x = n0, y = m0, z = -1; }
};

// dE GEMM: one partial per K split, [split][R][rank] (a 3-D output map)
struct PartialEpi {
  static constexpr bool kTma = true;
  __device__ float row_scale(int) const { return 1.f; }
  __device__ int tma_mode() const { return 1; }
  __device__ void coords(int m0, int n0, int split, int& x, int& y, int& z) const { x = n0, y = m0, z = split; }
};

// dW2 GEMM: [V][rank], stored, or added to what is there (tensor reduce-add)
struct WeightEpi {
  static constexpr bool kTma = true;
  int accumulate;
  __device__ float row_scale(int) const { return 1.f; }
  __device__ int tma_mode() const { return accumulate ? 2 : 1; }
  __device__ void coords(int m0, int n0, int, int& x, int& y, int& z) const { x = n0, y = m0, z = -1; }
};

// ---- dE = sum of the partials (+ dc proj_e), then dW1[prev] += dE.  The partials are
// [splits][R][rank]: the K splits of the dE GEMM, or the vocabulary-parallel ranks' parts
// in rank order.
__global__ void __launch_bounds__(256) de_reduce_kernel(const HeadsArgs a, const float* parts, const int splits) {
  const int64_t n = a.R * a.rank;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = i / a.rank, j = i - r * a.rank;
    const bool live = a.ws.m[r] != 0 && a.valid[r] != 0;
    float acc = 0.f;
    if (live) {
      const float* dp = parts + size_t(r) * a.rank + j;
      const size_t stride = size_t(a.R) * a.rank;
      float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;  // loads in flight together; fixed order
      int s = 0;
      for (; s + 4 <= splits; s += 4) {
        p0 += dp[s * stride];
        p1 += dp[(s + 1) * stride];
        p2 += dp[(s + 2) * stride];
        p3 += dp[(s + 3) * stride];
      }
      for (; s < splits; ++s) p0 += dp[s * stride];
      acc = (p0 + p1) + (p2 + p3);
      if (a.conf_w != nullptr && a.conf_with_markov)
        acc += a.ws.stats[r * kStride + kStDC] * bf(a.conf_w[a.H + j]);
      const int64_t pv = a.prev_ids[r];
      if (a.dw1 != nullptr) atomicAdd(a.dw1 + size_t(pv) * a.rank + j, acc);
    }
    a.ws.de[i] = acc;
  }
}

// ---- one vocabulary-parallel rank's part of dE: the K splits of its dE GEMM summed in
// the order de_reduce_kernel uses (0 on rows without a gradient)
__global__ void __launch_bounds__(256) de_split_sum_kernel(const HeadsArgs a, const int splits, float* out) {
  const int64_t n = a.R * a.rank;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = i / a.rank, j = i - r * a.rank;
    float acc = 0.f;
    if (a.ws.m[r] != 0 && a.valid[r] != 0) {
      const float* dp = a.ws.dep + size_t(r) * a.rank + j;
      const size_t stride = size_t(a.R) * a.rank;
      float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
      int s = 0;
      for (; s + 4 <= splits; s += 4) {
        p0 += dp[s * stride];
        p1 += dp[(s + 1) * stride];
        p2 += dp[(s + 2) * stride];
        p3 += dp[(s + 3) * stride];
      }
      for (; s < splits; ++s) p0 += dp[s * stride];
      acc = (p0 + p1) + (p2 + p3);
    }
    out[i] = acc;
  }
}

// ---- dproj = sum_r dc_r [h_r ; e_r] and dbias = sum_r dc_r: partial sums over blocks
// of kDprojRows rows (eight columns per thread, every row's loads in flight together),
// then the partials summed in a fixed order
__global__ void __launch_bounds__(256) dproj_part_kernel(const HeadsArgs a) {
  const int64_t cols = a.H + (a.conf_with_markov ? a.rank : 0);
  const int64_t c8 = 8 * (blockIdx.x * int64_t(blockDim.x) + threadIdx.x);  // first of 8 columns
  const int64_t r0 = int64_t(blockIdx.y) * kDprojRows;
  if (c8 >= cols) return;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int rr = 0; rr < kDprojRows; ++rr) {
    const int64_t r = r0 + rr;
    if (r >= a.R) break;  // the same r in every thread
    const bool live = a.ws.m[r] != 0 && a.valid[r] != 0;
    const float dc = live ? a.ws.stats[r * kStride + kStDC] : 0.f;
    const uint16_t* src = c8 < a.H ? a.hidden + size_t(r) * a.H + c8 : a.ws.eall + size_t(r) * a.rank + (c8 - a.H);
    const uint4 q = *reinterpret_cast<const uint4*>(src);
    const uint16_t* x = reinterpret_cast<const uint16_t*>(&q);
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = fmaf(dc, bf(x[k]), acc[k]);
  }
  float4* out = reinterpret_cast<float4*>(a.ws.dpp + size_t(blockIdx.y) * cols + c8);
  out[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  out[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

// 32 columns per block; 8 threads per column sum interleaved partials, combined in a
// fixed order in shared memory
__global__ void __launch_bounds__(256) dproj_final_kernel(const HeadsArgs a) {
  const int64_t cols = a.H + (a.conf_with_markov ? a.rank : 0);
  const int64_t nchunks = (a.R + kDprojRows - 1) / kDprojRows;
  const int cl = threadIdx.x & 31, part = threadIdx.x >> 5;
  const int64_t j = blockIdx.x * 32 + cl;
  __shared__ float sp[8][32];
  float acc = 0.f;
  if (j < cols)
    for (int64_t c = part; c < nchunks; c += 8) acc += a.ws.dpp[size_t(c) * cols + j];
  sp[part][cl] = acc;
  __syncthreads();
  if (part == 0 && j < cols) {
    float t = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) t += sp[k][cl];
    a.dconf_w[j] = a.accumulate ? a.dconf_w[j] + t : t;
  }
  if (blockIdx.x == 0) {
    __shared__ float pb[8];
    float b = 0.f;
    for (int64_t r = threadIdx.x; r < a.R; r += blockDim.x)
      if (a.ws.m[r] != 0 && a.valid[r] != 0) b += a.ws.stats[r * kStride + kStDC];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) b += __shfl_xor_sync(0xffffffffu, b, off);
    if ((threadIdx.x & 31) == 0) pb[threadIdx.x / 32] = b;
    __syncthreads();
    if (threadIdx.x == 0) {
      float t = 0.f;
      for (int i = 0; i < int(blockDim.x / 32); ++i) t += pb[i];
      if (a.dconf_b) *a.dconf_b = a.accumulate ? *a.dconf_b + t : t;
    }
  }
}

// ---- dh_r = dc_r proj_h on supervised valid rows, 0 elsewhere (bf16, eight per thread)
__global__ void __launch_bounds__(256) dhidden_kernel(const HeadsArgs a) {
  const int64_t n8 = a.R * a.H / 8;
  const int64_t h8 = a.H / 8;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n8; i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = i / h8, j8 = (i - r * h8) * 8;
    const bool live = a.ws.m[r] != 0 && a.valid[r] != 0;
    const float dc = live ? a.ws.stats[r * kStride + kStDC] : 0.f;
    const uint4 w = *reinterpret_cast<const uint4*>(a.conf_w + j8);
    const uint16_t* wv = reinterpret_cast<const uint16_t*>(&w);
    uint4 o;
    uint16_t* ov = reinterpret_cast<uint16_t*>(&o);
#pragma unroll
    for (int k = 0; k < 8; ++k) ov[k] = __bfloat16_as_ushort(__float2bfloat16_rn(dc * bf(wv[k])));
    *reinterpret_cast<uint4*>(a.dhidden + size_t(r) * a.H + j8) = o;
  }
}

// ---- teacher from hidden states: gather (with the target's final RMS norm when the
// states are pre-norm: y = w * x / sqrt(mean(x^2) + eps)), then t = lm_head . y per
// supervised row.  The norm runs in FP64 and its result goes to bf16 through FP32 (one
// rounding each), so the bf16 values do not depend on the order of the sum of squares.
__global__ void __launch_bounds__(256) gather_hidden_kernel(const TeacherArgs a) {
  const int warps = blockDim.x / 32;
  const int lane = threadIdx.x & 31;
  const int n_sup = a.ws.hdr->n_sup;
  for (int64_t si = int64_t(blockIdx.x) * warps + threadIdx.x / 32; si < n_sup; si += int64_t(gridDim.x) * warps) {
    const int64_t row = a.ws.sup_list[si];
    const uint4* src = reinterpret_cast<const uint4*>(a.hidden + size_t(row) * a.Ht);
    uint4* dst = reinterpret_cast<uint4*>(a.ws.hsup + size_t(si) * a.Ht);
    if (a.norm_w == nullptr) {
      for (int64_t j = lane; j < a.Ht / 8; j += 32) dst[j] = src[j];
      continue;
    }
    double ss = 0.0;
    for (int64_t j = lane; j < a.Ht / 8; j += 32) {
      const uint4 q = src[j];
      const uint16_t* x = reinterpret_cast<const uint16_t*>(&q);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const double v = double(bf(x[k]));
        ss = fma(v, v, ss);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const double rs = 1.0 / sqrt(ss / double(a.Ht) + double(a.norm_eps));
    const uint4* wv = reinterpret_cast<const uint4*>(a.norm_w);
    for (int64_t j = lane; j < a.Ht / 8; j += 32) {
      const uint4 q = src[j], wq = wv[j];
      const uint16_t* x = reinterpret_cast<const uint16_t*>(&q);
      const uint16_t* w = reinterpret_cast<const uint16_t*>(&wq);
      uint4 o;
      uint16_t* ov = reinterpret_cast<uint16_t*>(&o);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float y = __double2float_rn(double(bf(w[k])) * double(bf(x[k])) * rs);
        ov[k] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
      }
      dst[j] = o;
    }
  }
}

// teacher GEMM: FP32 teacher rows of the chunk, row i of the chunk being supervised-
// list position row0 + i (rows past the last supervised row are never read)
struct TeacherEpi {
  static constexpr bool kTma = true;
  __device__ float row_scale(int) const { return 1.f; }
  __device__ int tma_mode() const { return 1; }
  __device__ void coords(int m0, int n0, int, int& x, int& y, int& z) const { x = n0, y = m0, z = -1; }
};

inline int grid_for(int64_t n, int per_block) {
  const int64_t g = (n + per_block - 1) / per_block;
  return int(std::max<int64_t>(1, std::min<int64_t>(g, 4096)));
}

}  // namespace

cudaError_t launch_heads_prep(const HeadsArgs& a, cudaStream_t s) {
  heads_prep_kernel<<<grid_for(a.R, 8), 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_gather_hidden(const TeacherArgs& a, cudaStream_t s) {
  gather_hidden_kernel<<<grid_for(a.R, 8), 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_teacher_chunk(const TeacherArgs& a, int64_t row0, cudaStream_t s) {
  const int64_t rows = std::min<int64_t>(teacher_chunk_rows(a.R), a.R - row0);
  if (rows <= 0) return cudaSuccess;
  // A = the chunk's hidden rows [rows][Ht] (K-major), B = lm_head [V][Ht] (K-major)
  CUtensorMap ma, mb;
  if (!tc::make_map(&ma, a.ws.hsup + size_t(row0) * a.Ht, rows, a.Ht, a.Ht, 64, 128)) return cudaErrorInvalidValue;
  if (!tc::make_map(&mb, a.lm_head, a.V, a.Ht, a.Ht, 64, 256)) return cudaErrorInvalidValue;
  CUtensorMap mo;
  if (!tc::make_out_map(&mo, a.ws.tchunk, rows, a.V, a.V)) return cudaErrorInvalidValue;
  return tc::gemm<256, false, false, 4>(ma, mb, int(rows), int(a.V), int(a.Ht), 1, TeacherEpi{}, &a.ws.hdr->status,
                                        s, &a.ws.hdr->n_sup, int(row0), &mo);
}

cudaError_t launch_markov_bias(const HeadsArgs& a, cudaStream_t s) {
  CUtensorMap ma, mb;
  if (!tc::make_map(&ma, a.ws.esup, a.R, a.rank, a.rank, 64, 128)) return cudaErrorInvalidValue;
  if (!tc::make_map(&mb, a.w2, a.V, a.rank, a.rank, 64, 256)) return cudaErrorInvalidValue;
  CUtensorMap mo;
  if (!tc::make_out_map(&mo, a.ws.bias, a.R, a.V, a.V)) return cudaErrorInvalidValue;
  BiasEpi epi{a.ws.sup_list, a.ws.hdr, a.valid};
  return tc::gemm<256, false, false, 4>(ma, mb, int(a.R), int(a.V), int(a.rank), 1, epi, &a.ws.hdr->status, s,
                                        &a.ws.hdr->n_sup, 0, &mo);
}

namespace {

// dE split partials into ws.dep and dW2 (its rows of the vocabulary) from the bf16 dlogits
cudaError_t markov_grad_gemms(const HeadsArgs& a, int splits, cudaStream_t s) {
  // dE partials: A = dlogits [R][V] (K-major), B = W2 as [V][rank] (MN-major)
  CUtensorMap ma, mb;
  if (!tc::make_map(&ma, a.dlogits, a.R, a.V, a.ld_g, 64, 128)) return cudaErrorInvalidValue;
  if (!tc::make_map(&mb, a.w2, a.V, a.rank, a.rank, 64, 64)) return cudaErrorInvalidValue;
  CUtensorMap mo;
  if (!tc::make_out_map(&mo, a.ws.dep, a.R, a.rank, a.rank, splits, a.R * a.rank)) return cudaErrorInvalidValue;
  cudaError_t e = tc::gemm<256, false, true, 4>(ma, mb, int(a.R), int(a.rank), int(a.V), splits, PartialEpi{},
                                                &a.ws.hdr->status, s, nullptr, 0, &mo);
  if (e != cudaSuccess) return e;
  // dW2 = dlogits^T . E: A = dlogits as [R][V] (MN-major, M = vocabulary),
  // B = E by row [R][rank] (MN-major)
  if (a.dw2 != nullptr) {
    CUtensorMap ma2, mb2;
    if (!tc::make_map(&ma2, a.dlogits, a.R, a.V, a.ld_g, 64, 64)) return cudaErrorInvalidValue;
    if (!tc::make_map(&mb2, a.ws.eall, a.R, a.rank, a.rank, 64, 64)) return cudaErrorInvalidValue;
    CUtensorMap mo2;
    if (!tc::make_out_map(&mo2, a.dw2, a.V, a.rank, a.rank)) return cudaErrorInvalidValue;
    e = tc::gemm<256, true, true, 4>(ma2, mb2, int(a.V), int(a.rank), int(a.R), 1, WeightEpi{a.accumulate},
                                     &a.ws.hdr->status, s, nullptr, 0, &mo2);
  }
  return e;
}

// dE from its partials, dW1, then the confidence head's gradients
cudaError_t merge_and_conf_grads(const HeadsArgs& a, const float* parts, int nparts, cudaStream_t s) {
  cudaError_t e = cudaSuccess;
  if (a.w1 != nullptr) {
    de_reduce_kernel<<<grid_for(a.R * a.rank, 256), 256, 0, s>>>(a, parts, nparts);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (a.conf_w != nullptr) {
    const int64_t cols = a.H + (a.conf_with_markov ? a.rank : 0);
    if (a.dconf_w != nullptr) {
      const dim3 grid(unsigned((cols / 8 + 255) / 256), unsigned((a.R + kDprojRows - 1) / kDprojRows));
      dproj_part_kernel<<<grid, 256, 0, s>>>(a);
      dproj_final_kernel<<<unsigned((cols + 31) / 32), 256, 0, s>>>(a);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (a.dhidden != nullptr) {
      dhidden_kernel<<<grid_for(a.R * a.H / 8, 256), 256, 0, s>>>(a);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_heads_bwd(const HeadsArgs& a, cudaStream_t s) {
  const int splits = a.w1 != nullptr ? heads_splits(a.R, a.V) : 0;
  if (a.w1 != nullptr) {
    const cudaError_t e = markov_grad_gemms(a, splits, s);
    if (e != cudaSuccess) return e;
  }
  return merge_and_conf_grads(a, a.ws.dep, splits, s);
}

cudaError_t launch_markov_bwd_shard(const HeadsArgs& a, float* de_part, cudaStream_t s) {
  const int splits = heads_splits(a.R, a.V);
  const cudaError_t e = markov_grad_gemms(a, splits, s);
  if (e != cudaSuccess) return e;
  de_split_sum_kernel<<<grid_for(a.R * a.rank, 256), 256, 0, s>>>(a, splits, de_part);
  return cudaGetLastError();
}

cudaError_t launch_heads_bwd_merge(const HeadsArgs& a, const float* de_all, int nranks, cudaStream_t s) {
  return merge_and_conf_grads(a, de_all, nranks, s);
}

}  // namespace dspark
