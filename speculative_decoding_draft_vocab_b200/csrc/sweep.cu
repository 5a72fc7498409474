// Row sweep: fused DSpark forward + backward over full-vocabulary rows.
//
// One thread-block cluster owns one supervised row at a time.  Each CTA of the
// cluster owns a contiguous 16-byte-aligned segment of the vocabulary; the segment
// of the next rows is streamed into shared memory by 1-D bulk async copies (TMA,
// no multicast) while the current row is processed from registers, so every logit
// is read from HBM exactly once.  The exponentials are taken once per element and
// kept on chip for the rest of the row (the draft's in registers, the teacher's in
// tensor memory); the three row-wide reductions
// (logsumexp; L1 and S; nothing else) combine per-CTA partials through distributed
// shared memory, in the same fixed order in every CTA, so every CTA sees bitwise
// the same row scalars.  dlogits are written in the same sweep.
//
// Per row r with corrected draft z and teacher t (Megatron-Bridge API doc,
// bridge.training.post_training.dspark.loss, _chunk_terms / dspark_loss):
//   lse_d = log sum exp z,  lse_t = log sum exp t,  CE = lse_d - z[id]
//   p = exp(z - lse_d), q = exp(t - lse_t), L1 = sum |p - q| (raw), S = sum p*sign(p-q)
//   dL/dz_j = g*w*[ce_alpha*(p_j - [j = id]) + l1_alpha*p_j*(sign(p_j - q_j) - S)]
// Everything is computed in base 2: offsets are kept as x*log2(e).  Each logit costs
// one ex2 for the draft and one for the teacher.
#include <cuda_bf16.h>
#include <algorithm>
#include <mutex>

#include "finalize.cuh"
#include "internal.cuh"
#include "ptx.cuh"

namespace dspark {

template <typename T> struct VecTraits;
template <> struct VecTraits<float> { static constexpr int EPV = 4; };
template <> struct VecTraits<__nv_bfloat16> { static constexpr int EPV = 8; };

template <typename T> __device__ __forceinline__ void unpack16(const uint4 q, float* o);
template <> __device__ __forceinline__ void unpack16<float>(const uint4 q, float* o) {
  o[0] = __uint_as_float(q.x); o[1] = __uint_as_float(q.y);
  o[2] = __uint_as_float(q.z); o[3] = __uint_as_float(q.w);
}
template <> __device__ __forceinline__ void unpack16<__nv_bfloat16>(const uint4 q, float* o) {
  o[0] = bf16lo(q.x); o[1] = bf16hi(q.x); o[2] = bf16lo(q.y); o[3] = bf16hi(q.y);
  o[4] = bf16lo(q.z); o[5] = bf16hi(q.z); o[6] = bf16lo(q.w); o[7] = bf16hi(q.w);
}

template <typename T> __device__ __forceinline__ uint4 pack16(const float* o);
template <> __device__ __forceinline__ uint4 pack16<float>(const float* o) {
  return make_uint4(__float_as_uint(o[0]), __float_as_uint(o[1]), __float_as_uint(o[2]),
                    __float_as_uint(o[3]));
}
template <> __device__ __forceinline__ uint4 pack16<__nv_bfloat16>(const float* o) {
  return make_uint4(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]), pack_bf16(o[4], o[5]),
                    pack_bf16(o[6], o[7]));
}

template <typename T> __device__ __forceinline__ float load_elem(const uint8_t* p);
template <> __device__ __forceinline__ float load_elem<float>(const uint8_t* p) {
  return *reinterpret_cast<const float*>(p);
}
template <> __device__ __forceinline__ float load_elem<__nv_bfloat16>(const uint8_t* p) {
  return __uint_as_float(uint32_t(*reinterpret_cast<const uint16_t*>(p)) << 16);
}

// ------------------------------------------------------------ reductions
// Partial of a logsumexp in base 2: (m, s) with s = sum 2^(x - m); m = -inf is empty.
// Combining takes the maximum first and then one rescaled sum, so each thread
// spends one ex2 per reduction level group rather than one per pairwise merge.
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}
// (m, s) of every lane -> the warp's (M, S), identical in all lanes.
__device__ __forceinline__ void warp_lse_merge(float& m, float& s) {
  const float M = warp_max(m);
  const float t = (m == -INFINITY) ? 0.f : s * ex2(m - M);
  s = warp_sum(t);
  m = M;
}

// One group of EPV values (one 16-byte vector of the output type) in the row's own
// type: 16 bytes, or 32 bytes when FP32 rows meet a 16-bit output type.
template <typename TZ, int EPV>
__device__ __forceinline__ void load_group(const uint8_t* p, float* f) {
  if constexpr (sizeof(TZ) * EPV == 16) {
    unpack16<TZ>(*reinterpret_cast<const uint4*>(p), f);
  } else {
    unpack16<float>(*reinterpret_cast<const uint4*>(p), f);
    unpack16<float>(*reinterpret_cast<const uint4*>(p + 16), f + 4);
  }
}

// Warp maximum of an FP32 value (one instruction on sm_100a; -inf is the identity).
__device__ __forceinline__ float warp_max_f32(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// Control block in shared memory.  NP = cluster size x warps per CTA: every warp of
// every CTA of the cluster pushes its partial of a row reduction into every CTA.
template <int NP>
struct Ctrl {
  uint64_t mbar_data[2];  // row segment (draft + teacher) landed
  uint64_t mbar_ga;       // every warp's logsumexp partials landed
  uint64_t mbar_gb;       // every CTA's (L1, S) partials landed
  float4 ga[NP];          // (m_z, s_z, m_t, s_t) of warp w of rank i at [i * NW + w]
  float4 gb[16];          // (L1, S, 0, 0) of rank i
  float4 red[32];         // per-warp partials
  float4 bcast;           // row logsumexps (base 2)
  float ztid;             // raw draft logit at the target id (owner only)
  int last;               // this CTA finished last and writes the report
  uint32_t tmem;          // TMEM base address of the teacher's exponentials
  float pad;
  // ring of the cluster's upcoming rows: row id, target id, loss weight
  int32_t rrow[64];
  int32_t rtok[64];
  float rw[64];
};

// Bytes of Ctrl<NP> (only ga[] depends on NP)
constexpr size_t ctrl_bytes(int np) { return sizeof(Ctrl<1>) + size_t(np - 1) * sizeof(float4); }
static_assert(sizeof(Ctrl<64>) == ctrl_bytes(64) && sizeof(Ctrl<160>) == ctrl_bytes(160), "control block size");

constexpr int kRing = 64;       // ring entries
constexpr int kRingFill = 32;   // entries loaded at a time

// (m, s) partials of a base-2 logsumexp: the maximum first, then one rescaled sum.
__device__ __forceinline__ void lse_pair_merge(float& m1, float& s1, float& m2, float& s2) {
  const float M1 = warp_max_f32(m1), M2 = warp_max_f32(m2);
  float t1 = (m1 == -INFINITY) ? 0.f : s1 * ex2(m1 - M1);
  float t2 = (m2 == -INFINITY) ? 0.f : s2 * ex2(m2 - M2);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    t1 += __shfl_xor_sync(0xffffffffu, t1, off);
    t2 += __shfl_xor_sync(0xffffffffu, t2, off);
  }
  m1 = M1, s1 = t1, m2 = M2, s2 = t2;
}

// One cluster of CL CTAs owns one supervised row at a time; CTA `rank` owns the
// rank-th contiguous segment of the vocabulary.  Draft values live in registers
// (NV 16-byte vectors per thread, as FP32 exponentials); the teacher segment is read
// twice from shared memory in pass 1 (maximum, then exponentials), and its FP32
// exponentials wait in tensor memory (TMEM, staging only: no MMA) for pass 2, so each
// teacher value costs one ex2.  Shared memory holds one draft landing buffer and two
// teacher buffers: the next row's copy is issued as soon as the current draft segment
// is in registers, one full row ahead of its use.
// TZ is the draft logits' type; TT the teacher rows' type (the logits type, or FP32
// rows of the teacher computed from hidden states); TO the type of the dlogits.  With
// HAS_B (the Markov head) the corrected row z = keep * base + bias is formed on chip
// from the base row and the FP32 bias row of the head (compact by supervised
// position; keep = 0 only on an invalid slot whose corrected row is all zero, where
// the bias is 0 as well).  A launch covers the supervised rows of positions
// [row0, row1) in the supervised list.
// The row scalars come from a shared ring filled 32 rows ahead; the partials of the
// row logsumexps go from every warp straight to every CTA of the cluster.
template <typename TZ, typename TT, typename TO, int CL, int NT, int NV, bool HAS_T, bool HAS_B>
__global__ void __launch_bounds__(NT, 1) sweep_kernel(const SweepArgs a) {
  constexpr int EPV = VecTraits<TO>::EPV;
  constexpr int ZB = EPV * int(sizeof(TZ));  // bytes of one draft group
  constexpr int BB = HAS_B ? EPV * 4 : 0;    // bytes of one bias group
  constexpr int TB = EPV * int(sizeof(TT));  // bytes of one teacher group
  constexpr bool kMarkov = HAS_B;
  // FP32 teacher rows under 16-bit outputs only come from the teacher chunks (compact);
  // the other builds carry none of that code
  constexpr bool kTChunk = sizeof(TT) == 4 && sizeof(TO) == 2;
  constexpr int NE = NV * EPV;
  constexpr int NW = NT / 32;
  constexpr int NP = CL * NW;
  static_assert(NW <= 32 && CL <= 16, "control block sizes");
  static_assert(NE % 4 == 0, "whole groups of four elements");
  using CtrlT = Ctrl<NP>;
  // With a teacher, pass 1 keeps the teacher's exponentials in TMEM for pass 2: warp w
  // owns columns [(w / 4) * NE, (w / 4 + 1) * NE) of the 32 lanes of quarter w mod 4.
  constexpr uint32_t kTmCols = HAS_T ? tm::alloc_cols(uint32_t(NW / 4) * NE) : 0u;
  static_assert(!HAS_T || (NW % 4 == 0 && kTmCols <= 256), "TMEM columns of a teacher build");
  extern __shared__ __align__(128) uint8_t smem[];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = cluster_ctarank();
  const uint32_t cid = cluster_id_x();
  const uint32_t G = nclusters_x();
  const uint32_t seg_bytes = uint32_t(a.seg_vec) * uint32_t(TB);   // teacher segment
  const uint32_t zseg_bytes = uint32_t(a.seg_vec) * uint32_t(ZB);  // draft segment
  const uint32_t bseg_bytes = uint32_t(a.seg_vec) * uint32_t(BB);  // bias segment
  // buffers: HAS_T: [draft][bias][teacher 0][teacher 1]; else [draft 0][draft 1][bias 0][bias 1]
  CtrlT* ctrl = reinterpret_cast<CtrlT*>(smem + (HAS_T ? size_t(zseg_bytes) + bseg_bytes + 2 * size_t(seg_bytes)
                                                        : 2 * (size_t(zseg_bytes) + bseg_bytes)));
  auto zbuf = [&](int j) -> uint8_t* { return HAS_T ? smem : smem + size_t(j & 1) * zseg_bytes; };
  auto bbuf = [&](int j) -> uint8_t* {
    return HAS_T ? smem + zseg_bytes : smem + 2 * size_t(zseg_bytes) + size_t(j & 1) * bseg_bytes;
  };
  auto tbuf = [&](int j) -> uint8_t* {
    if constexpr (ZB == TB && BB == 0) return smem + size_t(1 + (j & 1)) * seg_bytes;  // zseg == seg
    else return smem + zseg_bytes + bseg_bytes + size_t(j & 1) * seg_bytes;
  };
  WsHeader* hdr = a.ws.hdr;

  const int v0 = int(rank) * a.seg_vec;
  const int nvec = max(0, min(a.seg_vec, a.vvec - v0));
  const uint32_t bytes = uint32_t(nvec) * uint32_t(TB);
  const uint32_t zbytes = uint32_t(nvec) * uint32_t(ZB);
  const uint32_t bbytes = uint32_t(nvec) * uint32_t(BB);
  const uint8_t* draft = static_cast<const uint8_t*>(a.draft);
  const uint8_t* target = static_cast<const uint8_t*>(a.target);
  const bool bwd = a.dlogits != nullptr;

  const uint32_t bar_d0 = smem_u32(&ctrl->mbar_data[0]);
  const uint32_t bar_d1 = smem_u32(&ctrl->mbar_data[1]);
  const uint32_t bar_ga = smem_u32(&ctrl->mbar_ga);
  const uint32_t bar_gb = smem_u32(&ctrl->mbar_gb);

  // thread 0: stream the segment of the row at list position sidx (draft, bias, teacher)
  auto issue = [&](int j, int64_t sidx, int64_t row) {
    const uint32_t bar = (j & 1) ? bar_d1 : bar_d0;
    const int64_t trow = (kTChunk && a.target_compact) ? sidx - a.row0 : row;  // teacher chunk
    mbar_arrive_expect_tx(bar, zbytes + bbytes + (HAS_T ? bytes : 0u));
    const uint64_t policy = l2_policy_evict_first();
    if (zbytes) {
      bulk_g2s(smem_u32(zbuf(j)), draft + (size_t(row) * a.ld_d + size_t(v0) * EPV) * sizeof(TZ),
               zbytes, bar, policy);
      if constexpr (HAS_B)  // the bias rows are compact by supervised position
        bulk_g2s(smem_u32(bbuf(j)), a.bias + (size_t(sidx) * a.ld_b + size_t(v0) * EPV),
                 bbytes, bar, policy);
      if constexpr (HAS_T)
        bulk_g2s(smem_u32(tbuf(j)), target + (size_t(trow) * a.ld_t + size_t(v0) * EPV) * sizeof(TT),
                 bytes, bar, policy);
    }
  };
  auto flag_timeout = [&]() { atomicOr(&hdr->status, kFlagTimeout); };

  if (tid == 0) {
    mbar_init(bar_d0, 1);
    mbar_init(bar_d1, 1);
    mbar_init(bar_ga, 1);
    mbar_init(bar_gb, 1);
    fence_mbar_init();
  }
  if constexpr (HAS_T) {
    if (warp == 0) {
      __syncwarp();
      tm::alloc(smem_u32(&ctrl->tmem), kTmCols);
    }
    tm::fence_before_sync();
  }
  // every CTA's barriers exist before any peer signals them
  __syncthreads();
  cluster_sync();
  uint32_t taddr = 0;  // this warp's first TMEM column
  if constexpr (HAS_T) {
    tm::fence_after_sync();
    taddr = ctrl->tmem + (uint32_t(32 * (warp & 3)) << 16) + uint32_t((warp >> 2) * NE);
  }
  // the mask prologue has finished and its writes are visible past this point
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // a programmatic dependent (the zero-row fill) may start once every CTA is here
  asm volatile("griddepcontrol.launch_dependents;");
  // this launch's supervised rows: list positions [row0, min(row1, n_sup))
  const int n_sup = max(0, min(hdr->n_sup, a.row1) - a.row0);
  const int my_n = (int(cid) < n_sup) ? (n_sup - 1 - int(cid)) / int(G) + 1 : 0;
  auto sidx_of = [&](int j) -> int64_t { return int64_t(a.row0) + cid + int64_t(j) * G; };

  // this cluster's share of zero rows: a slice per supervised row, stored by warps
  // 1 .. NW-1 while warp 0 merges the row's logsumexp partials; the id of the next
  // slice's first row is loaded a slice ahead
  const int n_zero = a.do_zero ? hdr->n_zero : 0;
  const int zfirst = ((int(cid) - n_sup) % int(G) + int(G)) % int(G);
  const int my_z = (bwd && zfirst < n_zero) ? (n_zero - 1 - zfirst) / int(G) + 1 : 0;
  const int ztot = my_z * nvec;
  const int zslice = my_n > 0 ? (ztot + my_n - 1) / my_n : ztot;
  auto zrow_id = [&](int rk) -> int32_t { return rk < my_z ? a.ws.zero_list[zfirst + size_t(rk) * G] : 0; };
  int32_t zr_pref = (my_z > 0 && warp != 0) ? zrow_id(0) : 0;
  auto write_zeros = [&](int q0, int q1) {
    if (warp == 0 || q0 >= q1) return;
    int rk = q0 / nvec;
    const int rk_end = (q1 - 1) / nvec;
    int32_t zr = zr_pref;
    for (; rk <= rk_end; ++rk) {
      const int32_t zr_next = zrow_id(rk + 1);  // in flight while this row is stored
      const int lo = max(q0 - rk * nvec, 0), hi = min(q1 - rk * nvec, nvec);
      uint8_t* base = static_cast<uint8_t*>(a.dlogits) + (size_t(zr) * a.ld_g + size_t(v0) * EPV) * sizeof(TO);
      for (int v = lo + tid - 32; v < hi; v += NT - 32)
        *reinterpret_cast<uint4*>(base + size_t(v) * 16) = make_uint4(0u, 0u, 0u, 0u);
      zr_pref = (hi == nvec) ? zr_next : zr;  // where the next slice starts
      zr = zr_next;
    }
  };

  // per-row scalars (row and target id fit 32 bits: R < 2^31, V <= 2^30) of the rows
  // j .. j + kRingFill - 1 in a shared ring, refilled kRingFill rows ahead
  // (the prologue wrote them compact by supervised position; with the Markov head bit 31
  // of the target id marks an all-zero corrected row)
  auto fill_ring = [&](int j0, int cnt) {
    if (tid < cnt && j0 + tid < my_n) {
      const int64_t si = sidx_of(j0 + tid);
      ctrl->rrow[(j0 + tid) % kRing] = a.ws.sup_list[si];
      ctrl->rtok[(j0 + tid) % kRing] = a.ws.sup_tok[si];
      ctrl->rw[(j0 + tid) % kRing] = a.ws.sup_w[si];
    }
  };
  fill_ring(0, kRing);
  __syncthreads();
  if (tid == 0) {
    if (my_n > 0) issue(0, sidx_of(0), ctrl->rrow[0]);
    if (!HAS_T && my_n > 1) issue(1, sidx_of(1), ctrl->rrow[1]);
  }

  for (int j = 0; j < my_n; ++j) {
    const uint32_t phase = uint32_t(j >> 1) & 1u;
    const uint32_t gphase = uint32_t(j) & 1u;
    const int32_t row = ctrl->rrow[j % kRing];
    const int32_t tokf = ctrl->rtok[j % kRing];
    const int32_t tok = tokf & 0x7fffffff;
    const bool zero_row = kMarkov && tokf < 0;  // corrected row all zero
    const int tv = tok / EPV - v0;  // target id's vector inside this segment
    const int te = tok % EPV;
    const uint8_t* zb = zbuf(j);
    const uint8_t* bb = bbuf(j);
    const uint8_t* tb = tbuf(j);
    if (!mbar_wait_bounded((j & 1) ? bar_d1 : bar_d0, phase) && tid == 0) flag_timeout();

    // ---- draft segment -> registers
    float xz[NE];
    const float keep = zero_row ? 0.f : 1.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int v = tid + i * NT;
      if (v < nvec) {
        load_group<TZ, EPV>(zb + size_t(v) * ZB, &xz[i * EPV]);
        if constexpr (HAS_B) {  // z = keep * base + bias
          float b8[EPV];
          load_group<float, EPV>(bb + size_t(v) * BB, b8);
#pragma unroll
          for (int e = 0; e < EPV; ++e) xz[i * EPV + e] = fmaf(xz[i * EPV + e], keep, b8[e]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < EPV; ++e) xz[i * EPV + e] = -INFINITY;
      }
    }
    if (tid == 0 && tv >= 0 && tv < nvec) {
      float zt = load_elem<TZ>(zb + size_t(tv) * ZB + size_t(te) * sizeof(TZ));
      if constexpr (HAS_B) zt = fmaf(zt, keep, load_elem<float>(bb + size_t(tv) * BB + size_t(te) * 4));
      ctrl->ztid = zt;
    }
    __syncthreads();  // the draft buffer is free again
    // rows j + kRingFill .. j + kRing - 1 into the half of the ring that row j is not in.
    // Only past this barrier: the slots hold rows j - kRingFill .. j - 1, and a warp still
    // in pass 3 of row j - 1 reads that row's weight (its entries are read from row
    // j + kRingFill on, many barriers later).
    if (j >= kRingFill && j % kRingFill == 0) fill_ring(j + kRingFill, kRingFill);
    if (tid == 0) {
      // HAS_T: draft buffer + the teacher buffer of row j-1 (its pass 2 is done).
      // Without a teacher the draft buffers alternate.
      if (HAS_T && j + 1 < my_n) issue(j + 1, sidx_of(j + 1), ctrl->rrow[(j + 1) % kRing]);
      if (!HAS_T && j + 2 < my_n) issue(j + 2, sidx_of(j + 2), ctrl->rrow[(j + 2) % kRing]);
    }

    // ---- pass 1: per-thread maxima, draft exponentials kept, sums (in this phase the
    // MUFU pipe, not the add chains, sets the pace)
    float mz = -INFINITY, mt = -INFINITY;
#pragma unroll
    for (int e = 0; e < NE; e += 2) mz = fmax3(mz, xz[e], xz[e + 1]);
    if constexpr (HAS_T && sizeof(TT) == 2) {  // bf16 pairs compared packed (exact)
      uint32_t mp = 0xff80ff80u;  // (-inf, -inf)
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int v = tid + i * NT;
        if (v < nvec) {
          const uint4 q = *reinterpret_cast<const uint4*>(tb + size_t(v) * TB);
          mp = bf2max(mp, bf2max(bf2max(q.x, q.y), bf2max(q.z, q.w)));
        }
      }
      mt = fmaxf(bf16lo(mp), bf16hi(mp));
    } else if constexpr (HAS_T) {
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int v = tid + i * NT;
        if (v < nvec) {
          float t8[EPV];
          load_group<TT, EPV>(tb + size_t(v) * TB, t8);
#pragma unroll
          for (int e = 0; e < EPV; e += 2) mt = fmax3(mt, t8[e], t8[e + 1]);
        }
      }
    }
    const float oz = (mz == -INFINITY) ? 0.f : mz * kLog2e;
    const float ot = (mt == -INFINITY) ? 0.f : mt * kLog2e;
    float sz = 0.f, st = 0.f;
#pragma unroll
    for (int e = 0; e < NE; ++e) {
      xz[e] = ex2(fmaf(xz[e], kLog2e, -oz));
      sz += xz[e];
    }
    if constexpr (HAS_T) {  // the teacher's exponentials, summed and kept in TMEM
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int v = tid + i * NT;
        float e8[EPV];
        if (v < nvec) {
          float t8[EPV];
          load_group<TT, EPV>(tb + size_t(v) * TB, t8);
#pragma unroll
          for (int e = 0; e < EPV; ++e) {
            e8[e] = ex2(fmaf(t8[e], kLog2e, -ot));
            st += e8[e];
          }
        } else {
#pragma unroll
          for (int e = 0; e < EPV; ++e) e8[e] = 0.f;
        }
        __syncwarp();
        tm::st<EPV>(taddr + uint32_t(i * EPV), e8);
      }
    }

    // ---- exchange A: every warp's (max, sum) pair into every CTA of the cluster
    {
      float m1 = (mz == -INFINITY) ? -INFINITY : oz, s1 = sz;
      float m2 = (mt == -INFINITY) ? -INFINITY : ot, s2 = st;
      lse_pair_merge(m1, s1, m2, s2);
      if (warp == 0 && lane == 0) mbar_arrive_expect_tx(bar_ga, NP * 16);
      if (lane < CL) {
        const uint32_t dst = dsmem_map(smem_u32(&ctrl->ga[int(rank) * NW + warp]), uint32_t(lane));
        st_async_f4(dst, make_float4(m1, s1, m2, s2), dsmem_map(bar_ga, uint32_t(lane)));
      }
    }
    write_zeros(j * zslice, min(ztot, (j + 1) * zslice));
    if (warp == 0) {
      if (!mbar_wait_bounded(bar_ga, gphase) && lane == 0) flag_timeout();
      // NP partials, in the same order in every CTA: the maxima first, then one
      // rescaled sum (lane l holds partials l, l + 32, ...; independent ex2s)
      constexpr int KP = (NP + 31) / 32;
      float4 q4[KP];
      float m1 = -INFINITY, m2 = -INFINITY;
#pragma unroll
      for (int kk = 0; kk < KP; ++kk) {
        const int k = lane + 32 * kk;
        q4[kk] = k < NP ? ctrl->ga[k] : make_float4(-INFINITY, 0.f, -INFINITY, 0.f);
        m1 = fmaxf(m1, q4[kk].x);
        m2 = fmaxf(m2, q4[kk].z);
      }
      m1 = warp_max_f32(m1);
      m2 = warp_max_f32(m2);
      float s1 = 0.f, s2 = 0.f;
#pragma unroll
      for (int kk = 0; kk < KP; ++kk) {
        s1 += q4[kk].x == -INFINITY ? 0.f : q4[kk].y * ex2(q4[kk].x - m1);
        s2 += q4[kk].z == -INFINITY ? 0.f : q4[kk].w * ex2(q4[kk].z - m2);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        s1 += __shfl_xor_sync(0xffffffffu, s1, off);
        s2 += __shfl_xor_sync(0xffffffffu, s2, off);
      }
      if (lane == 0) ctrl->bcast = make_float4(m1 + log2f(s1), HAS_T ? m2 + log2f(s2) : 0.f, 0.f, 0.f);
    }
    __syncthreads();
    const float4 lse4 = ctrl->bcast;
    const float lz2 = lse4.x;  // lse_d in base-2 units
    const float lt2 = lse4.y;
    const float az = (mz == -INFINITY) ? 0.f : ex2(oz - lz2);  // p = e * az
    const float at = (!HAS_T || mt == -INFINITY) ? 0.f : ex2(ot - lt2);

    // ---- pass 2: L1 and S.  q is formed from pass 1's own exponentials (read back
    // from TMEM) exactly as p is, so equal draft and teacher rows give p == q bit for
    // bit.  xz <- u = p * sign(p - q) (an exact tie takes the sub-gradient +p).
    float L1 = 0.f, S = 0.f;
    if constexpr (HAS_T) {
      tm::wait_st();
      float l4[4] = {0.f, 0.f, 0.f, 0.f}, s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int v = tid + i * NT;
        float e8[EPV];
        __syncwarp();
        tm::ld<EPV>(taddr + uint32_t(i * EPV), e8);
        if (v < nvec) {
#pragma unroll
          for (int e = 0; e < EPV; ++e) {
            const float q = __fmul_rn(e8[e], at);
            const float p = __fmul_rn(xz[i * EPV + e], az);
            const float d = __fsub_rn(p, q);
            const float u = copysignf(p, d);
            l4[e & 3] += fabsf(d);
            s4[e & 3] += u;
            xz[i * EPV + e] = u;
          }
        }
      }
      float l1p = (l4[0] + l4[1]) + (l4[2] + l4[3]);
      float sp = (s4[0] + s4[1]) + (s4[2] + s4[3]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        l1p += __shfl_xor_sync(0xffffffffu, l1p, off);
        sp += __shfl_xor_sync(0xffffffffu, sp, off);
      }
      if (lane == 0) ctrl->red[warp] = make_float4(l1p, sp, 0.f, 0.f);
      __syncthreads();
      if (warp == 0) {
        const float4 r4 = lane < NW ? ctrl->red[lane] : make_float4(0.f, 0.f, 0.f, 0.f);
        float x = r4.x, y = r4.y;
#pragma unroll
        for (int off = (NW & (NW - 1)) == 0 ? NW / 2 : 16; off > 0; off >>= 1) {  // NW partials in lanes 0 .. NW-1
          x += __shfl_xor_sync(0xffffffffu, x, off);
          y += __shfl_xor_sync(0xffffffffu, y, off);
        }
        if (lane == 0) mbar_arrive_expect_tx(bar_gb, CL * 16);
        __syncwarp();
        if (lane < CL) {
          const uint32_t dst = dsmem_map(smem_u32(&ctrl->gb[rank]), uint32_t(lane));
          st_async_f4(dst, make_float4(x, y, 0.f, 0.f), dsmem_map(bar_gb, uint32_t(lane)));
        }
      }
      if (!mbar_wait_bounded(bar_gb, gphase) && tid == 0) flag_timeout();
#pragma unroll
      for (int i = 0; i < CL; ++i) {  // same order in every CTA
        const float4 q4 = ctrl->gb[i];
        L1 += q4.x;
        S += q4.y;
      }
    }

    // ---- per-row statistics
    float* st_row = a.ws.stats + size_t(row) * kStride;
    if (tid == 0) {
      if (rank == 0) {
        st_row[kStLseD] = lz2 * kLn2;
        st_row[kStLseT] = lt2 * kLn2;
        st_row[kStL1] = L1;
        st_row[kStS] = S;
      }
      if (tv >= 0 && tv < nvec) {
        st_row[kStCE] = lz2 * kLn2 - ctrl->ztid;
        st_row[kStZT] = ctrl->ztid;
      }
    }

    // ---- pass 3: dlogits = p*(cce - cl1*S) + cl1*u, minus cce at the target id
    if (bwd) {
      // an invalid Markov slot's corrected row is a constant: nothing flows to base
      const bool zero_out = zero_row;
      const float g = a.grad_scale ? *a.grad_scale : 1.f;
      const float gw = zero_out ? 0.f : g * ctrl->rw[j % kRing];
      const float cce = gw * a.ce_alpha, cl1 = gw * a.l1_alpha;
      const float k0 = cce - cl1 * S;
      uint8_t* out = static_cast<uint8_t*>(a.dlogits) + (size_t(row) * a.ld_g + size_t(v0) * EPV) * sizeof(TO);
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int v = tid + i * NT;
        if (v < nvec) {
          float o[EPV];
#pragma unroll
          for (int e = 0; e < EPV; ++e) {
            if constexpr (HAS_T) o[e] = fmaf(xz[i * EPV + e], cl1, fabsf(xz[i * EPV + e]) * k0);
            else o[e] = (xz[i * EPV + e] * az) * cce;
          }
          if (v == tv) {
#pragma unroll
            for (int e = 0; e < EPV; ++e)
              if (e == te) o[e] -= cce;
          }
          *reinterpret_cast<uint4*>(out + size_t(v) * 16) = pack16<TO>(o);
        }
      }
    }
  }

  // ---- what is left of this cluster's zero rows (all of them if it had no row)
  write_zeros(my_n * zslice, ztot);
  if constexpr (HAS_T) tm::fence_before_sync();
  // no CTA leaves while a peer may still signal or read its shared memory
  __syncthreads();
  cluster_sync();
  if constexpr (HAS_T) {
    if (warp == 0) {  // every warp's TMEM reads completed before the barrier
      tm::fence_after_sync();
      __syncwarp();
      tm::dealloc(ctrl->tmem, kTmCols);
    }
  }

  // ---- the last CTA to finish writes the per-row epilogue and the report (in the
  // launch that covers the last rows)
  if (!a.do_final) return;
  if (tid == 0) {
    __threadfence();
    ctrl->last = atomicAdd(&hdr->done, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (ctrl->last) {
    __threadfence();
    if (a.fin.K <= NT) finalize_rows_smem(a.fin, reinterpret_cast<double*>(smem));
    else finalize_rows(a.fin, reinterpret_cast<double*>(smem));
    if (tid == 0) hdr->done = 0;
  }
}

// ------------------------------------------------------------------ host side
namespace {

constexpr size_t kMaxSmem = 227 * 1024;

struct LaunchCache {
  std::mutex mu;
  int dev = -1;
  size_t smem = 0;
  int clusters = 0;
};

// Dynamic shared memory of a build: the row buffers and the control block of CL CTAs x
// (NT / 32) warps.
template <typename TZ, typename TT, typename TO, int CL>
size_t smem_bytes(int64_t V, bool has_t, bool has_b, int nt) {
  constexpr int EPV = VecTraits<TO>::EPV;
  const int64_t vvec = V / EPV;
  const int64_t seg_vec = (vvec + CL - 1) / CL;
  const size_t zseg = size_t(seg_vec) * EPV * sizeof(TZ), tseg = size_t(seg_vec) * EPV * sizeof(TT);
  const size_t bseg = has_b ? size_t(seg_vec) * EPV * 4 : 0;
  return (has_t ? zseg + bseg + 2 * tseg : 2 * (zseg + bseg)) + ctrl_bytes(CL * (nt / 32));
}

template <typename TZ, typename TT, typename TO, int CL, int NT, int NV, bool HAS_T, bool HAS_B>
cudaError_t launch_cfg(const SweepArgs& a0, cudaStream_t s, int* ctas) {
  constexpr int EPV = VecTraits<TO>::EPV;
  SweepArgs a = a0;
  a.vvec = int32_t(a.V / EPV);
  a.seg_vec = (a.vvec + CL - 1) / CL;
  a.nbuf = 2;
  // at least the report's scratch (reused at the end)
  const size_t smem = std::max<size_t>(smem_bytes<TZ, TT, TO, CL>(a.V, HAS_T, HAS_B, NT),
                                       (size_t(kNAcc + 1) * NT + kNAcc) * sizeof(double));
  if (smem > kMaxSmem) return cudaErrorInvalidValue;

  auto kern = sweep_kernel<TZ, TT, TO, CL, NT, NV, HAS_T, HAS_B>;
  static LaunchCache cache;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = CL;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  int clusters = 0;
  {
    std::lock_guard<std::mutex> lk(cache.mu);
    if (cache.dev != dev || cache.smem != smem) {
      err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kMaxSmem));
      if (err != cudaSuccess) return err;
      if (CL > 8) {
        err = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (err != cudaSuccess) return err;
      }
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3(CL, 1, 1);
      q.blockDim = dim3(NT, 1, 1);
      q.dynamicSmemBytes = smem;
      q.attrs = at;
      q.numAttrs = 1;
      int n = 0;
      err = cudaOccupancyMaxActiveClusters(&n, kern, &q);
      if (err != cudaSuccess || n <= 0) {
        cudaGetLastError();
        int sms = 0;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        n = sms / CL > 0 ? sms / CL : 1;
      }
      cache.dev = dev;
      cache.smem = smem;
      cache.clusters = n;
    }
    clusters = cache.clusters;
  }
  // programmatic dependent launch: the grid is scheduled while the kernel before it
  // runs and waits for it (griddepcontrol.wait) before reading its results
  cudaLaunchAttribute at2[2];
  at2[0] = at[0];
  at2[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at2[1].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(clusters * CL), 1, 1);
  cfg.blockDim = dim3(NT, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = at2;
  cfg.numAttrs = 2;
  err = cudaLaunchKernelEx(&cfg, kern, a);
  if (err != cudaSuccess) cudaGetLastError();  // a refused launch leaves no error for later calls
  if (ctas) *ctas = clusters * CL;
  return err;
}

// Builds, smallest first.  A build covers rows of up to CL * NT * NV * (elements per
// 16-byte output vector) logits when its shared-memory buffers fit.
struct Build {
  int cl, nt, nv;
};
constexpr int kNumBuilds = 5;
// (5-CTA clusters of 640 threads for the recipe vocabulary: more SMs in use than 4-CTA
// clusters, which leave GPC remainders idle, and 5 warps per scheduler with 48 values per
// thread; measured 6 % faster than 4 x 512)
constexpr Build kBf16Builds[kNumBuilds] = {{1, 256, 1}, {2, 512, 2}, {4, 512, 4}, {5, 640, 6}, {8, 512, 5}};
constexpr Build kF32Builds[kNumBuilds] = {{1, 256, 1}, {2, 512, 2}, {4, 512, 8}, {8, 512, 10}, {16, 512, 5}};
// the heads' kinds (Markov bias rows, FP32 teacher chunks) with bf16 logits
constexpr Build kHeadBuilds[kNumBuilds] = {{1, 256, 1}, {2, 512, 2}, {4, 512, 4}, {8, 512, 5}, {16, 512, 3}};
// Markov bias rows and FP32 teacher chunks together: 10-CTA clusters fit the recipe
// vocabulary's buffers (measured 5 % faster than 16-CTA clusters on the whole call)
constexpr Build kTeacherBiasBuilds[kNumBuilds] = {{1, 256, 1}, {2, 512, 2}, {4, 512, 4}, {10, 512, 4}, {16, 512, 3}};

using bf16 = __nv_bfloat16;

template <typename TZ, typename TT, typename TO>
size_t smem_for(int cl, int nt, int64_t V, bool has_t, bool has_b) {
  switch (cl) {
    case 1: return smem_bytes<TZ, TT, TO, 1>(V, has_t, has_b, nt);
    case 2: return smem_bytes<TZ, TT, TO, 2>(V, has_t, has_b, nt);
    case 4: return smem_bytes<TZ, TT, TO, 4>(V, has_t, has_b, nt);
    case 5: return smem_bytes<TZ, TT, TO, 5>(V, has_t, has_b, nt);
    case 8: return smem_bytes<TZ, TT, TO, 8>(V, has_t, has_b, nt);
    case 10: return smem_bytes<TZ, TT, TO, 10>(V, has_t, has_b, nt);
    default: return smem_bytes<TZ, TT, TO, 16>(V, has_t, has_b, nt);
  }
}

size_t kind_smem(int kind, int cl, int nt, int64_t V, bool has_t) {
  switch (kind) {
    case kSweepBf16: return smem_for<bf16, bf16, bf16>(cl, nt, V, has_t, false);
    case kSweepF32: return smem_for<float, float, float>(cl, nt, V, has_t, false);
    case kSweepZ32: return smem_for<bf16, bf16, bf16>(cl, nt, V, has_t, true);
    case kSweepT32: return smem_for<bf16, float, bf16>(cl, nt, V, has_t, false);
    default: return smem_for<bf16, float, bf16>(cl, nt, V, has_t, true);
  }
}

int pick_build(int kind, int64_t V, bool has_t) {
  const Build* b = kind == kSweepBf16 ? kBf16Builds
                 : kind == kSweepF32 ? kF32Builds
                 : kind == kSweepZT32 ? kTeacherBiasBuilds : kHeadBuilds;
  const int epv = kind == kSweepF32 ? 4 : 8;
  for (int i = 0; i < kNumBuilds; ++i) {
    if (int64_t(b[i].cl) * b[i].nt * b[i].nv * epv < V) continue;
    if (kind_smem(kind, b[i].cl, b[i].nt, V, has_t) <= kMaxSmem) return i;
  }
  return -1;
}

template <typename TZ, typename TT, typename TO, bool HT, bool HB>
cudaError_t dispatch(int i, const SweepArgs& a, cudaStream_t s, int* ctas) {
  if constexpr (sizeof(TZ) == 4) {
    switch (i) {
      case 0: return launch_cfg<TZ, TT, TO, 1, 256, 1, HT, HB>(a, s, ctas);
      case 1: return launch_cfg<TZ, TT, TO, 2, 512, 2, HT, HB>(a, s, ctas);
      case 2: return launch_cfg<TZ, TT, TO, 4, 512, 8, HT, HB>(a, s, ctas);
      case 3: return launch_cfg<TZ, TT, TO, 8, 512, 10, HT, HB>(a, s, ctas);
      case 4: return launch_cfg<TZ, TT, TO, 16, 512, 5, HT, HB>(a, s, ctas);
    }
  } else if constexpr (sizeof(TT) == 2 && !HB) {
    switch (i) {
      case 0: return launch_cfg<TZ, TT, TO, 1, 256, 1, HT, HB>(a, s, ctas);
      case 1: return launch_cfg<TZ, TT, TO, 2, 512, 2, HT, HB>(a, s, ctas);
      case 2: return launch_cfg<TZ, TT, TO, 4, 512, 4, HT, HB>(a, s, ctas);
      case 3: return launch_cfg<TZ, TT, TO, 5, 640, 6, HT, HB>(a, s, ctas);
      case 4: return launch_cfg<TZ, TT, TO, 8, 512, 5, HT, HB>(a, s, ctas);
    }
  } else if constexpr (sizeof(TT) == 4 && HB) {  // kTeacherBiasBuilds
    switch (i) {
      case 0: return launch_cfg<TZ, TT, TO, 1, 256, 1, HT, HB>(a, s, ctas);
      case 1: return launch_cfg<TZ, TT, TO, 2, 512, 2, HT, HB>(a, s, ctas);
      case 2: return launch_cfg<TZ, TT, TO, 4, 512, 4, HT, HB>(a, s, ctas);
      case 3: return launch_cfg<TZ, TT, TO, 10, 512, 4, HT, HB>(a, s, ctas);
      case 4: return launch_cfg<TZ, TT, TO, 16, 512, 3, HT, HB>(a, s, ctas);
    }
  } else {  // kHeadBuilds
    switch (i) {
      case 0: return launch_cfg<TZ, TT, TO, 1, 256, 1, HT, HB>(a, s, ctas);
      case 1: return launch_cfg<TZ, TT, TO, 2, 512, 2, HT, HB>(a, s, ctas);
      case 2: return launch_cfg<TZ, TT, TO, 4, 512, 4, HT, HB>(a, s, ctas);
      case 3: return launch_cfg<TZ, TT, TO, 8, 512, 5, HT, HB>(a, s, ctas);
      case 4: return launch_cfg<TZ, TT, TO, 16, 512, 3, HT, HB>(a, s, ctas);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool sweep_supported(int kind, int64_t V, bool has_target) { return pick_build(kind, V, has_target) >= 0; }

cudaError_t launch_sweep(int kind, bool has_target, const SweepArgs& a, cudaStream_t s, int* ctas) {
  const int i = pick_build(kind, a.V, has_target);
  if (i < 0) return cudaErrorInvalidValue;
  switch (kind) {
    case kSweepBf16:
      return has_target ? dispatch<bf16, bf16, bf16, true, false>(i, a, s, ctas)
                        : dispatch<bf16, bf16, bf16, false, false>(i, a, s, ctas);
    case kSweepF32:
      return has_target ? dispatch<float, float, float, true, false>(i, a, s, ctas)
                        : dispatch<float, float, float, false, false>(i, a, s, ctas);
    case kSweepZ32:
      return has_target ? dispatch<bf16, bf16, bf16, true, true>(i, a, s, ctas)
                        : dispatch<bf16, bf16, bf16, false, true>(i, a, s, ctas);
    case kSweepT32:
      return dispatch<bf16, float, bf16, true, false>(i, a, s, ctas);
    case kSweepZT32:
      return dispatch<bf16, float, bf16, true, true>(i, a, s, ctas);
  }
  return cudaErrorInvalidValue;
}

// ------------------------------------------------------------ zero-row fill
// One CTA per unsupervised row at a time, 16-byte zero stores over the whole row.  It
// reads the prologue's list, complete before any sweep CTA passed its own dependency
// wait, which is where the sweep releases this grid; it waits for the sweep at its end.
constexpr int kZeroThreads = 1024;

__global__ void __launch_bounds__(kZeroThreads) zero_rows_kernel(const SweepArgs a, int vvec, int osize) {
  const int n_zero = a.ws.hdr->n_zero;
  for (int k = blockIdx.x; k < n_zero; k += gridDim.x) {
    uint8_t* out = static_cast<uint8_t*>(a.dlogits) + size_t(a.ws.zero_list[k]) * a.ld_g * size_t(osize);
    for (int v = threadIdx.x; v < vvec; v += kZeroThreads)
      *reinterpret_cast<uint4*>(out + size_t(v) * 16) = make_uint4(0u, 0u, 0u, 0u);
  }
  // whatever follows on the stream waits for this grid: it must find the sweep done too
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

cudaError_t launch_zero_rows(int kind, const SweepArgs& a, int sweep_ctas, cudaStream_t s) {
  const int osize = kind == kSweepF32 ? 4 : 2;
  const int vvec = int(a.V * osize / 16);
  int dev = 0, sms = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return err;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(std::max(sms - sweep_ctas, 8)), 1, 1);
  cfg.blockDim = dim3(kZeroThreads, 1, 1);
  cfg.stream = s;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  err = cudaLaunchKernelEx(&cfg, zero_rows_kernel, a, vvec, osize);
  if (err != cudaSuccess) cudaGetLastError();
  return err;
}

// ------------------------------------------------------- backward-only stream
// dlogits from saved row statistics: one more read of the logits, no reductions.  An
// exact tie p_j == q_j takes sign +1, the sub-gradient the forward's S counted.
// Covers the supervised rows of list positions [row0, row1) and, with do_zero, the
// unsupervised rows.
template <typename TZ, typename TT, typename TO, bool HAS_T, bool HAS_B>
__global__ void __launch_bounds__(256) bwd_stream_kernel(const SweepArgs a) {
  constexpr int EPV = VecTraits<TO>::EPV;
  constexpr int ZB = EPV * int(sizeof(TZ));
  constexpr int TB = EPV * int(sizeof(TT));
  constexpr bool kMarkov = HAS_B;
  constexpr bool kTChunk = sizeof(TT) == 4 && sizeof(TO) == 2;
  const int vvec = int(a.V / EPV);
  const int n_sup = max(0, min(a.ws.hdr->n_sup, a.row1) - a.row0);
  const int n_zero = a.do_zero ? a.ws.hdr->n_zero : 0;
  for (int idx = blockIdx.y; idx < n_sup + n_zero; idx += gridDim.y) {
    const bool unsup = idx >= n_sup;
    const int64_t sidx = int64_t(a.row0) + idx;
    const int64_t row = unsup ? a.ws.zero_list[idx - n_sup] : a.ws.sup_list[sidx];
    uint8_t* out = static_cast<uint8_t*>(a.dlogits) + size_t(row) * a.ld_g * sizeof(TO);
    const bool zero_row = unsup || (kMarkov && a.invalid_zero && a.valid[row] == 0);
    if (zero_row) {
      for (int v = blockIdx.x * blockDim.x + threadIdx.x; v < vvec; v += gridDim.x * blockDim.x)
        *reinterpret_cast<uint4*>(out + size_t(v) * 16) = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const float* st = a.ws.stats + size_t(row) * kStride;
    const float g = a.grad_scale ? *a.grad_scale : 1.f;
    const float gw = g * a.ws.w[row];
    const float cce = gw * a.ce_alpha, cl1 = gw * a.l1_alpha;
    const float S = st[kStS];
    const float kpos = cce + cl1 * (1.f - S), kneg = cce + cl1 * (-1.f - S);
    const float lz2 = st[kStLseD] * kLog2e, lt2 = st[kStLseT] * kLog2e;
    const int64_t tok = a.tids[row];
    const int64_t trow = (kTChunk && a.target_compact) ? int64_t(idx) : row;
    const uint8_t* zr = static_cast<const uint8_t*>(a.draft) + size_t(row) * a.ld_d * sizeof(TZ);
    const float* br = HAS_B ? a.bias + size_t(sidx) * a.ld_b : nullptr;
    const uint8_t* tr = static_cast<const uint8_t*>(a.target) + size_t(trow) * a.ld_t * sizeof(TT);
    for (int v = blockIdx.x * blockDim.x + threadIdx.x; v < vvec; v += gridDim.x * blockDim.x) {
      float z[EPV], t[EPV], o[EPV];
      load_group<TZ, EPV>(zr + size_t(v) * ZB, z);
      if constexpr (HAS_B) {  // a valid slot (the zero rows were handled above): z = base + bias
        float b8[EPV];
        load_group<float, EPV>(reinterpret_cast<const uint8_t*>(br + size_t(v) * EPV), b8);
#pragma unroll
        for (int e = 0; e < EPV; ++e) z[e] += b8[e];
      }
      if constexpr (HAS_T) load_group<TT, EPV>(tr + size_t(v) * TB, t);
#pragma unroll
      for (int e = 0; e < EPV; ++e) {
        const float p = ex2(fmaf(z[e], kLog2e, -lz2));
        if constexpr (HAS_T) {
          const float d = p - ex2(fmaf(t[e], kLog2e, -lt2));
          o[e] = p * (d >= 0.f ? kpos : kneg);
        } else {
          o[e] = p * cce;
        }
        if (int64_t(v) * EPV + e == tok) o[e] -= cce;
      }
      *reinterpret_cast<uint4*>(out + size_t(v) * 16) = pack16<TO>(o);
    }
  }
}

cudaError_t launch_bwd_stream(int kind, bool has_target, const SweepArgs& a, int64_t R, cudaStream_t s) {
  const int epv = kind == kSweepF32 ? 4 : 8;
  const int64_t vvec = a.V / epv;
  const unsigned gx = unsigned(std::min<int64_t>((vvec + 1023) / 1024, 64));
  dim3 grid(gx > 0 ? gx : 1, unsigned(std::max<int64_t>(1, std::min<int64_t>(R, 65535))), 1);
  switch (kind) {
    case kSweepBf16:
      if (has_target) bwd_stream_kernel<bf16, bf16, bf16, true, false><<<grid, 256, 0, s>>>(a);
      else bwd_stream_kernel<bf16, bf16, bf16, false, false><<<grid, 256, 0, s>>>(a);
      break;
    case kSweepF32:
      if (has_target) bwd_stream_kernel<float, float, float, true, false><<<grid, 256, 0, s>>>(a);
      else bwd_stream_kernel<float, float, float, false, false><<<grid, 256, 0, s>>>(a);
      break;
    case kSweepZ32:
      if (has_target) bwd_stream_kernel<bf16, bf16, bf16, true, true><<<grid, 256, 0, s>>>(a);
      else bwd_stream_kernel<bf16, bf16, bf16, false, true><<<grid, 256, 0, s>>>(a);
      break;
    case kSweepT32:
      bwd_stream_kernel<bf16, float, bf16, true, false><<<grid, 256, 0, s>>>(a);
      break;
    case kSweepZT32:
      bwd_stream_kernel<bf16, float, bf16, true, true><<<grid, 256, 0, s>>>(a);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace dspark
