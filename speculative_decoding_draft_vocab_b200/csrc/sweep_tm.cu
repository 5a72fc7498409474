// Row sweep with the teacher's exponentials held in tensor memory (TMEM), rows
// software-pipelined across the three passes: the fused DSpark forward + backward over
// bf16 draft and teacher rows.
//
// Per row r with draft z and teacher t (Megatron-Bridge API doc,
// bridge.training.post_training.dspark.loss, _chunk_terms / dspark_loss):
//   lse_d = log sum exp z,  lse_t = log sum exp t,  CE = lse_d - z[id]
//   p = exp(z - lse_d), q = exp(t - lse_t), L1 = sum |p - q| (raw), S = sum p*sign(p-q)
//   dL/dz_j = g*w*[ce_alpha*(p_j - [j = id]) + l1_alpha*p_j*(sign(p_j - q_j) - S)]
// computed in base 2 (offsets kept as x*log2(e)).
//
// Work split.  A thread-block cluster of CL CTAs owns one supervised row at a time; CTA
// `rank` owns the rank-th contiguous segment of the vocabulary.  Each CTA has NWC compute
// warps and one producer warp.  The producer streams the segment of every row into a
// ring of slabs in shared memory with 1-D bulk async copies (TMA, no multicast); slab i
// of a row holds the vectors tid + i*NTC of the segment, draft and teacher, so compute
// thread tid finds its i-th vector in slab i.  A compute thread owns NV 16-byte vectors
// (NE = 8*NV logits) of the row:
//   pass 1: the draft vectors become FP32 exponentials in registers, the teacher
//           vectors FP32 exponentials in TMEM (the thread's own TMEM lane, columns of
//           its warp), each logit read from shared memory once more for the second
//           read of the teacher (its maximum comes first); the slabs are then released;
//   pass 2: p and q from the registers and TMEM, L1 and S, and u = p*sign(p - q)
//           written back over q in TMEM;
//   pass 3: dlogits = p*(cce - cl1*S) + cl1*u, minus cce at the target id, from TMEM.
// The two row-wide reductions (the logsumexp partials after pass 1, the (L1, S)
// partials after pass 2) go from every warp straight into every CTA of the cluster
// (st.async with mbarrier complete_tx); every warp of every CTA merges all CL*NWC
// partials in the same fixed order, so the row scalars are bitwise the same everywhere.
// The passes of consecutive rows interleave: iteration j runs pass 1 of row j, pass 3
// of row j-1 (whose (L1, S) exchange was in flight during pass 1), then pass 2 of row j
// (whose logsumexp exchange was in flight during pass 3).  Both exchanges and the TMEM
// rows are double-buffered by row parity, and no CTA-wide barrier sits in the row loop.
#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>

#include "finalize.cuh"
#include "internal.cuh"
#include "ptx.cuh"

namespace dspark {

namespace {

// ------------------------------------------------------------------- TMEM
__device__ __forceinline__ void tm_alloc(uint32_t slot_saddr, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_saddr), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tm_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tm_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tm_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tm_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Eight consecutive FP32 columns of this thread's TMEM lane (warp-collective).
__device__ __forceinline__ void tm_st8(uint32_t taddr, const float* v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
               ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
                 "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
                 "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
               : "memory");
}
// Issues the load; the values are valid after tm_wait_ld8() on the same registers.
__device__ __forceinline__ void tm_ld8(uint32_t taddr, uint32_t* r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
}
// Waits for every TMEM load this thread issued; the registers are named as operands so
// no use of them is scheduled before the wait.
__device__ __forceinline__ void tm_wait_ld8(uint32_t* r) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7])
               :
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_local(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Store 8 bytes into (possibly another CTA's) shared memory, completion counted on the
// mbarrier at cluster address `bar` (same CTA as `addr`).
__device__ __forceinline__ void st_async_f2(uint32_t addr, float x, float y, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];"
               ::"r"(addr), "f"(x), "f"(y), "r"(bar) : "memory");
}

__device__ __forceinline__ float warp_max_f(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// Two base-2 logsumexp partials (m, s) of every lane -> the warp's, identical in all
// lanes (the maximum first, then one rescaled sum per lane).
__device__ __forceinline__ void lse2_warp(float& m1, float& s1, float& m2, float& s2) {
  const float M1 = warp_max_f(m1), M2 = warp_max_f(m2);
  float t1 = (m1 == -INFINITY) ? 0.f : s1 * ex2(m1 - M1);
  float t2 = (m2 == -INFINITY) ? 0.f : s2 * ex2(m2 - M2);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    t1 += __shfl_xor_sync(0xffffffffu, t1, off);
    t2 += __shfl_xor_sync(0xffffffffu, t2, off);
  }
  m1 = M1, s1 = t1, m2 = M2, s2 = t2;
}

constexpr uint32_t pow2_cols(int n) {
  uint32_t c = 32;
  while (c < uint32_t(n)) c <<= 1;
  return c;
}

constexpr int kMaxSlabs = 16;  // ring slots
// Registers per thread.  The register file is split over the SM's four schedulers
// (16384 registers each) and a CTA's warps are dealt round-robin to them, so a build with
// at most 13 warps (NWC <= 12 plus the producer) puts at most 4 warps on one scheduler:
// 4 x 32 x 128 = 16384.
constexpr int kTmRegs = 128;
constexpr int kRowRing = 32;   // row scalars in flight (> kMaxSlabs + 3 rows)

// Control block; NP = CL * NWC partials per exchange.
template <int NP>
struct CtrlTm {
  uint64_t full[kMaxSlabs];   // slab landed (producer arm + TMA bytes)
  uint64_t empty[kMaxSlabs];  // slab read by every compute warp
  uint64_t bar_a[2];          // logsumexp partials of every warp landed (row parity)
  uint64_t bar_b[2];          // (L1, S) partials of every warp landed (row parity)
  float4 ga[2][NP];           // (m_z, s_z, m_t, s_t) of warp w of rank i at [i * NWC + w]
  float2 gb[2][NP];           // (L1, S) of warp w of rank i
  int32_t rrow[kRowRing];     // row id, target id, loss weight of the cluster's j-th row
  int32_t rtok[kRowRing];
  float rw[kRowRing];
  uint32_t tmem_base;
  int last;
};

// TT: the teacher rows' type (bf16 logits, or FP32 rows of the teacher computed from
// hidden states, compact by supervised position); HAS_B: the Markov head's FP32 bias rows
// (compact by supervised position) are added to the base rows on chip, z = keep*base +
// bias, keep = 0 only on an invalid slot whose corrected row is all zero.
template <typename TT, bool HAS_B, int CL, int NWC, int NV>
__global__ void __maxnreg__(kTmRegs) sweep_tm_kernel(const SweepArgs a, const int S) {
  constexpr int EPV = 8;              // logits per 16-byte bf16 vector
  constexpr int BB = HAS_B ? 32 : 0;  // bytes of a vector's bias values
  constexpr int TB = EPV * int(sizeof(TT));  // bytes of a vector's teacher values
  constexpr bool kT32 = sizeof(TT) == 4;
  constexpr int NTC = NWC * 32;       // compute threads
  constexpr int NE = NV * EPV;        // logits per compute thread
  constexpr int NP = CL * NWC;
  constexpr int COLS = (NWC / 4) * NE;  // TMEM columns of one row (per lane quarter)
  constexpr uint32_t TCOLS = pow2_cols(2 * COLS);
  static_assert(NWC % 4 == 0 && 2 * COLS <= 512, "TMEM layout");
  static_assert(NWC + 1 <= 13, "at most 4 warps of kTmRegs registers per scheduler");
  using CtrlT = CtrlTm<NP>;
  extern __shared__ __align__(128) uint8_t smem[];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = cluster_ctarank();
  const uint32_t cid = cluster_id_x();
  const uint32_t G = nclusters_x();
  // slab: NTC draft vectors, NTC bias vectors (HAS_B), NTC teacher vectors
  const uint32_t slab_bytes = uint32_t(NTC) * uint32_t(16 + BB + TB);
  constexpr uint32_t kOffB = uint32_t(NTC) * 16u;
  constexpr uint32_t kOffT = uint32_t(NTC) * uint32_t(16 + BB);
  CtrlT* ctrl = reinterpret_cast<CtrlT*>(smem + size_t(S) * slab_bytes);
  WsHeader* hdr = a.ws.hdr;
  const int v0 = int(rank) * a.seg_vec;
  const int nvec = max(0, min(a.seg_vec, a.vvec - v0));
  const bool bwd = a.dlogits != nullptr;
  bool alive = true;  // false once a wait ran out: later waits are skipped
  auto wait = [&](uint32_t bar, uint32_t parity) {
    if (alive && !mbar_wait_bounded(bar, parity)) {
      alive = false;
      atomicOr(&hdr->status, kFlagTimeout);
    }
  };

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&ctrl->full[s]), 1);
      mbar_init(smem_u32(&ctrl->empty[s]), NWC);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&ctrl->bar_a[b]), 1);
      mbar_init(smem_u32(&ctrl->bar_b[b]), 1);
    }
    fence_mbar_init();
  }
  __syncwarp();  // warp 0 is whole again (thread 0 set the barriers up) for the aligned alloc
  if (warp == 0) tm_alloc(smem_u32(&ctrl->tmem_base), TCOLS);
  tm_fence_before();
  __syncthreads();
  tm_fence_after();
  const uint32_t tmem = ctrl->tmem_base;
  // every CTA's barriers exist before any peer signals them
  cluster_sync();
  // the mask prologue has finished and its writes are visible past this point
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int n_sup = max(0, min(hdr->n_sup, a.row1) - a.row0);
  const int my_n = (int(cid) < n_sup) ? (n_sup - 1 - int(cid)) / int(G) + 1 : 0;
  auto sidx_of = [&](int j) -> int64_t { return int64_t(a.row0) + cid + int64_t(j) * G; };

  if (warp == NWC) {
    // ------------------------------------------------------------ producer warp
    if (lane == 0) {
      const uint8_t* draft = static_cast<const uint8_t*>(a.draft);
      const uint8_t* target = static_cast<const uint8_t*>(a.target);
      const uint64_t policy = l2_policy_evict_first();
      int64_t g = 0;
      for (int j = 0; j < my_n; ++j) {
        const int64_t si = sidx_of(j);
        const int32_t row = a.ws.sup_list[si];
        ctrl->rrow[j % kRowRing] = row;
        ctrl->rtok[j % kRowRing] = a.ws.sup_tok[si];
        ctrl->rw[j % kRowRing] = a.ws.sup_w[si];
        // the teacher chunk's rows are compact by supervised position
        const int64_t trow = (kT32 && a.target_compact) ? si - a.row0 : row;
        const uint8_t* zr = draft + (size_t(row) * a.ld_d + size_t(v0) * EPV) * 2;
        const uint8_t* br = HAS_B ? reinterpret_cast<const uint8_t*>(a.bias + size_t(si) * a.ld_b + size_t(v0) * EPV)
                                  : nullptr;
        const uint8_t* tr = target + (size_t(trow) * a.ld_t + size_t(v0) * EPV) * sizeof(TT);
        for (int i = 0; i < NV; ++i, ++g) {
          const int slot = int(g % S);
          const uint32_t use = uint32_t(g / S);
          if (use > 0) wait(smem_u32(&ctrl->empty[slot]), (use - 1) & 1u);
          const int nv_i = max(0, min(NTC, nvec - i * NTC));
          const uint32_t full = smem_u32(&ctrl->full[slot]);
          // the arrive releases the row scalars written above to the compute warps
          mbar_arrive_expect_tx(full, uint32_t(nv_i) * uint32_t(16 + BB + TB));
          if (nv_i) {
            const uint32_t dst = smem_u32(smem + size_t(slot) * slab_bytes);
            bulk_g2s(dst, zr + size_t(i) * NTC * 16, uint32_t(nv_i) * 16u, full, policy);
            if constexpr (HAS_B)
              bulk_g2s(dst + kOffB, br + size_t(i) * NTC * BB, uint32_t(nv_i) * uint32_t(BB), full, policy);
            bulk_g2s(dst + kOffT, tr + size_t(i) * NTC * TB, uint32_t(nv_i) * uint32_t(TB), full, policy);
          }
        }
      }
      // every copy this thread issued has landed before the CTA moves on (a no-op unless
      // a wait ran out above): the latest use of each slot, each wait bounded again
      for (int slot = 0; slot < S && slot < g; ++slot) {
        const int64_t last_use = (g - 1 - slot) / S;
        if (!mbar_wait_bounded(smem_u32(&ctrl->full[slot]), uint32_t(last_use) & 1u)) {
          atomicOr(&hdr->status, kFlagTimeout);
          break;
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ compute warps
    const uint32_t t_addr0 = tmem + (uint32_t((warp & 3) * 32) << 16) + uint32_t((warp >> 2) * NE);
    auto taddr = [&](int parity, int e) -> uint32_t { return t_addr0 + uint32_t(parity * COLS + e); };
    const float g_scale = a.grad_scale ? *a.grad_scale : 1.f;

    // this cluster's share of zero rows: a slice per supervised row, written in pass 3
    const int n_zero = a.do_zero ? hdr->n_zero : 0;
    const int zfirst = ((int(cid) - n_sup) % int(G) + int(G)) % int(G);
    const int my_z = (bwd && zfirst < n_zero) ? (n_zero - 1 - zfirst) / int(G) + 1 : 0;
    const int ztot = my_z * nvec;
    const int zslice = my_n > 0 ? (ztot + my_n - 1) / my_n : ztot;
    auto write_zeros = [&](int q0, int q1) {
      if (q0 >= q1) return;
      for (int rk = q0 / nvec; rk <= (q1 - 1) / nvec; ++rk) {
        const int32_t zr = a.ws.zero_list[zfirst + size_t(rk) * G];
        const int lo = max(q0 - rk * nvec, 0), hi = min(q1 - rk * nvec, nvec);
        uint8_t* base = static_cast<uint8_t*>(a.dlogits) + (size_t(zr) * a.ld_g + size_t(v0) * EPV) * 2;
        for (int v = lo + tid; v < hi; v += NTC)
          *reinterpret_cast<uint4*>(base + size_t(v) * 16) = make_uint4(0u, 0u, 0u, 0u);
      }
    };

    float xz[NE];
    float zt = 0.f;  // raw draft logit at the target id (its owner only)
    int64_t g = 0;   // slabs consumed
    for (int j = 0; j <= my_n; ++j) {
      const bool cur = j < my_n;
      const int par = j & 1;
      // ======================================================== pass 1 of row j
      float oz = 0.f, ot = 0.f, sz = 0.f, st = 0.f;
      bool hz = false, ht = false;
      int32_t tok = 0;
      if (cur) {
        const int64_t g0 = g;
        uint32_t tmax2 = 0xff80ff80u;  // two bf16 -inf (bf16 teacher)
        float mt32 = -INFINITY;        // FP32 teacher
        float mz = -INFINITY;
        float keep = 1.f;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
          const int slot = int((g0 + i) % S);
          wait(smem_u32(&ctrl->full[slot]), uint32_t((g0 + i) / S) & 1u);
          if (i == 0) {
            const int32_t tokf = ctrl->rtok[j % kRowRing];
            tok = tokf & 0x7fffffff;
            if (HAS_B && tokf < 0) keep = 0.f;  // the corrected row is all zero
          }
          const int v = tid + i * NTC;
          const uint8_t* sb = smem + size_t(slot) * slab_bytes;
          if (v < nvec) {
            const uint4 qz = *reinterpret_cast<const uint4*>(sb + size_t(tid) * 16);
            float x[EPV];
            x[0] = bf16lo(qz.x); x[1] = bf16hi(qz.x); x[2] = bf16lo(qz.y); x[3] = bf16hi(qz.y);
            x[4] = bf16lo(qz.z); x[5] = bf16hi(qz.z); x[6] = bf16lo(qz.w); x[7] = bf16hi(qz.w);
            if constexpr (HAS_B) {  // z = keep * base + bias
              const uint4 b0 = *reinterpret_cast<const uint4*>(sb + kOffB + size_t(tid) * 32);
              const uint4 b1 = *reinterpret_cast<const uint4*>(sb + kOffB + size_t(tid) * 32 + 16);
              x[0] = fmaf(x[0], keep, __uint_as_float(b0.x)); x[1] = fmaf(x[1], keep, __uint_as_float(b0.y));
              x[2] = fmaf(x[2], keep, __uint_as_float(b0.z)); x[3] = fmaf(x[3], keep, __uint_as_float(b0.w));
              x[4] = fmaf(x[4], keep, __uint_as_float(b1.x)); x[5] = fmaf(x[5], keep, __uint_as_float(b1.y));
              x[6] = fmaf(x[6], keep, __uint_as_float(b1.z)); x[7] = fmaf(x[7], keep, __uint_as_float(b1.w));
            }
            mz = fmax3(mz, fmax3(x[0], x[1], x[2]), fmax3(x[3], x[4], x[5]));
            mz = fmax3(mz, x[6], x[7]);
            if constexpr (kT32) {
              const uint4 t0 = *reinterpret_cast<const uint4*>(sb + kOffT + size_t(tid) * 32);
              const uint4 t1 = *reinterpret_cast<const uint4*>(sb + kOffT + size_t(tid) * 32 + 16);
              mt32 = fmax3(mt32, fmax3(__uint_as_float(t0.x), __uint_as_float(t0.y), __uint_as_float(t0.z)),
                           fmax3(__uint_as_float(t0.w), __uint_as_float(t1.x), __uint_as_float(t1.y)));
              mt32 = fmax3(mt32, __uint_as_float(t1.z), __uint_as_float(t1.w));
            } else {
              const uint4 qt = *reinterpret_cast<const uint4*>(sb + kOffT + size_t(tid) * 16);
              tmax2 = bf2max(bf2max(tmax2, bf2max(qt.x, qt.y)), bf2max(qt.z, qt.w));
            }
#pragma unroll
            for (int e = 0; e < EPV; ++e) xz[i * EPV + e] = x[e];
            if (v == tok / EPV - v0) {  // one thread of the cluster holds the target id
              const int te = tok % EPV;
#pragma unroll
              for (int e = 0; e < EPV; ++e)
                if (e == te) zt = x[e];
            }
          } else {
#pragma unroll
            for (int e = 0; e < EPV; ++e) xz[i * EPV + e] = -INFINITY;
          }
        }
        const float mt = kT32 ? mt32 : fmaxf(bf16lo(tmax2), bf16hi(tmax2));
        hz = mz != -INFINITY;
        ht = mt != -INFINITY;
        oz = hz ? mz * kLog2e : 0.f;
        ot = ht ? mt * kLog2e : 0.f;
#pragma unroll
        for (int e = 0; e < NE; ++e) {
          xz[e] = ex2(fmaf(xz[e], kLog2e, -oz));
          sz += xz[e];
        }
        // the teacher's second read: exponentials into TMEM, then the slab is free
#pragma unroll
        for (int i = 0; i < NV; ++i) {
          const int slot = int((g0 + i) % S);
          const int v = tid + i * NTC;
          float et[EPV];
          if (v < nvec) {
            const uint8_t* tp = smem + size_t(slot) * slab_bytes + kOffT + size_t(tid) * TB;
            if constexpr (kT32) {
              const uint4 t0 = *reinterpret_cast<const uint4*>(tp);
              const uint4 t1 = *reinterpret_cast<const uint4*>(tp + 16);
              et[0] = __uint_as_float(t0.x); et[1] = __uint_as_float(t0.y); et[2] = __uint_as_float(t0.z);
              et[3] = __uint_as_float(t0.w); et[4] = __uint_as_float(t1.x); et[5] = __uint_as_float(t1.y);
              et[6] = __uint_as_float(t1.z); et[7] = __uint_as_float(t1.w);
            } else {
              const uint4 qt = *reinterpret_cast<const uint4*>(tp);
              et[0] = bf16lo(qt.x); et[1] = bf16hi(qt.x); et[2] = bf16lo(qt.y); et[3] = bf16hi(qt.y);
              et[4] = bf16lo(qt.z); et[5] = bf16hi(qt.z); et[6] = bf16lo(qt.w); et[7] = bf16hi(qt.w);
            }
#pragma unroll
            for (int e = 0; e < EPV; ++e) {
              et[e] = ex2(fmaf(et[e], kLog2e, -ot));
              st += et[e];
            }
          } else {
#pragma unroll
            for (int e = 0; e < EPV; ++e) et[e] = 0.f;
          }
          __syncwarp();  // the TMEM store is warp-collective
          tm_st8(taddr(par, i * EPV), et);
          __syncwarp();
          if (lane == 0) mbar_arrive_local(smem_u32(&ctrl->empty[slot]));
        }
        g = g0 + NV;
        // exchange A: this warp's (max, sum) pairs into every CTA of the cluster
        float m1 = hz ? oz : -INFINITY, s1 = sz, m2 = ht ? ot : -INFINITY, s2 = st;
        lse2_warp(m1, s1, m2, s2);
        const uint32_t bar = smem_u32(&ctrl->bar_a[par]);
        if (warp == 0 && lane == 0) mbar_arrive_expect_tx(bar, NP * 16);
        __syncwarp();
        if (lane < CL)
          st_async_f4(dsmem_map(smem_u32(&ctrl->ga[par][int(rank) * NWC + warp]), uint32_t(lane)),
                      make_float4(m1, s1, m2, s2), dsmem_map(bar, uint32_t(lane)));
      }
      // ======================================================== pass 3 of row j-1
      if (j > 0) {
        const int pp = par ^ 1;
        const int jr = (j - 1) % kRowRing;
        wait(smem_u32(&ctrl->bar_b[pp]), uint32_t((j - 1) >> 1) & 1u);
        float l1 = 0.f, S_ = 0.f;
        {
          float x = 0.f, y = 0.f;
#pragma unroll
          for (int k = lane; k < NP; k += 32) {
            const float2 q2 = ctrl->gb[pp][k];
            x += q2.x;
            y += q2.y;
          }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) {
            x += __shfl_xor_sync(0xffffffffu, x, off);
            y += __shfl_xor_sync(0xffffffffu, y, off);
          }
          l1 = x, S_ = y;
        }
        const int32_t prow = ctrl->rrow[jr];
        if (rank == 0 && warp == 0 && lane == 0) {
          float* st_row = a.ws.stats + size_t(prow) * kStride;
          st_row[kStL1] = l1;
          st_row[kStS] = S_;
        }
        if (bwd) {
          const int32_t ptokf = ctrl->rtok[jr];
          const int32_t ptok = ptokf & 0x7fffffff;
          // an invalid Markov slot's corrected row is a constant: nothing flows to the base
          const float gw = (HAS_B && ptokf < 0) ? 0.f : g_scale * ctrl->rw[jr];
          const float cce = gw * a.ce_alpha, cl1 = gw * a.l1_alpha;
          const float k0 = cce - cl1 * S_;
          const int tv = ptok / EPV - v0, te = ptok % EPV;
          uint8_t* out = static_cast<uint8_t*>(a.dlogits) + (size_t(prow) * a.ld_g + size_t(v0) * EPV) * 2;
          __syncwarp();  // TMEM accesses are warp-collective
          tm_wait_st();  // u of row j-1 (stored in its pass 2) is in TMEM
          uint32_t rb[2][EPV];
          tm_ld8(taddr(pp, 0), rb[0]);
#pragma unroll
          for (int i = 0; i < NV; ++i) {
            uint32_t* r = rb[i & 1];
            __syncwarp();
            tm_wait_ld8(r);
            if (i + 1 < NV) tm_ld8(taddr(pp, (i + 1) * EPV), rb[(i + 1) & 1]);  // in flight meanwhile
            const int v = tid + i * NTC;
            if (v < nvec) {
              float o[EPV];
#pragma unroll
              for (int e = 0; e < EPV; ++e) {
                const float u = __uint_as_float(r[e]);
                o[e] = fmaf(u, cl1, fabsf(u) * k0);
              }
              if (v == tv) {
#pragma unroll
                for (int e = 0; e < EPV; ++e)
                  if (e == te) o[e] -= cce;
              }
              *reinterpret_cast<uint4*>(out + size_t(v) * 16) =
                  make_uint4(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]), pack_bf16(o[4], o[5]),
                             pack_bf16(o[6], o[7]));
            }
          }
          write_zeros((j - 1) * zslice, min(ztot, j * zslice));
        }
      }
      if (!cur) break;
      // ======================================================== pass 2 of row j
      float lz2, lt2;
      {
        wait(smem_u32(&ctrl->bar_a[par]), uint32_t(j >> 1) & 1u);
        // all CL * NWC partials, in the same order in every warp of every CTA
        float m1 = -INFINITY, s1 = 0.f, m2 = -INFINITY, s2 = 0.f;
#pragma unroll
        for (int k = lane; k < NP; k += 32) {
          const float4 q4 = ctrl->ga[par][k];
          const float n1 = fmaxf(m1, q4.x), n2 = fmaxf(m2, q4.z);
          s1 = (n1 == -INFINITY) ? 0.f : s1 * ex2(m1 - n1) + (q4.x == -INFINITY ? 0.f : q4.y * ex2(q4.x - n1));
          s2 = (n2 == -INFINITY) ? 0.f : s2 * ex2(m2 - n2) + (q4.z == -INFINITY ? 0.f : q4.w * ex2(q4.z - n2));
          m1 = n1, m2 = n2;
        }
        lse2_warp(m1, s1, m2, s2);
        lz2 = m1 + log2f(s1);
        lt2 = m2 + log2f(s2);
      }
      {
        const int32_t row = ctrl->rrow[j % kRowRing];
        float* st_row = a.ws.stats + size_t(row) * kStride;
        if (rank == 0 && warp == 0 && lane == 0) {
          st_row[kStLseD] = lz2 * kLn2;
          st_row[kStLseT] = lt2 * kLn2;
        }
        const int tv = tok / EPV - v0;
        if (tv >= 0 && tv < nvec && tid == tv % NTC) {  // the thread that holds the target id
          st_row[kStCE] = lz2 * kLn2 - zt;
          st_row[kStZT] = zt;
        }
      }
      const float az = hz ? ex2(oz - lz2) : 0.f;  // p = e * az
      const float at = ht ? ex2(ot - lt2) : 0.f;  // q = e * at
      float l4[4] = {0.f, 0.f, 0.f, 0.f}, s4[4] = {0.f, 0.f, 0.f, 0.f};
      __syncwarp();  // TMEM accesses are warp-collective
      tm_wait_st();  // this row's teacher exponentials are in TMEM
      uint32_t rb[2][EPV];
      tm_ld8(taddr(par, 0), rb[0]);
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        uint32_t* r = rb[i & 1];
        tm_wait_ld8(r);
        if (i + 1 < NV) tm_ld8(taddr(par, (i + 1) * EPV), rb[(i + 1) & 1]);  // in flight meanwhile
        float u[EPV];
#pragma unroll
        for (int e = 0; e < EPV; ++e) {
          // an exact tie p == q takes the sub-gradient +p; equal draft and teacher rows
          // give p == q bit for bit (the same operations on the same values)
          const float q = __fmul_rn(__uint_as_float(r[e]), at);
          const float p = __fmul_rn(xz[i * EPV + e], az);
          const float d = __fsub_rn(p, q);
          u[e] = copysignf(p, d);
          l4[e & 3] += fabsf(d);
          s4[e & 3] += u[e];
        }
        tm_st8(taddr(par, i * EPV), u);
      }
      float l1p = (l4[0] + l4[1]) + (l4[2] + l4[3]);
      float sp = (s4[0] + s4[1]) + (s4[2] + s4[3]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        l1p += __shfl_xor_sync(0xffffffffu, l1p, off);
        sp += __shfl_xor_sync(0xffffffffu, sp, off);
      }
      // exchange B: this warp's (L1, S) pair into every CTA of the cluster
      const uint32_t bar = smem_u32(&ctrl->bar_b[par]);
      if (warp == 0 && lane == 0) mbar_arrive_expect_tx(bar, NP * 8);
      __syncwarp();
      if (lane < CL)
        st_async_f2(dsmem_map(smem_u32(&ctrl->gb[par][int(rank) * NWC + warp]), uint32_t(lane)), l1p, sp,
                    dsmem_map(bar, uint32_t(lane)));
    }
    // what is left of this cluster's zero rows (all of them if it had no row)
    if (bwd) write_zeros(my_n * zslice, ztot);
    __syncwarp();
    tm_wait_st();
  }

  // no CTA leaves while a peer may still signal or read its shared memory; TMEM is freed
  // once every warp's TMEM accesses are complete
  tm_fence_before();
  __syncthreads();
  cluster_sync();
  tm_fence_after();
  if (warp == 0) tm_dealloc(tmem, TCOLS);

  // ---- the last CTA to finish writes the per-row epilogue and the report
  if (!a.do_final) return;
  if (tid == 0) {
    __threadfence();
    ctrl->last = atomicAdd(&hdr->done, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (ctrl->last) {
    __threadfence();
    finalize_rows(a.fin, reinterpret_cast<double*>(smem));
    if (tid == 0) hdr->done = 0;
  }
}

// ------------------------------------------------------------------ host side
constexpr size_t kMaxSmemTm = 227 * 1024;
constexpr size_t kRingBudget = 200 * 1024;  // ring bytes; the rest holds the control block
constexpr size_t kOneCtaPerSm = 120 * 1024;  // at least this much: one CTA per SM (TMEM)

struct TmCache {
  std::mutex mu;
  int dev = -1;
  size_t smem = 0;
  int clusters = 0;
};

template <typename TT, bool HAS_B, int CL, int NWC, int NV>
cudaError_t launch_tm(const SweepArgs& a0, cudaStream_t s) {
  constexpr int NTC = NWC * 32, NT = NTC + 32;
  SweepArgs a = a0;
  a.vvec = int32_t(a.V / 8);
  a.seg_vec = (a.vvec + CL - 1) / CL;
  const size_t slab = size_t(NTC) * (16 + (HAS_B ? 32 : 0) + 8 * sizeof(TT));
  const int S = int(std::min<size_t>(kMaxSlabs, kRingBudget / slab));
  if (S < NV) return cudaErrorInvalidValue;
  const size_t ctrl = sizeof(CtrlTm<CL * NWC>);
  size_t smem = size_t(S) * slab + ctrl;
  smem = std::max(smem, size_t(NT / 32) * kNAcc * sizeof(double));
  smem = std::max(smem, kOneCtaPerSm);
  if (smem > kMaxSmemTm) return cudaErrorInvalidValue;
  auto kern = sweep_tm_kernel<TT, HAS_B, CL, NWC, NV>;
  static TmCache cache;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = CL;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  int clusters = 0;
  {
    std::lock_guard<std::mutex> lk(cache.mu);
    if (cache.dev != dev || cache.smem != smem) {
      err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kMaxSmemTm));
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
  // programmatic dependent launch: scheduled while the kernel before it runs, waits for it
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(clusters * CL), 1, 1);
  cfg.blockDim = dim3(NT, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  err = cudaLaunchKernelEx(&cfg, kern, a, S);
  if (err != cudaSuccess) cudaGetLastError();  // a refused launch leaves no error for later calls
  return err;
}

// Builds, smallest first: a build covers rows of up to CL * NWC * 32 * NV * 8 logits.
struct TmBuild {
  int cl, nwc, nv;
};
constexpr int kNumTmBuilds = 5;
// bf16 draft and teacher: 32 bytes per vector in the ring
constexpr TmBuild kTmBuilds[kNumTmBuilds] = {{1, 4, 1}, {2, 8, 2}, {4, 12, 3}, {8, 12, 4}, {8, 12, 7}};
// with bias rows and/or an FP32 teacher (48 to 80 bytes per vector): the largest rows over
// 16-CTA clusters of 8 compute warps, so that the ring still holds more than a row
constexpr TmBuild kTmHeadBuilds[kNumTmBuilds] = {{1, 4, 1}, {2, 8, 2}, {4, 12, 3}, {8, 12, 4}, {16, 8, 5}};

int pick_tm(int kind, int64_t V) {
  const TmBuild* b = kind == kSweepBf16 ? kTmBuilds : kTmHeadBuilds;
  for (int i = 0; i < kNumTmBuilds; ++i)
    if (int64_t(b[i].cl) * b[i].nwc * 32 * b[i].nv * 8 >= V) return i;
  return -1;
}

template <typename TT, bool HB>
cudaError_t dispatch_tm(int i, bool heads_table, const SweepArgs& a, cudaStream_t s) {
  switch (i) {
    case 0: return launch_tm<TT, HB, 1, 4, 1>(a, s);
    case 1: return launch_tm<TT, HB, 2, 8, 2>(a, s);
    case 2: return launch_tm<TT, HB, 4, 12, 3>(a, s);
    case 3: return launch_tm<TT, HB, 8, 12, 4>(a, s);
    case 4: return heads_table ? launch_tm<TT, HB, 16, 8, 5>(a, s) : launch_tm<TT, HB, 8, 12, 7>(a, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool sweep_tm_supported(int kind, int64_t V) {
  return (kind == kSweepBf16 || kind == kSweepZ32 || kind == kSweepT32 || kind == kSweepZT32) &&
         pick_tm(kind, V) >= 0;
}

cudaError_t launch_sweep_tm(int kind, const SweepArgs& a, cudaStream_t s) {
  const int i = pick_tm(kind, a.V);
  if (i < 0) return cudaErrorInvalidValue;
  switch (kind) {
    case kSweepBf16: return dispatch_tm<__nv_bfloat16, false>(i, false, a, s);
    case kSweepZ32: return dispatch_tm<__nv_bfloat16, true>(i, true, a, s);
    case kSweepT32: return dispatch_tm<float, false>(i, true, a, s);
    case kSweepZT32: return dispatch_tm<float, true>(i, true, a, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace dspark
