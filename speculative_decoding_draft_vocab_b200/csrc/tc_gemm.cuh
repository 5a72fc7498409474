// A bf16 x bf16 -> fp32 GEMM on the 5th-generation tensor cores (tcgen05 + TMEM),
// D[M, N] = sum_k A[m, k] * B[n, k], with a caller-supplied epilogue.
//
// One CTA of 192 threads per SM, persistent over (m-tile, n-tile, k-split) work items:
//   warp 0      one thread issues the TMA tile loads into a STAGES-deep shared ring
//   warp 1      allocates TMEM; one thread issues tcgen05.mma (M=128, N=BN, K=16
//               per instruction, 4 per 64-wide stage) and tcgen05.commit
//   warps 2..5  epilogue: tcgen05.ld of the accumulator, one TMEM lane (= one tile
//               row) per thread, 32 columns at a time.  Two kinds of epilogue:
//               - tensor store (Epi::kTma): the 32 x 32 block goes into a 128-byte-
//                 swizzled shared tile (double-buffered per warp), each row scaled by
//                 the functor's row_scale (0 drops a row), and one lane hands it to the
//                 TMA engine as a tensor store or a tensor reduce-add into the output
//                 tensor map;
//               - functor: the block is transposed through a padded 32 x 33 shared
//                 tile and the functor's lanes walk the columns of one row at a time;
//                 its row_state(m0, lane) is taken once per tile.
// The accumulator is double-buffered in TMEM (2 x BN columns) so the epilogue of one
// tile overlaps the MMAs of the next.  Operands are 128-byte-swizzled tiles, either
// K-major (rows of 64 K values) or MN-major (rows of 64 M/N values per K index).
// Every wait is bounded; a timeout raises a status flag and the kernel still ends.
#pragma once
#include <cuda.h>

#include "ptx.cuh"

namespace dspark {
namespace tc {

constexpr int BM = 128;         // tile rows (TMEM lanes)
constexpr int BK = 64;          // K per stage: one 128-byte swizzle row of bf16
constexpr int kThreads = 192;   // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr uint32_t kTimeoutFlag = 1u << 1;

// ---- descriptors (SM100 shared-memory matrix descriptor, 128-byte swizzle)
// start address, leading and stride byte offsets in 16-byte units; version 1 (bit 46);
// layout SWIZZLE_128B (2) in bits 61-63.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         (uint64_t((sbo_bytes >> 4) & 0x3FFFu) << 32) | (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// Instruction descriptor of kind::f16 with bf16 A and B, fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(a_mn) << 15) | (uint32_t(b_mn) << 16) |
         (uint32_t(n >> 3) << 17) | (uint32_t(m >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate),
        "r"(0u), "r"(0u), "r"(0u), "r"(0u) : "memory");
}

// Arrive on `bar` once every tcgen05 op this thread issued before has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(bar) : "memory");
}

__device__ __forceinline__ void fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t slot_saddr, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(slot_saddr), "r"(ncols) : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"(map), "r"(x), "r"(y), "r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Epilogue staging, 1024-byte aligned: per epilogue warp either one padded 32 x 33 fp32
// tile (functor epilogue) or two 4 KB swizzled 32 x 32 fp32 tiles (tensor store).
constexpr int kTileLd = 33;
constexpr size_t kStageBytes = 4 * 2 * 4096;

// Shared memory a configuration needs (dynamic; the base is aligned to 1024 inside):
// the operand ring, 1 KB of barriers, the epilogue staging.
template <int BN, int STAGES>
constexpr size_t gemm_smem_bytes() {
  return size_t(STAGES) * (BM * BK * 2 + BN * BK * 2) + 1024 + kStageBytes + 1024;
}

// Tensor store / reduce-add of a shared tile into the output tensor map (bulk group of
// the issuing thread).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];"
               ::"l"(map), "r"(x), "r"(y), "r"(src) : "memory");
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];"
               ::"l"(map), "r"(x), "r"(y), "r"(z), "r"(src) : "memory");
}
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.bulk_group [%0, {%1, %2}], [%3];"
               ::"l"(map), "r"(x), "r"(y), "r"(src) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

// Work item w -> (m-tile, n-tile, k-split) and its range of 64-wide K chunks.  The
// m-tile is the fastest index: CTAs running at the same time share their B tiles (the
// large operand of the row-skinny products) through L2 instead of each m-tile
// streaming all of B from HBM again.  With a device-side row bound (rows m_base + m
// at or past *m_bound are not needed) only the first m_eff() m-tiles take part.
struct WorkMap {
  int m_tiles, n_tiles, ksplit, kchunks;
  const int32_t* m_bound;
  int m_base;
  __device__ __forceinline__ int m_eff() const {
    if (m_bound == nullptr) return m_tiles;
    const int rem = *m_bound - m_base;
    return rem <= 0 ? 0 : min(m_tiles, (rem + BM - 1) / BM);
  }
  __device__ __forceinline__ int items(int me) const { return me * n_tiles * ksplit; }
  __device__ __forceinline__ void decode(int w, int me, int& mt, int& nt, int& s, int& kc0, int& kc1) const {
    mt = w % me;
    const int t = w / me;
    s = t % ksplit;
    nt = t / ksplit;
    kc0 = int((int64_t(s) * kchunks) / ksplit);
    kc1 = int((int64_t(s + 1) * kchunks) / ksplit);
  }
};

// A_MN / B_MN: operand stored MN-major (the M or N index is the contiguous one).
// Tensor maps: K-major A = [M rows][K] box {64, 128}; MN-major A = [K rows][M] box
// {64, 64}; K-major B = [N rows][K] box {64, BN}; MN-major B = [K rows][N] box {64, 64}.
template <int BN, bool A_MN, bool B_MN, int STAGES, class Epi>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const __grid_constant__ CUtensorMap tmO, const WorkMap wm, const Epi epi, uint32_t* status) {
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "N tile");
  constexpr uint32_t SA = BM * BK * 2, SB = BN * BK * 2, SS = SA + SB;
  constexpr uint32_t kIdesc = idesc_bf16(BM, BN, A_MN, B_MN);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + size_t(STAGES) * SS);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * STAGES;
  const uint32_t accf0 = empty0 + 8 * STAGES;
  const uint32_t acce0 = accf0 + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
  uint8_t* stage = smem + size_t(STAGES) * SS + 1024;  // 1024-byte aligned

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int ME = wm.m_eff();  // the same in every role
  const int W = wm.items(ME);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf0 + 8 * b, 1);
      mbar_init(acce0 + 8 * b, 4);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 2 * BN);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  bool timed_out = false;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    int it = 0;
    for (int w = blockIdx.x; w < W; w += gridDim.x) {
      int mt, nt, s, kc0, kc1;
      wm.decode(w, ME, mt, nt, s, kc0, kc1);
      for (int kc = kc0; kc < kc1; ++kc, ++it) {
        const int st = it % STAGES;
        const uint32_t round = uint32_t(it / STAGES);
        if (!mbar_wait_bounded(empty0 + 8 * st, (round & 1u) ^ 1u)) timed_out = true;
        const uint32_t fb = full0 + 8 * st;
        mbar_arrive_expect_tx(fb, SS);
        const uint32_t sa = smem_u32(smem + size_t(st) * SS), sb = sa + SA;
        const int k0 = kc * BK;
        if constexpr (!A_MN) {
          tma_load_2d(sa, &tmA, k0, mt * BM, fb);
        } else {
#pragma unroll
          for (int c = 0; c < BM / 64; ++c) tma_load_2d(sa + c * 8192, &tmA, mt * BM + c * 64, k0, fb);
        }
        if constexpr (!B_MN) {
          tma_load_2d(sb, &tmB, k0, nt * BN, fb);
        } else {
#pragma unroll
          for (int c = 0; c < BN / 64; ++c) tma_load_2d(sb + c * 8192, &tmB, nt * BN + c * 64, k0, fb);
        }
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    int it = 0, tl = 0;
    for (int w = blockIdx.x; w < W; w += gridDim.x, ++tl) {
      int mt, nt, s, kc0, kc1;
      wm.decode(w, ME, mt, nt, s, kc0, kc1);
      const int b = tl & 1;
      const uint32_t use = uint32_t(tl >> 1);
      if (!mbar_wait_bounded(acce0 + 8 * b, (use & 1u) ^ 1u)) timed_out = true;
      fence_after_sync();
      const uint32_t d_tmem = tmem_base + uint32_t(b * BN);
      for (int kc = kc0; kc < kc1; ++kc, ++it) {
        const int st = it % STAGES;
        const uint32_t round = uint32_t(it / STAGES);
        if (!mbar_wait_bounded(full0 + 8 * st, round & 1u)) timed_out = true;
        fence_after_sync();
        const uint32_t sa = smem_u32(smem + size_t(st) * SS), sb = sa + SA;
#pragma unroll
        for (int ks = 0; ks < BK / 16; ++ks) {
          // K-major: the next 16 K values are 32 bytes further along each 128-byte row;
          // MN-major: 16 more K rows of 128 bytes.
          const uint64_t ad = A_MN ? sdesc(sa + ks * 2048, 8192, 1024) : sdesc(sa + ks * 32, 16, 1024);
          const uint64_t bd = B_MN ? sdesc(sb + ks * 2048, 8192, 1024) : sdesc(sb + ks * 32, 16, 1024);
          mma_bf16(d_tmem, ad, bd, kIdesc, (kc > kc0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(empty0 + 8 * st);  // frees the stage once these MMAs have read it
      }
      mma_commit(accf0 + 8 * b);      // accumulator ready
    }
  } else if (warp >= 2) {
    // ---------------- epilogue: warp w reads TMEM lanes 32*(w % 4) .. +31
    const int q = warp & 3;
    float* tile = reinterpret_cast<float*>(stage + q * 8192);  // functor epilogue
    const uint32_t tbuf0 = smem_u32(stage + q * 8192);         // tensor-store epilogue
    int blk = 0;
    int tl = 0;
    for (int w = blockIdx.x; w < W; w += gridDim.x, ++tl) {
      int mt, nt, s, kc0, kc1;
      wm.decode(w, ME, mt, nt, s, kc0, kc1);
      const int b = tl & 1;
      const uint32_t use = uint32_t(tl >> 1);
      if (!mbar_wait_bounded(accf0 + 8 * b, use & 1u)) timed_out = true;
      fence_after_sync();
      const uint32_t taddr = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(b * BN);
      const int m0 = mt * BM + q * 32;
      if constexpr (Epi::kTma) {
        const float scale = epi.row_scale(m0 + lane);  // this thread's row, once per tile
        // a 32-row block wholly past the device-side row bound is not needed: not stored
        const bool needed = wm.m_bound == nullptr || wm.m_base + m0 < *wm.m_bound;
#pragma unroll 1
        for (int c = 0; needed && c < BN / 32; ++c, ++blk) {
          float v[32];
          __syncwarp();  // the TMEM load is warp-collective
          tmem_ld32(taddr + uint32_t(c * 32), v);
          const uint32_t buf = tbuf0 + uint32_t(blk & 1) * 4096u;
          if (lane == 0) bulk_wait_read<1>();  // the store that last used this buffer has read it
          __syncwarp();
          // row `lane`: 128 bytes, 16-byte chunk k at chunk k ^ (lane % 8) (128-byte swizzle)
#pragma unroll
          for (int k = 0; k < 8; ++k)
            st_shared_v4(buf + uint32_t(lane) * 128u + uint32_t((k ^ (lane & 7)) * 16), v[4 * k] * scale,
                         v[4 * k + 1] * scale, v[4 * k + 2] * scale, v[4 * k + 3] * scale);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            int x, y, z;
            epi.coords(m0, nt * BN + c * 32, s, x, y, z);
            if (epi.tma_mode() == 2) tma_reduce_add_2d(&tmO, buf, x, y);
            else if (z >= 0) tma_store_3d(&tmO, buf, x, y, z);
            else tma_store_2d(&tmO, buf, x, y);
            bulk_commit();
          }
        }
      } else {
        // per-row state of the functor (e.g. gathered row ids), fetched once per tile
        const uint64_t rs = epi.row_state(m0, lane);
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          float v[32];
          __syncwarp();  // the TMEM load is warp-collective
          tmem_ld32(taddr + uint32_t(c * 32), v);
#pragma unroll
          for (int i = 0; i < 32; ++i) tile[lane * kTileLd + i] = v[i];  // row lane, column i
          __syncwarp();
          // rows m0 .. m0 + 31, columns n0 .. n0 + 31: element (r, j) at tile[r * kTileLd + j]
          epi(m0, nt * BN + c * 32, s, static_cast<const float*>(tile), lane, rs);
          __syncwarp();
        }
      }
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce0 + 8 * b);
    }
    // the staging tiles stay until the TMA engine has read them
    if constexpr (Epi::kTma) {
      if (lane == 0) bulk_wait_read<0>();
    }
  }
  if (timed_out) atomicOr(status, kTimeoutFlag);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem_base, 2 * BN);
}

}  // namespace tc
}  // namespace dspark
