// Test harness for the tcgen05 GEMM of the library (compiled by tests/test_tc_gemm_gpu.py):
// D = A . B^T with a plain fp32 store epilogue, for every operand-major combination.
#include <cstdint>

#include "tc_host.cuh"

using namespace dspark;

struct SplitStoreEpi {  // partial of K split s at d[s][m][n]; the block is rows m0.., columns n0..
  static constexpr bool kTma = false;
  float* d;
  int M, N;
  __device__ uint64_t row_state(int, int) const { return 0; }
  __device__ void operator()(int m0, int n0, int split, const float* t, int lane, uint64_t) const {
    const int n = n0 + lane;
    if (n >= N) return;
    for (int r = 0; r < 32 && m0 + r < M; ++r) d[(int64_t(split) * M + m0 + r) * N + n] = t[r * tc::kTileLd + lane];
  }
};

template <int BN, bool AMN, bool BMN>
static int run(const void* a, const void* b, float* d, int M, int N, int K, int ksplit, uint32_t* status) {
  CUtensorMap ma, mb;
  // K-major A: [M][K] box {64, 128}; MN-major A: [K][M] box {64, 64}
  const bool ok_a = AMN ? tc::make_map(&ma, a, K, M, M, 64, 64) : tc::make_map(&ma, a, M, K, K, 64, 128);
  const bool ok_b = BMN ? tc::make_map(&mb, b, K, N, N, 64, 64) : tc::make_map(&mb, b, N, K, K, 64, BN);
  if (!ok_a || !ok_b) return -1;
  SplitStoreEpi epi{d, M, N};
  return int(tc::gemm<BN, AMN, BMN, 4>(ma, mb, M, N, K, ksplit, epi, status, nullptr));
}

// a_mn: a is [K][M] (M contiguous) instead of [M][K]; b_mn: b is [K][N] instead of [N][K].
// d receives ksplit partials [ksplit][M][N].  Returns a cudaError_t (or -1 for a bad map).
extern "C" int tc_gemm_test(const void* a, const void* b, float* d, int M, int N, int K, int a_mn, int b_mn,
                            int bn, int ksplit, uint32_t* status) {
  if (bn == 256) {
    if (!a_mn && !b_mn) return run<256, false, false>(a, b, d, M, N, K, ksplit, status);
    if (!a_mn && b_mn) return run<256, false, true>(a, b, d, M, N, K, ksplit, status);
    if (a_mn && !b_mn) return run<256, true, false>(a, b, d, M, N, K, ksplit, status);
    return run<256, true, true>(a, b, d, M, N, K, ksplit, status);
  }
  if (bn == 128) {
    if (!a_mn && !b_mn) return run<128, false, false>(a, b, d, M, N, K, ksplit, status);
    if (a_mn && b_mn) return run<128, true, true>(a, b, d, M, N, K, ksplit, status);
  }
  return -2;
}

// Gathered A: the rows of the bf16 matrix `src` [src_rows][src_cols] listed in `list`
// (`*len` of them, a device count) form A, fetched by four-row gathers.  a_mn = 0: A's
// rows are M indices (D[M = positions, N] = sum over K = src_cols); a_mn = 1: A's rows are
// K indices (D[M = src_cols, N] = sum over K = positions, bounded on the device by *len).
// b is [N][K] (K-major) for a_mn = 0 and [K][N] (MN-major) for a_mn = 1.
extern "C" int tc_gemm_gather_test(const void* src, int src_rows, int src_cols, const int32_t* list,
                                   const int32_t* len, int positions, const void* b, int N, float* d, int a_mn,
                                   int ksplit, uint32_t* status) {
  CUtensorMap ma, mb;
  if (!tc::make_row_map(&ma, src, src_rows, src_cols, src_cols, 64)) return -1;
  tc::GemmOpts o;
  o.list = list;
  o.list_len = len;
  o.zero_row = src_rows;
  if (!a_mn) {
    if (!tc::make_map(&mb, b, N, src_cols, src_cols, 64, 256)) return -1;
    o.m_bound = len;
    SplitStoreEpi epi{d, positions, N};
    return int(tc::gemm<256, false, false, 4, SplitStoreEpi, true>(ma, mb, positions, N, src_cols, ksplit, epi,
                                                                    status, nullptr, o));
  }
  if (!tc::make_map(&mb, b, positions, N, N, 64, 64)) return -1;
  o.k_bound = len;
  SplitStoreEpi epi{d, src_cols, N};
  return int(tc::gemm<256, true, true, 4, SplitStoreEpi, true>(ma, mb, src_cols, N, positions, 1, epi, status,
                                                                nullptr, o));
}
