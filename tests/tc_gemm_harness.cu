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
