// gemm.cu -- bf16 GEMM on tcgen05 tensor cores for the token mixer's projections, with an
// optional gate epilogue.
//
//   C[M][N] = A[M][K] B[K][N]     A row-major (the activations, K contiguous), B row-major (a
//                                 weight stored input x output, N contiguous), fp32 accumulation
//
// One CTA per 128 x BN output tile, four warps.  Thread 0 streams the K dimension through a ring
// of shared-memory stages with TMA (A as a [128][64] box, B as BN/64 boxes of [64][64], all with
// 128-byte swizzle); thread 32 issues the tcgen05.mma of each stage (A K-major, B MN-major, the
// fp32 accumulator in TMEM) and returns the stage to the producer with tcgen05.commit.  After
// the last stage every warp reads its 32 TMEM lanes and runs the epilogue:
//   plain   bf16 result, staged in shared memory and written by TMA stores (rows past M are
//           clipped by the tensor map);
//   gates   the [b | a] projection of the gated delta rule (N = 2 Hv): beta = sigmoid(b) and
//           g = -exp(A_log) softplus(a + dt_bias) per value head, written as fp32 [M][Hv] rows
//           (the same reading of the gates as the token mixer's documentation states).
// Tails: rows past M and columns past K or N read zeros (TMA fill); N may be smaller than BN.
// Every wait is bounded (%globaltimer); a wait that runs out reports GDN_ERR_TIMEOUT.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "tc.cuh"

namespace gdn {

constexpr uint32_t kGemmATile = 16384;  // [128 rows][64 K] bf16
constexpr int kGemmThreads = 128;

template <int BN>
struct GemmCfg {
  static_assert(BN == 64 || BN == 128 || BN == 256, "tile width");
  static constexpr uint32_t kBTile = 64u * BN * 2;            // [64 K rows][BN] bf16
  static constexpr uint32_t kStage = kGemmATile + kBTile;
  static constexpr int kStages = BN == 256 ? 4 : (BN == 128 ? 6 : 8);
  static constexpr uint32_t kRing = kStage * kStages;
  static constexpr uint32_t kSmem = kRing + 1024 + 256;       // + alignment + barriers
};

enum GemmEpi : int { kEpiBf16 = 0, kEpiGates = 1 };

struct GemmArgs {
  int M, N, K;
  // gates epilogue
  const float* a_log;
  const float* dt_bias;
  float* beta;
  float* g;
  int Hv;
  int32_t* status;
};

template <int BN, int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_bf16_kernel(GemmArgs p, const __grid_constant__ CUtensorMap mapA,
                     const __grid_constant__ CUtensorMap mapB,
                     const __grid_constant__ CUtensorMap mapC) {
  using Cfg = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + Cfg::kRing);  // [kStages]
  uint64_t* empty = full + Cfg::kStages;                           // [kStages]
  uint64_t* done = empty + Cfg::kStages;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * BN, m0 = blockIdx.y * 128;
  const int ksteps = (p.K + 63) / 64;

  if (tid == 0) {
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tslot, BN);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  bool ok = true;

  if (tid == 0) {
    // producer: stage s of step k waits until the MMAs of step k - kStages released it
    for (int k = 0; k < ksteps && ok; ++k) {
      const int s = k % Cfg::kStages;
      if (k >= Cfg::kStages) ok = mbar_wait(empty + s, ((k / Cfg::kStages) - 1) & 1);
      if (!ok) break;
      uint8_t* a_dst = sm + s * Cfg::kStage;
      uint8_t* b_dst = a_dst + kGemmATile;
      mbar_arrive_expect_tx(full + s, Cfg::kStage);
      tma_load_2d(a_dst, &mapA, full + s, k * 64, m0);
#pragma unroll
      for (int j = 0; j < BN / 64; ++j) tma_load_2d(b_dst + j * 8192, &mapB, full + s, n0 + 64 * j, k * 64);
    }
  } else if (tid == 32) {
    // MMA issuer: four K steps of 16 per stage into the one accumulator
    constexpr uint32_t id = idesc_bf16(128, BN, false, true);
    for (int k = 0; k < ksteps && ok; ++k) {
      const int s = k % Cfg::kStages;
      ok = mbar_wait(full + s, (k / Cfg::kStages) & 1);
      if (!ok) break;
      tc_fence_after();
      const uint32_t sa = smem_u32(sm + s * Cfg::kStage), sb = sa + kGemmATile;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem, desc_kmajor(sa, kk, kGemmATile), desc_mnmajor(sb, kk, 8192), id,
                 (k > 0 || kk > 0) ? 1u : 0u);
      mma_commit(empty + s);
    }
    if (ok) mma_commit(done);
  }
  // every thread waits for the accumulator (or learns that a wait ran out)
  if (__syncthreads_or(!ok)) {
    if (tid == 0) report_status(p.status, GDN_ERR_TIMEOUT);
    // give copies and products already issued a bounded time to land
    if (tid == 0)
      for (int s = 0; s < Cfg::kStages; ++s) mbar_wait(empty + s, 0, 1000000ull);
    __syncthreads();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, BN);
    return;
  }
  ok = mbar_wait(done, 0);
  if (__syncthreads_or(!ok)) {
    if (tid == 0) report_status(p.status, GDN_ERR_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, BN);
    return;
  }
  tc_fence_after();
  const int row = warp * 32 + lane;  // TMEM lane = row of the tile
  const uint32_t lane_addr = tmem_at(tmem, warp * 32, 0);
  if constexpr (EPI == kEpiBf16) {
    // the ring is free: stage the bf16 tile as BN/64 row tiles of [128][64], then TMA stores
#pragma unroll
    for (int j = 0; j < BN / 64; ++j) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float v[32];
        tmem_ld32(lane_addr + j * 64 + half * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q)
          st_row8_bf16(sm + j * 16384, 16384, row, half * 4 + q, v + 8 * q);
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
#pragma unroll
      for (int j = 0; j < BN / 64; ++j)
        if (n0 + 64 * j < p.N) tma_store_2d(&mapC, sm + j * 16384, n0 + 64 * j, m0);
      bulk_commit();
      bulk_wait_reads();
    }
  } else {
    // gates: columns [0, Hv) are b, [Hv, 2 Hv) are a (2 Hv <= BN)
    const int Hv = p.Hv;
    const int grow = m0 + row;
    float v[BN];
#pragma unroll
    for (int c = 0; c < BN / 32; ++c) {
      float t[32];
      tmem_ld32(lane_addr + c * 32, t);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; ++e) v[c * 32 + e] = t[e];
    }
    if (grow < p.M) {
#pragma unroll 4
      for (int hh = 0; hh < BN / 2; ++hh) {
        if (hh >= Hv) break;
        const float b = v[hh];
        const float a = v[Hv + hh < BN ? Hv + hh : 0] + __ldg(p.dt_bias + hh);
        const float sp = a > 20.f ? a : log1pf(expf(a));  // softplus
        p.beta[(size_t)grow * Hv + hh] = 1.f / (1.f + expf(-b));
        p.g[(size_t)grow * Hv + hh] = -expf(__ldg(p.a_log + hh)) * sp;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, BN);
}

}  // namespace gdn

namespace gdn_host {

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// [rows][cols] bf16 row-major, box [box_rows][64 cols], 128-byte swizzle.
static bool map_2d(CUtensorMap* m, const void* base, size_t rows, size_t cols, uint32_t box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int EPI>
static cudaError_t launch_gemm(const gdn::GemmArgs& p, const CUtensorMap& mA,
                               const CUtensorMap& mB, const CUtensorMap& mC, cudaStream_t s) {
  using Cfg = gdn::GemmCfg<BN>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(gdn::gemm_bf16_kernel<BN, EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const dim3 grid((p.N + BN - 1) / BN, (p.M + 127) / 128);
  gdn::gemm_bf16_kernel<BN, EPI><<<grid, gdn::kGemmThreads, Cfg::kSmem, s>>>(p, mA, mB, mC);
  return cudaGetLastError();
}

// C[M][N] (bf16) = A[M][K] B[K][N], all row-major bf16; 16-byte aligned rows (K, N multiples
// of 8).  The tile width follows N.
cudaError_t gemm_bf16(const void* A, const void* B, void* C, int M, int N, int K,
                      int32_t* status, cudaStream_t s) {
  if (M == 0 || N == 0) return cudaSuccess;
  CUtensorMap mA, mB, mC;
  if (!map_2d(&mA, A, M, K, 128) || !map_2d(&mB, B, K, N, 64) || !map_2d(&mC, C, M, N, 128))
    return cudaErrorInvalidValue;
  gdn::GemmArgs p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.status = status;
  if (N % 256 == 0) return launch_gemm<256, gdn::kEpiBf16>(p, mA, mB, mC, s);
  if (N % 128 == 0) return launch_gemm<128, gdn::kEpiBf16>(p, mA, mB, mC, s);
  return launch_gemm<64, gdn::kEpiBf16>(p, mA, mB, mC, s);
}

// The [b | a] projection (N = 2 Hv <= 64) with the gates in the epilogue: beta, g [M][Hv] fp32.
cudaError_t gemm_bf16_gates(const void* A, const void* B, int M, int Hv, int K,
                            const float* a_log, const float* dt_bias, float* beta, float* g,
                            int32_t* status, cudaStream_t s) {
  if (M == 0) return cudaSuccess;
  if (2 * Hv > 64) return cudaErrorInvalidValue;
  CUtensorMap mA, mB;
  if (!map_2d(&mA, A, M, K, 128) || !map_2d(&mB, B, K, 2 * Hv, 64)) return cudaErrorInvalidValue;
  gdn::GemmArgs p{};
  p.M = M;
  p.N = 2 * Hv;
  p.K = K;
  p.a_log = a_log;
  p.dt_bias = dt_bias;
  p.beta = beta;
  p.g = g;
  p.Hv = Hv;
  p.status = status;
  return launch_gemm<64, gdn::kEpiGates>(p, mA, mB, mA, s);
}

}  // namespace gdn_host
