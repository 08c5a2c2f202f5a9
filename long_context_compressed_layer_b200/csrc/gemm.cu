// Grouped output projection (cyqw.cn DeepSeek-V4 walkthrough §2.2: with 128 query heads
// the output projection first reduces each group of heads, then projects the
// concatenation; "DeepSeek-V4：百万上下文的工程答案", Hybrid Attention: it follows the
// shared-KV MQA).
//
// Both stages are BF16 GEMM tiles C[128 x 128] = A[128 x K] B[128 x K]^T with fp32
// accumulation in TMEM and a BF16 (round-to-nearest-even) epilogue: one CTA per
// (row tile, column tile, group). Warp 0 streams 64-wide K blocks of A and B by TMA
// (128-byte swizzle) into a 3-stage ring (two CTAs fit an SM), warp 1 issues tcgen05.mma kind::f16 (BF16),
// warps 2-5 (one per TMEM lane quadrant, one row per thread) convert and store. The
// group index selects column offsets of A and C and a row offset of B, so stage 1 runs
// all groups in one launch over the [T][H * 512] attention output.
#include "common.cuh"

namespace csa {

constexpr int kGmStages = 3;
constexpr int kGmTile = 128;
constexpr int kGmKBlk = 64;
constexpr int kGmThreads = 192;

struct GmSmem {
  uint8_t a[kGmStages][kGmTile * 128];
  uint8_t b[kGmStages][kGmTile * 128];
  uint64_t full[kGmStages], empty[kGmStages], acc_full;
  uint32_t tmem_base;
};

struct GmParams {
  int M, K;                 // rows of C, reduction length
  int a_x_group, b_y_group; // per-group offsets: A column, B row (elements)
  int64_t c_x_group;        // per-group C column offset
  uint16_t* C;
  int64_t ldc;
  int32_t* dev_status;
};

__global__ void __launch_bounds__(kGmThreads, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap amap,
                     const __grid_constant__ CUtensorMap bmap, GmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  GmSmem& s = *reinterpret_cast<GmSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kGmTile, n0 = blockIdx.y * kGmTile, z = blockIdx.z;
  const int nk = p.K / kGmKBlk;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kGmStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    mbar_init(&s.acc_full, 1);
    mbar_fence_init();
    prefetch_tensormap(&amap);
    prefetch_tensormap(&bmap);
  }
  if (warp == 1) tmem_alloc(&s.tmem_base, 128);
  pdl_wait();
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      int kb = 0;
      for (; kb < nk; ++kb) {
        const int st = kb % kGmStages;
        if (!mbar_wait(&s.empty[st], ((kb / kGmStages) & 1) ^ 1, p.dev_status)) break;
        mbar_arrive_expect_tx(&s.full[st], 2 * kGmTile * 128);
        tma_load_2d(s.a[st], &amap, &s.full[st], z * p.a_x_group + kb * kGmKBlk, t0);
        tma_load_2d(s.b[st], &bmap, &s.full[st], kb * kGmKBlk, z * p.b_y_group + n0);
      }
      for (int i = kb - kGmStages < 0 ? 0 : kb - kGmStages; i < kb; ++i)  // drain
        mbar_wait(&s.full[i % kGmStages], (i / kGmStages) & 1, p.dev_status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id = idesc_bf16(kGmTile, kGmTile, false);
      for (int kb = 0; kb < nk; ++kb) {
        const int st = kb % kGmStages;
        if (!mbar_wait(&s.full[st], (kb / kGmStages) & 1, p.dev_status)) break;
        tc_fence_after();
        for (int kk = 0; kk < 4; ++kk)
          mma_f16(tmem, smem_desc(smem_u32(s.a[st]) + kk * 32, 16, 1024, kSwizzle128B),
                  smem_desc(smem_u32(s.b[st]) + kk * 32, 16, 1024, kSwizzle128B), id,
                  (kb > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&s.empty[st]);
      }
      mma_commit(&s.acc_full);
      mbar_wait(&s.acc_full, 0, p.dev_status);
    }
    __syncwarp();
  } else {
    const int quad = warp & 3, t = t0 + quad * 32 + lane;
    const bool ok = mbar_wait(&s.acc_full, 0, p.dev_status);
    tc_fence_after();
    uint16_t* crow = p.C + (size_t)t * p.ldc + z * p.c_x_group + n0;
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t v[32];
      __syncwarp();  // the TMEM load is warp-collective
      tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + cc * 32, v);
      tmem_ld_wait();
      if (!ok || t >= p.M) continue;
      uint4* dst = reinterpret_cast<uint4*>(crow + cc * 32);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          w[e] = (uint32_t)f32_to_bf16_bits(__uint_as_float(v[q * 8 + 2 * e])) |
                 ((uint32_t)f32_to_bf16_bits(__uint_as_float(v[q * 8 + 2 * e + 1])) << 16);
        dst[q] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// C[:, group] (M x N per group, BF16) = A[:, group] B[group]^T over K, for G groups.
cudaError_t launch_gemm_bf16(const CUtensorMap& amap, const CUtensorMap& bmap, int M, int N,
                             int K, int G, int a_x_group, int b_y_group, int64_t c_x_group,
                             uint16_t* C, int64_t ldc, int32_t* dev_status,
                             cudaStream_t stream) {
  GmParams p{M, K, a_x_group, b_y_group, c_x_group, C, ldc, dev_status};
  const size_t smem = sizeof(GmSmem) + 1024;
  static std::atomic<uint64_t> configured{0};
  if (cudaError_t e = configure_smem_once(gemm_bf16_kernel, smem, configured);
      e != cudaSuccess)
    return e;
  dim3 grid((M + kGmTile - 1) / kGmTile, N / kGmTile, G);
  return launch_pdl(gemm_bf16_kernel, grid, dim3(kGmThreads), smem, stream, amap, bmap, p);
}

}  // namespace csa
