// Indexer queries: the low-rank up-projection of the query latent into the indexer heads,
// quantised to MXFP4 in the layout csa_indexer_topk reads (cyqw.cn DeepSeek-V4
// walkthrough §2.2: low-rank indexer queries, down-projected then up-projected, the down
// projection shared with the main attention; §3.4: the indexer QK path is FP4).
//
// One CTA per (128-token tile, indexer head): y[t][0..127] = sum_j W[h*128 + .][j] c[t][j]
// is a 128 x 128 x r BF16 GEMM tile. Warp 0 streams the K blocks of c and W (64 BF16
// each, 128-byte swizzle) by TMA into a 3-stage ring (two CTAs fit an SM); warp 1 issues four
// tcgen05.mma kind::f16 (BF16, K = 16) per block into 128 fp32 TMEM columns; warps 2-5
// (one per TMEM lane quadrant, one token per thread) read the token's 128 values, and
// per 32-value block form the MXFP4 shared exponent and E2M1 codes, writing 64 code
// bytes and 4 scale bytes per (token, head). Tokens past T come in as zeros (TMA fill)
// and are not stored.
#include "common.cuh"

namespace csa {

constexpr int kIqStages = 3;
constexpr int kIqTile = 128;   // tokens per CTA = MMA M; one head's 128 dims = MMA N
constexpr int kIqKBlk = 64;    // BF16 elements per K block (one 128-byte swizzle row)
constexpr int kIqThreads = 192;

struct IqSmem {
  uint8_t a[kIqStages][kIqTile * 128];  // c tile [128 tokens x 64], 128-B swizzle
  uint8_t b[kIqStages][kIqTile * 128];  // W tile [128 dims x 64]
  uint64_t full[kIqStages], empty[kIqStages], acc_full;
  uint32_t tmem_base;
};

struct IqParams {
  int T, r, H_I;
  uint8_t* q_fp4;
  uint8_t* q_sf;
  float* dbg;
  int32_t* dev_status;
};

__global__ void __launch_bounds__(kIqThreads, 1)
    iquery_kernel(const __grid_constant__ CUtensorMap cmap,
                  const __grid_constant__ CUtensorMap wmap, IqParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  IqSmem& s = *reinterpret_cast<IqSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kIqTile, h = blockIdx.y;
  const int nk = p.r / kIqKBlk;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kIqStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    mbar_init(&s.acc_full, 1);
    mbar_fence_init();
    prefetch_tensormap(&cmap);
    prefetch_tensormap(&wmap);
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
        const int st = kb % kIqStages;
        if (!mbar_wait(&s.empty[st], ((kb / kIqStages) & 1) ^ 1, p.dev_status)) break;
        mbar_arrive_expect_tx(&s.full[st], 2 * kIqTile * 128);
        tma_load_2d(s.a[st], &cmap, &s.full[st], kb * kIqKBlk, t0);
        tma_load_2d(s.b[st], &wmap, &s.full[st], kb * kIqKBlk, h * kIqTile);
      }
      for (int i = kb - kIqStages < 0 ? 0 : kb - kIqStages; i < kb; ++i)  // drain
        mbar_wait(&s.full[i % kIqStages], (i / kIqStages) & 1, p.dev_status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id = idesc_bf16(kIqTile, kIqTile, false);
      bool ok = true;
      for (int kb = 0; kb < nk && ok; ++kb) {
        const int st = kb % kIqStages;
        ok = mbar_wait(&s.full[st], (kb / kIqStages) & 1, p.dev_status);
        if (!ok) break;
        tc_fence_after();
        for (int kk = 0; kk < 4; ++kk)
          mma_f16(tmem, smem_desc(smem_u32(s.a[st]) + kk * 32, 16, 1024, kSwizzle128B),
                  smem_desc(smem_u32(s.b[st]) + kk * 32, 16, 1024, kSwizzle128B), id,
                  (kb > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&s.empty[st]);
      }
      mma_commit(&s.acc_full);  // also the completion of everything issued above
      mbar_wait(&s.acc_full, 0, p.dev_status);  // nothing in flight when TMEM is released
    }
    __syncwarp();
  } else {
    const int quad = warp & 3, t = t0 + quad * 32 + lane;
    const bool ok = mbar_wait(&s.acc_full, 0, p.dev_status);
    tc_fence_after();
    uint32_t sf_word = 0;
    for (int sb = 0; sb < 4; ++sb) {  // 32-value blocks
      uint32_t v[32];
      __syncwarp();  // the TMEM load is warp-collective
      tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + sb * 32, v);
      tmem_ld_wait();
      if (!ok || t >= p.T) continue;
      float amax = 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) amax = fmaxf(amax, fabsf(__uint_as_float(v[e])));
      const int ex = mxfp4_exponent(amax);
      uint32_t w4[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t wd = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e)
          wd |= e2m1_code(ldexpf(__uint_as_float(v[q * 8 + e]), -ex)) << (4 * e);
        w4[q] = wd;
      }
      uint4* dst = reinterpret_cast<uint4*>(p.q_fp4 + ((size_t)t * p.H_I + h) * 64 + 16 * sb);
      *dst = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      sf_word |= (uint32_t)(ex + 127) << (8 * sb);
      if (p.dbg) {
        float4* dd = reinterpret_cast<float4*>(p.dbg + ((size_t)t * p.H_I + h) * 128 + 32 * sb);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          dd[q] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                              __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
      }
    }
    if (ok && t < p.T)
      *reinterpret_cast<uint32_t*>(p.q_sf + ((size_t)t * p.H_I + h) * 4) = sf_word;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

cudaError_t launch_iquery(const csa_iquery_args& a, const CUtensorMap& cmap,
                          const CUtensorMap& wmap, cudaStream_t stream) {
  IqParams p{a.T, a.r, a.H_I, a.q_fp4, a.q_sf, a.dbg, a.dev_status};
  const size_t smem = sizeof(IqSmem) + 1024;
  static std::atomic<uint64_t> configured{0};
  if (cudaError_t e = configure_smem_once(iquery_kernel, smem, configured);
      e != cudaSuccess)
    return e;
  dim3 grid((a.T + kIqTile - 1) / kIqTile, a.H_I);
  return launch_pdl(iquery_kernel, grid, dim3(kIqThreads), smem, stream, cmap, wmap, p);
}

}  // namespace csa
