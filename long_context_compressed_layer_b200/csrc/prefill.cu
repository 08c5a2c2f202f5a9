// Per-query inputs of a causal CSA prefill (cyqw.cn DeepSeek-V4 walkthrough §2.2: each
// new token is a query over the compressed entries that are complete at its position and
// over the 128 most recent uncompressed tokens; §3.5: the window of the prefix arrives as
// state).
//
// prefill_prep_kernel writes, for the T new tokens of one sequence:
//   n_all[r]  = the entries eligible at position t = P + r: floor((t + 1) / m) when the
//              block closing at t counts, floor(t / m) under the strict reading (only
//              blocks completed before t);
//   pos_all[r] = P + r;
//   lin[i], i = 0 .. T + 126: the window row of position P - 127 + i in consecutive order,
//     taken from the prefix ring swa_prefix[p % 128] for p < P (rows of negative
//     positions are never read and are left as they are), and for p >= P formed from the
//     token itself: RMSNorm (fp32, eps, optional weight) of a[p - P], RoPE at position p
//     on the interleaved pairs of dims 448..511, rounded to BF16. The rows are stored
//     widened to FP16 (exact for the BF16 values of normalised rows), the form the
//     attention kernel stages.
// One warp per row; lane l owns dims 16l .. 16l + 15 (two 16-byte loads and stores), so a
// 1 KB row moves in one coalesced pass. The squares are summed per lane, then by a fixed
// butterfly, so the result does not depend on scheduling.
#include "common.cuh"

namespace csa {

// 8 BF16 values -> 8 FP16 values (the same conversion the attention staging applies)
__device__ __forceinline__ uint4 bf16x8_widen(uint4 v) {
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e)
    w[e] = pack_half2(bf16_bits_to_f32(w[e] & 0xFFFF), bf16_bits_to_f32(w[e] >> 16));
  return make_uint4(w[0], w[1], w[2], w[3]);
}

struct PrepParams {
  int64_t P;
  int T, m, strict;
  float eps, rope_base;
  const uint16_t* a;
  const float* norm_w;
  const uint16_t* swa_prefix;
  __half* lin;
  int32_t* n_all;
  int32_t* pos_all;
};

__global__ void __launch_bounds__(256) prefill_prep_kernel(PrepParams p) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gtid < p.T) {
    p.n_all[gtid] = (int32_t)((p.P + gtid + (p.strict ? 0 : 1)) / p.m);
    p.pos_all[gtid] = (int32_t)(p.P + gtid);
  }
  const int64_t i = (int64_t)blockIdx.x * (blockDim.x / 32) + warp;
  if (i >= (int64_t)p.T + kWin - 1) return;
  const int64_t pp = p.P - (kWin - 1) + i;
  uint4* dst = reinterpret_cast<uint4*>(p.lin + i * kD + 16 * lane);
  if (pp < 0) return;
  if (pp < p.P) {
    const uint4* src = reinterpret_cast<const uint4*>(p.swa_prefix + (pp % kWin) * kD + 16 * lane);
    dst[0] = bf16x8_widen(src[0]);
    dst[1] = bf16x8_widen(src[1]);
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(p.a + (pp - p.P) * kD + 16 * lane);
  const uint4 v0 = src[0], v1 = src[1];
  const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  float y[16];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    y[2 * e] = bf16_bits_to_f32(w[e] & 0xFFFF);
    y[2 * e + 1] = bf16_bits_to_f32(w[e] >> 16);
  }
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < 16; ++e) ss = fmaf(y[e], y[e], ss);
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = __fdiv_rn(1.f, sqrtf(ss / (float)kD + p.eps));
  const int d0 = 16 * lane;
#pragma unroll
  for (int e = 0; e < 16; ++e) y[e] = y[e] * inv * (p.norm_w ? __ldg(p.norm_w + d0 + e) : 1.f);
  if (d0 >= kNope) {
#pragma unroll
    for (int e = 0; e < 16; e += 2) {
      float cs, sn;
      rope_cos_sin((double)pp, (d0 + e - kNope) >> 1, (double)p.rope_base, &cs, &sn);
      const float x0 = y[e], x1 = y[e + 1];
      y[e] = x0 * cs - x1 * sn;
      y[e + 1] = x0 * sn + x1 * cs;
    }
  }
  uint32_t o[8];
#pragma unroll
  for (int e = 0; e < 8; ++e)  // the BF16 window value, then its exact FP16 form
    o[e] = pack_half2(bf16_bits_to_f32(f32_to_bf16_bits(y[2 * e])),
                      bf16_bits_to_f32(f32_to_bf16_bits(y[2 * e + 1])));
  dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
  dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
}

cudaError_t launch_prefill_prep(const csa_prefill_args& a, __half* lin, int32_t* n_all,
                                int32_t* pos_all, cudaStream_t stream) {
  PrepParams p{a.P, a.T, a.m, a.strict_eligibility, a.eps, a.rope_base, a.a, a.norm_w,
               a.swa_prefix, lin, n_all, pos_all};
  const int64_t rows = (int64_t)a.T + kWin - 1;
  const int64_t blocks_rows = (rows + 7) / 8, blocks_ids = ((int64_t)a.T + 255) / 256;
  const int64_t blocks = blocks_rows > blocks_ids ? blocks_rows : blocks_ids;
  return launch_pdl(prefill_prep_kernel, dim3((unsigned)blocks), dim3(256), 0, stream, p);
}

}  // namespace csa

namespace csa {

// Paged prefill (csa_pages in csa_prefill_args): the call runs on a contiguous staging copy
// of the sequence's cache. page_gather_kernel copies entries 0 .. n_kv-1 (rows and scales)
// and the keys of entries 0 .. n_keys-1 (rows, and the scale group of every 128 entries)
// from their pages; page_scatter_kernel copies the rows and scales of entries
// j0 .. j1-1 (the ones the call compressed) back to their pages. One warp per entry.
__global__ void __launch_bounds__(256) page_gather_kernel(PageMap pm, const uint8_t* kv,
                                                          const float* kv_scale,
                                                          const uint8_t* k_fp4,
                                                          const uint8_t* k_sf, uint8_t* kv_c,
                                                          float* sc_c, uint8_t* kf_c,
                                                          uint8_t* ksf_c, int64_t n_kv,
                                                          int64_t n_keys, int32_t* dev_status) {
  pdl_wait();
  pdl_trigger();
  const int64_t j = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (j >= n_kv && j >= n_keys) return;
  const int64_t e = page_entry(pm, 0, j);
  if (e < 0) {
    if (lane == 0) report(dev_status, CSA_ERR_DEVICE);
    return;
  }
  if (j < n_kv) {
    const uint4* src = reinterpret_cast<const uint4*>(kv + (size_t)e * kRow);
    uint4* dst = reinterpret_cast<uint4*>(kv_c + (size_t)j * kRow);
    for (int u = lane; u < kRow / 16; u += 32) dst[u] = src[u];
    if (lane == 0) sc_c[j] = kv_scale[e];
  }
  if (j < n_keys) {
    if (lane < 4)
      reinterpret_cast<uint4*>(kf_c + (size_t)j * 64)[lane] =
          reinterpret_cast<const uint4*>(k_fp4 + (size_t)e * 64)[lane];
    if ((j & 127) == 0)  // the group's 512 scale bytes (a page holds whole groups)
      reinterpret_cast<uint4*>(ksf_c + (size_t)(j / 128) * 512)[lane] =
          reinterpret_cast<const uint4*>(k_sf + (size_t)(e / 128) * 512)[lane];
  }
}

__global__ void __launch_bounds__(256) page_scatter_kernel(PageMap pm, const uint8_t* kv_c,
                                                           const float* sc_c, uint8_t* kv,
                                                           float* kv_scale, int64_t j0,
                                                           int64_t j1, int32_t* dev_status) {
  pdl_wait();
  pdl_trigger();
  const int64_t j = j0 + (((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (j >= j1) return;
  const int64_t e = page_entry(pm, 0, j);
  if (e < 0) {
    if (lane == 0) report(dev_status, CSA_ERR_DEVICE);
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(kv_c + (size_t)j * kRow);
  uint4* dst = reinterpret_cast<uint4*>(kv + (size_t)e * kRow);
  for (int u = lane; u < kRow / 16; u += 32) dst[u] = src[u];
  if (lane == 0) kv_scale[e] = sc_c[j];
}

cudaError_t launch_page_gather(const PageMap& pm, const uint8_t* kv, const float* kv_scale,
                               const uint8_t* k_fp4, const uint8_t* k_sf, uint8_t* kv_c,
                               float* sc_c, uint8_t* kf_c, uint8_t* ksf_c, int64_t n_kv,
                               int64_t n_keys, int32_t* dev_status, cudaStream_t stream) {
  const int64_t n = n_kv > n_keys ? n_kv : n_keys;
  if (n <= 0) return cudaSuccess;
  return launch_pdl(page_gather_kernel, dim3((unsigned)((n + 7) / 8)), dim3(256), 0, stream, pm,
                    kv, kv_scale, k_fp4, k_sf, kv_c, sc_c, kf_c, ksf_c, n_kv, n_keys,
                    dev_status);
}

cudaError_t launch_page_scatter(const PageMap& pm, const uint8_t* kv_c, const float* sc_c,
                                uint8_t* kv, float* kv_scale, int64_t j0, int64_t j1,
                                int32_t* dev_status, cudaStream_t stream) {
  if (j1 <= j0) return cudaSuccess;
  return launch_pdl(page_scatter_kernel, dim3((unsigned)((j1 - j0 + 7) / 8)), dim3(256), 0,
                    stream, pm, kv_c, sc_c, kv, kv_scale, j0, j1, dev_status);
}

}  // namespace csa
