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
