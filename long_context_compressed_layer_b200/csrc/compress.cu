// Gated-softmax block compression of the KV stream into stored CSA/HCA entries
// (cyqw.cn DeepSeek-V4 walkthrough §2.2: two independent KV sequences merged with
// softmax-normalised gate weights, overlapping adjacent blocks; chooseai.net §一:
// positional bias in the merge, RoPE dims BF16 and the rest FP8; walkthrough §2.3:
// RMSNorm on the KV entries).
//
// One CTA of 128 threads produces one entry; thread i owns dims 4i .. 4i+3, so every
// token row is read with one 8-byte (bf16) and one 16-byte (fp32 logit) load per thread,
// fully coalesced. The softmax over the 2m (or m) candidates of each dim is an online
// max/sum in fp32. RMSNorm and the E4M3 amax are block reductions. The kernel is a pure
// HBM stream: for CSA it reads 2m token rows of a/b (1 KB each) and za/zb (2 KB each)
// per entry and writes 580 bytes.
#include "common.cuh"

namespace csa {

__device__ __forceinline__ float block_sum_128(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  return red[0] + red[1] + red[2] + red[3];
}

__device__ __forceinline__ float block_max_128(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  return fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
}

struct Online4 {
  float mx[4], den[4], num[4];
  __device__ void init() {
#pragma unroll
    for (int c = 0; c < 4; ++c) { mx[c] = -INFINITY; den[c] = 0.f; num[c] = 0.f; }
  }
  // Add one candidate token (4 values, 4 logits) to the running softmax of each dim.
  __device__ void add(const uint2 xb, const float4 z, float bias) {
    const float x[4] = {bf16_bits_to_f32(xb.x & 0xFFFF), bf16_bits_to_f32(xb.x >> 16),
                        bf16_bits_to_f32(xb.y & 0xFFFF), bf16_bits_to_f32(xb.y >> 16)};
    const float l[4] = {z.x + bias, z.y + bias, z.z + bias, z.w + bias};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (l[c] > mx[c]) {
        const float r = expf(mx[c] - l[c]);  // 0 on the first candidate
        den[c] = den[c] * r + 1.f;
        num[c] = num[c] * r + x[c];
        mx[c] = l[c];
      } else {
        const float g = expf(l[c] - mx[c]);
        den[c] += g;
        num[c] += g * x[c];
      }
    }
  }
};

__global__ void __launch_bounds__(128) compress_kernel(csa_compress_args a, int N) {
  __shared__ float red[4];
  __shared__ float rot[32][2];
  const int i = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int m = a.m;
  pdl_wait();
  pdl_trigger();
  const size_t tok0 = (size_t)b * a.T + (size_t)m * i;
  const int d0 = 4 * tid;

  if (tid < 32) {  // RoPE angle of the entry's block-start position, in double precision
    float c, s;
    rope_cos_sin((double)(a.pos0 + (int64_t)m * i), tid, (double)a.rope_base, &c, &s);
    rot[tid][0] = c;
    rot[tid][1] = s;
  }

  Online4 acc;
  acc.init();
  for (int r = 0; r < m; ++r) {  // own block: a with za + bias[r]
    const size_t o = (tok0 + r) * kD + d0;
    const uint2 xb = *reinterpret_cast<const uint2*>(a.a + o);
    const float4 z = *reinterpret_cast<const float4*>(a.za + o);
    acc.add(xb, z, __ldg(a.bias + r));
  }
  if (a.overlap) {  // previous block: b with zb + bias[m + r]
    const uint16_t* pb = nullptr;
    const float* pz = nullptr;
    if (i > 0) {
      pb = a.b + (tok0 - m) * kD;
      pz = a.zb + (tok0 - m) * kD;
    } else if (a.pos0 > 0) {
      pb = a.prev_b + (size_t)b * m * kD;
      pz = a.prev_zb + (size_t)b * m * kD;
    }
    if (pb) {
      for (int r = 0; r < m; ++r) {
        const uint2 xb = *reinterpret_cast<const uint2*>(pb + (size_t)r * kD + d0);
        const float4 z = *reinterpret_cast<const float4*>(pz + (size_t)r * kD + d0);
        acc.add(xb, z, __ldg(a.bias + m + r));
      }
    }
  }
  float y[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) y[c] = __fdiv_rn(acc.num[c], acc.den[c]);

  // RMSNorm
  const float ss = block_sum_128(y[0] * y[0] + y[1] * y[1] + y[2] * y[2] + y[3] * y[3], red);
  const float inv = __fdiv_rn(1.f, sqrtf(ss / (float)kD + a.eps));
#pragma unroll
  for (int c = 0; c < 4; ++c) y[c] = y[c] * inv * (a.norm_w ? __ldg(a.norm_w + d0 + c) : 1.f);

  // RoPE on the interleaved pairs of dims 448..511
  if (d0 >= kNope) {
#pragma unroll
    for (int c = 0; c < 4; c += 2) {
      const int j = (d0 + c - kNope) >> 1;
      const float cs = rot[j][0], sn = rot[j][1];
      const float x0 = y[c], x1 = y[c + 1];
      y[c] = x0 * cs - x1 * sn;
      y[c + 1] = x0 * sn + x1 * cs;
    }
  }

  const size_t row = (size_t)b * a.Nmax + (size_t)(a.pos0 / m) + i;
  if (a.dbg) {
    float4 v = make_float4(y[0], y[1], y[2], y[3]);
    *reinterpret_cast<float4*>(a.dbg + ((size_t)b * N + i) * kD + d0) = v;
  }

  // Split store: E4M3 with one fp32 scale for dims 0..447, BF16 for 448..511.
  float am = 0.f;
  if (d0 < kNope) am = fmaxf(fmaxf(fabsf(y[0]), fabsf(y[1])), fmaxf(fabsf(y[2]), fabsf(y[3])));
  const float amax = block_max_128(am, red);
  const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  uint8_t* dst = a.kv + row * kRow;
  if (d0 < kNope) {
    uint32_t packed = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c)
      packed |= (uint32_t)f32_to_e4m3_sat(__fdiv_rn(y[c], scale)) << (8 * c);
    *reinterpret_cast<uint32_t*>(dst + d0) = packed;
  } else {
    uint2 v;
    v.x = (uint32_t)f32_to_bf16_bits(y[0]) | ((uint32_t)f32_to_bf16_bits(y[1]) << 16);
    v.y = (uint32_t)f32_to_bf16_bits(y[2]) | ((uint32_t)f32_to_bf16_bits(y[3]) << 16);
    *reinterpret_cast<uint2*>(dst + kNope + 2 * (d0 - kNope)) = v;
  }
  if (tid == 0) a.kv_scale[row] = scale;
}

// Indexer-key compression: the same gated merge on the 128-dim indexer-key stream (no norm,
// no RoPE), stored as MXFP4 for the FP4 indexer (walkthrough §3.4). One CTA of 128
// threads per entry, thread d owning dim d, so each warp holds one 32-element block:
// the block maximum is a warp reduction, the shared exponent floor(log2 amax) - 2 comes
// from frexpf, scaling by a power of two is exact, and each element is rounded to the
// nearest E2M1 value (ties to the even code, saturating at 6). Lanes pair their nibbles
// with a shuffle (element 2i in the low nibble).
__global__ void __launch_bounds__(128) ikey_compress_kernel(csa_ikey_args a, int N) {
  const int i = blockIdx.x, b = blockIdx.y, d = threadIdx.x, lane = d & 31, s = d >> 5;
  constexpr int kDI = CSA_INDEX_DIM;
  const int m = a.m;
  pdl_wait();
  pdl_trigger();
  const size_t tok0 = (size_t)b * a.T + (size_t)m * i;
  float mx = -INFINITY, den = 0.f, num = 0.f;
  auto add = [&](uint16_t xb, float z) {
    const float x = bf16_bits_to_f32(xb);
    if (z > mx) {
      const float r = expf(mx - z);  // 0 on the first candidate
      den = den * r + 1.f;
      num = num * r + x;
      mx = z;
    } else {
      const float g = expf(z - mx);
      den += g;
      num += g * x;
    }
  };
  for (int r = 0; r < m; ++r) {
    const size_t o = (tok0 + r) * kDI + d;
    add(a.a[o], a.za[o] + __ldg(a.bias + r));
  }
  if (a.overlap) {
    const uint16_t* pb = nullptr;
    const float* pz = nullptr;
    if (i > 0) {
      pb = a.b + (tok0 - m) * kDI;
      pz = a.zb + (tok0 - m) * kDI;
    } else if (a.pos0 > 0) {
      pb = a.prev_b + (size_t)b * m * kDI;
      pz = a.prev_zb + (size_t)b * m * kDI;
    }
    if (pb)
      for (int r = 0; r < m; ++r) add(pb[(size_t)r * kDI + d], pz[(size_t)r * kDI + d] + __ldg(a.bias + m + r));
  }
  const float y = __fdiv_rn(num, den);
  if (a.dbg) a.dbg[((size_t)b * N + i) * kDI + d] = y;
  float amax = fabsf(y);
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const int e = mxfp4_exponent(amax);
  const uint32_t nib = e2m1_code(ldexpf(y, -e));
  const uint32_t hi = __shfl_down_sync(0xffffffffu, nib, 1);
  const int64_t row = a.pos0 / m + i;
  if ((lane & 1) == 0)
    a.k_fp4[((size_t)b * a.Nmax + row) * (kDI / 2) + 16 * s + (lane >> 1)] = (uint8_t)(nib | (hi << 4));
  if (lane == 0) {
    const int64_t g = row / 128, r = row % 128;
    a.k_sf[(size_t)b * (a.Nmax / 128) * 512 + g * 512 + 16 * (r % 32) + 4 * (r / 32) + s] =
        (uint8_t)(e + 127);
  }
}

cudaError_t launch_ikey_compress(const csa_ikey_args& a, cudaStream_t stream) {
  const int N = a.T / a.m;
  if (N == 0 || a.B == 0) return cudaSuccess;
  return launch_pdl(ikey_compress_kernel, dim3(N, a.B), dim3(128), 0, stream, a, N);
}

cudaError_t launch_compress(const csa_compress_args& a, cudaStream_t stream) {
  const int N = a.T / a.m;
  if (N == 0 || a.B == 0) return cudaSuccess;
  dim3 grid(N, a.B);
  return launch_pdl(compress_kernel, grid, dim3(128), 0, stream, a, N);
}

}  // namespace csa
