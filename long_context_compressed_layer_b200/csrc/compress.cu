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

// One entry from its block: the gated merge of the own block (m tokens of a / za, logits
// + bias[r]) and, when pb != nullptr, the previous block (m tokens of pb / pz, logits +
// bias[m + r]); RMSNorm; RoPE on the last 64 dims at position pos; the split store into
// dst (576 bytes) and *dst_scale; y before quantisation to dbg when given. Token rows are
// kD apart. 128 threads, thread i owning dims 4i .. 4i+3.
__device__ __forceinline__ void compress_block(const uint16_t* own_a, const float* own_za,
                                               const uint16_t* pb, const float* pz, int m,
                                               const float* bias, const float* norm_w,
                                               float eps, int64_t pos, float rope_base,
                                               uint8_t* dst, float* dst_scale, float* dbg,
                                               float* red, float (*rot)[2]) {
  const int tid = threadIdx.x, d0 = 4 * tid;
  if (tid < 32) {  // RoPE angle of the entry's block-start position, in double precision
    float c, s;
    rope_cos_sin((double)pos, tid, (double)rope_base, &c, &s);
    rot[tid][0] = c;
    rot[tid][1] = s;
  }

  Online4 acc;
  acc.init();
  for (int r = 0; r < m; ++r) {  // own block: a with za + bias[r]
    const size_t o = (size_t)r * kD + d0;
    const uint2 xb = *reinterpret_cast<const uint2*>(own_a + o);
    const float4 z = *reinterpret_cast<const float4*>(own_za + o);
    acc.add(xb, z, __ldg(bias + r));
  }
  if (pb) {  // previous block: b with zb + bias[m + r]
    for (int r = 0; r < m; ++r) {
      const uint2 xb = *reinterpret_cast<const uint2*>(pb + (size_t)r * kD + d0);
      const float4 z = *reinterpret_cast<const float4*>(pz + (size_t)r * kD + d0);
      acc.add(xb, z, __ldg(bias + m + r));
    }
  }
  float y[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) y[c] = __fdiv_rn(acc.num[c], acc.den[c]);

  // RMSNorm
  const float ss = block_sum_128(y[0] * y[0] + y[1] * y[1] + y[2] * y[2] + y[3] * y[3], red);
  const float inv = __fdiv_rn(1.f, sqrtf(ss / (float)kD + eps));
#pragma unroll
  for (int c = 0; c < 4; ++c) y[c] = y[c] * inv * (norm_w ? __ldg(norm_w + d0 + c) : 1.f);

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

  if (dbg) *reinterpret_cast<float4*>(dbg + d0) = make_float4(y[0], y[1], y[2], y[3]);

  // Split store: E4M3 with one fp32 scale for dims 0..447, BF16 for 448..511.
  float am = 0.f;
  if (d0 < kNope) am = fmaxf(fmaxf(fabsf(y[0]), fabsf(y[1])), fmaxf(fabsf(y[2]), fabsf(y[3])));
  const float amax = block_max_128(am, red);
  const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
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
  if (tid == 0) *dst_scale = scale;
}

__global__ void __launch_bounds__(128) compress_kernel(csa_compress_args a, int N) {
  __shared__ float red[4];
  __shared__ float rot[32][2];
  const int i = blockIdx.x, b = blockIdx.y;
  const int m = a.m;
  pdl_wait();
  pdl_trigger();
  const size_t tok0 = (size_t)b * a.T + (size_t)m * i;
  const uint16_t* pb = nullptr;
  const float* pz = nullptr;
  if (a.overlap) {
    if (i > 0) {
      pb = a.b + (tok0 - m) * kD;
      pz = a.zb + (tok0 - m) * kD;
    } else if (a.pos0 > 0) {
      pb = a.prev_b + (size_t)b * m * kD;
      pz = a.prev_zb + (size_t)b * m * kD;
    }
  }
  const size_t row = (size_t)b * a.Nmax + (size_t)(a.pos0 / m) + i;
  compress_block(a.a + tok0 * kD, a.za + tok0 * kD, pb, pz, m, a.bias, a.norm_w, a.eps,
                 a.pos0 + (int64_t)m * i, a.rope_base, a.kv + row * kRow, a.kv_scale + row,
                 a.dbg ? a.dbg + ((size_t)b * N + i) * kD : nullptr, red, rot);
}

// Indexer-key compression: the same gated merge on the 128-dim indexer-key stream (no norm,
// no RoPE), stored as MXFP4 for the FP4 indexer (walkthrough §3.4). One CTA of 128
// threads per entry, thread d owning dim d, so each warp holds one 32-element block:
// the block maximum is a warp reduction, the shared exponent floor(log2 amax) - 2 comes
// from frexpf, scaling by a power of two is exact, and each element is rounded to the
// nearest E2M1 value (ties to the even code, saturating at 6). Lanes pair their nibbles
// with a shuffle (element 2i in the low nibble).
// One MXFP4 indexer key from its block (own rows own_a / own_za, previous rows pb / pz or
// none; rows CSA_INDEX_DIM apart): 64 code bytes to dst_codes, the four block scales to
// the grouped scale bytes of entry `row` in sf_group_base, y to dbg when given. 128
// threads, thread d owning dim d.
__device__ __forceinline__ void ikey_block(const uint16_t* own_a, const float* own_za,
                                           const uint16_t* pb, const float* pz, int m,
                                           const float* bias, uint8_t* dst_codes,
                                           uint8_t* sf_base, int64_t row, float* dbg) {
  constexpr int kDI = CSA_INDEX_DIM;
  const int d = threadIdx.x, lane = d & 31, s = d >> 5;
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
  for (int r = 0; r < m; ++r) add(own_a[(size_t)r * kDI + d], own_za[(size_t)r * kDI + d] + __ldg(bias + r));
  if (pb)
    for (int r = 0; r < m; ++r)
      add(pb[(size_t)r * kDI + d], pz[(size_t)r * kDI + d] + __ldg(bias + m + r));
  const float y = __fdiv_rn(num, den);
  if (dbg) dbg[d] = y;
  float amax = fabsf(y);
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const int e = mxfp4_exponent(amax);
  const uint32_t nib = e2m1_code(ldexpf(y, -e));
  const uint32_t hi = __shfl_down_sync(0xffffffffu, nib, 1);
  if ((lane & 1) == 0) dst_codes[16 * s + (lane >> 1)] = (uint8_t)(nib | (hi << 4));
  if (lane == 0) {
    const int64_t g = row / 128, r = row % 128;
    sf_base[g * 512 + 16 * (r % 32) + 4 * (r / 32) + s] = (uint8_t)(e + 127);
  }
}

__global__ void __launch_bounds__(128) ikey_compress_kernel(csa_ikey_args a, int N) {
  const int i = blockIdx.x, b = blockIdx.y;
  constexpr int kDI = CSA_INDEX_DIM;
  const int m = a.m;
  pdl_wait();
  pdl_trigger();
  const size_t tok0 = (size_t)b * a.T + (size_t)m * i;
  const uint16_t* pb = nullptr;
  const float* pz = nullptr;
  if (a.overlap) {
    if (i > 0) {
      pb = a.b + (tok0 - m) * kDI;
      pz = a.zb + (tok0 - m) * kDI;
    } else if (a.pos0 > 0) {
      pb = a.prev_b + (size_t)b * m * kDI;
      pz = a.prev_zb + (size_t)b * m * kDI;
    }
  }
  const int64_t row = a.pos0 / m + i;
  ikey_block(a.a + tok0 * kDI, a.za + tok0 * kDI, pb, pz, m, a.bias,
             a.k_fp4 + ((size_t)b * a.Nmax + row) * (kDI / 2),
             a.k_sf + (size_t)b * (a.Nmax / 128) * 512, row,
             a.dbg ? a.dbg + ((size_t)b * N + i) * kDI : nullptr);
}

cudaError_t launch_ikey_compress(const csa_ikey_args& a, cudaStream_t stream) {
  const int N = a.T / a.m;
  if (N == 0 || a.B == 0) return cudaSuccess;
  return launch_pdl(ikey_compress_kernel, dim3(N, a.B), dim3(128), 0, stream, a, N);
}

// Decode-step state update (walkthrough §3.5: the state cache holds the window tokens and
// the tail of the unfinished block; complete blocks go to the compressed cache). One CTA
// per sequence appends its new token t: the token joins the tail of block t / m (a / za
// at slot t % m; b / zb in the two-block ring slot (t / m) & 1, which the next block reads
// as its previous block), its window row (RMSNorm, RoPE at t, BF16) overwrites ring row
// t % 128, and when t closes its block the entry is compressed from the tails exactly as
// csa_compress would, n_entries becomes t / m + 1, and the optional indexer-key stream is
// compressed to its MXFP4 key the same way.
__global__ void __launch_bounds__(128) append_kernel(csa_append_args a) {
  __shared__ float red[4];
  __shared__ float rot[32][2];
  constexpr int kDI = CSA_INDEX_DIM;
  const int b = blockIdx.x, tid = threadIdx.x, d0 = 4 * tid, m = a.m;
  pdl_wait();
  pdl_trigger();
  const int64_t t = a.pos[b];
  if (t < 0 || t / m >= a.Nmax) {
    if (tid == 0) report(a.dev_status, CSA_ERR_DEVICE);
    return;
  }
  const int r = (int)(t % m);
  const int64_t blk = t / m;
  const size_t tail = (size_t)b * m * kD;                 // [B][m][512]
  const size_t ring = ((size_t)b * 2 + (blk & 1)) * m * kD;  // [B][2][m][512]
  // the token joins the tails
  const uint2 av = *reinterpret_cast<const uint2*>(a.a + (size_t)b * kD + d0);
  *reinterpret_cast<uint2*>(a.tail_a + tail + (size_t)r * kD + d0) = av;
  *reinterpret_cast<float4*>(a.tail_za + tail + (size_t)r * kD + d0) =
      *reinterpret_cast<const float4*>(a.za + (size_t)b * kD + d0);
  if (a.overlap) {
    *reinterpret_cast<uint2*>(a.tail_b + ring + (size_t)r * kD + d0) =
        *reinterpret_cast<const uint2*>(a.b + (size_t)b * kD + d0);
    *reinterpret_cast<float4*>(a.tail_zb + ring + (size_t)r * kD + d0) =
        *reinterpret_cast<const float4*>(a.zb + (size_t)b * kD + d0);
  }
  if (a.ia) {
    const size_t itail = (size_t)b * m * kDI, iring = ((size_t)b * 2 + (blk & 1)) * m * kDI;
    a.itail_a[itail + (size_t)r * kDI + tid] = a.ia[(size_t)b * kDI + tid];
    a.itail_za[itail + (size_t)r * kDI + tid] = a.iza[(size_t)b * kDI + tid];
    a.itail_b[iring + (size_t)r * kDI + tid] = a.ib[(size_t)b * kDI + tid];
    a.itail_zb[iring + (size_t)r * kDI + tid] = a.izb[(size_t)b * kDI + tid];
  }
  {  // the window row of t: RMSNorm then RoPE at t, in BF16
    float y[4] = {bf16_bits_to_f32(av.x & 0xFFFF), bf16_bits_to_f32(av.x >> 16),
                  bf16_bits_to_f32(av.y & 0xFFFF), bf16_bits_to_f32(av.y >> 16)};
    const float ss = block_sum_128(y[0] * y[0] + y[1] * y[1] + y[2] * y[2] + y[3] * y[3], red);
    const float inv = __fdiv_rn(1.f, sqrtf(ss / (float)kD + a.eps));
#pragma unroll
    for (int c = 0; c < 4; ++c) y[c] = y[c] * inv * (a.norm_w ? __ldg(a.norm_w + d0 + c) : 1.f);
    if (d0 >= kNope) {
#pragma unroll
      for (int c = 0; c < 4; c += 2) {
        float cs, sn;
        rope_cos_sin((double)t, (d0 + c - kNope) >> 1, (double)a.rope_base, &cs, &sn);
        const float x0 = y[c], x1 = y[c + 1];
        y[c] = x0 * cs - x1 * sn;
        y[c + 1] = x0 * sn + x1 * cs;
      }
    }
    uint2 v;
    v.x = (uint32_t)f32_to_bf16_bits(y[0]) | ((uint32_t)f32_to_bf16_bits(y[1]) << 16);
    v.y = (uint32_t)f32_to_bf16_bits(y[2]) | ((uint32_t)f32_to_bf16_bits(y[3]) << 16);
    *reinterpret_cast<uint2*>(a.swa + ((size_t)b * kWin + t % kWin) * kD + d0) = v;
  }
  if (r != m - 1) return;  // uniform: the block is still open
  // the entry's place in the cache (contiguous, or the slot of its page)
  const int64_t e = page_entry(page_map(a.pages, a.Nmax), b, blk);
  if (e < 0) {
    if (tid == 0) report(a.dev_status, CSA_ERR_DEVICE);
    return;
  }
  __syncthreads();  // every thread's tail rows are written before any is read
  const bool prev = a.overlap && blk > 0;
  const size_t pring = ((size_t)b * 2 + ((blk + 1) & 1)) * m * kD;
  compress_block(a.tail_a + tail, a.tail_za + tail, prev ? a.tail_b + pring : nullptr,
                 prev ? a.tail_zb + pring : nullptr, m, a.bias, a.norm_w, a.eps, blk * m,
                 a.rope_base, a.kv + (size_t)e * kRow, a.kv_scale + e, nullptr, red, rot);
  if (a.ia) {
    const size_t itail = (size_t)b * m * kDI, ipring = ((size_t)b * 2 + ((blk + 1) & 1)) * m * kDI;
    ikey_block(a.itail_a + itail, a.itail_za + itail, prev ? a.itail_b + ipring : nullptr,
               prev ? a.itail_zb + ipring : nullptr, m, a.ibias,
               a.k_fp4 + (size_t)e * (kDI / 2), a.k_sf, e, nullptr);
  }
  if (tid == 0) a.n_entries[b] = (int32_t)(blk + 1);
}

cudaError_t launch_append(const csa_append_args& a, cudaStream_t stream) {
  if (a.B == 0) return cudaSuccess;
  return launch_pdl(append_kernel, dim3(a.B), dim3(128), 0, stream, a);
}

cudaError_t launch_compress(const csa_compress_args& a, cudaStream_t stream) {
  const int N = a.T / a.m;
  if (N == 0 || a.B == 0) return cudaSuccess;
  dim3 grid(N, a.B);
  return launch_pdl(compress_kernel, grid, dim3(128), 0, stream, a, N);
}

}  // namespace csa
