// Shared-KV MQA decode over compressed entries plus the sliding window, with the sink
// logit in the softmax denominator ("DeepSeek-V4：百万上下文的工程答案", Hybrid Attention:
// shared key-value MQA, Attention sink; cyqw.cn DeepSeek-V4 walkthrough §2.2: the 128
// most recent uncompressed tokens join the core attention; Partial RoPE: the output is
// de-rotated by the query position).
//
// The rows a query attends to form one list: the selected entries (CSA) or all eligible
// entries (HCA), then the 128 window tokens t-127 .. t. The list is cut into chunks of
// 64 rows. attn_chunk_kernel handles one (sequence, chunk), or one (sequence, chunk, half
// of the output dims) when twice the chunks still fit one wave of CTAs on the SMs (then a
// chunk's two CTAs compute the same S and softmax):
//   - Q [H heads x 512] arrives by TMA (128-byte swizzle, K-major), padded to 128 rows,
//     and is widened in place from BF16 to FP16 (exact for |q| >= 2^-14);
//   - the 64 rows are gathered and dequantised to FP16 in shared memory (E4M3 code x entry
//     scale, RoPE dims, window rows), in the same swizzled layout, which serves as K-major
//     B for S = Q V^T and as MN-major B for O = P V. FP16 (11 significant bits) rather
//     than BF16 (8) keeps the staging error well inside the output tolerance;
//   - tcgen05.mma kind::f16 computes S[128 x 64] in TMEM; one thread per head turns its row
//     into exp(tau*S - m) (fp32), keeps m and l = sum, and writes P as FP16 (K-major A);
//   - tcgen05.mma N = 256 products compute this CTA's halves of O[128 x 512] in TMEM (S's
//     columns are reused);
//   - O / l (FP16, [8-dim group][head][8] so every warp store covers 512 contiguous bytes),
//     m and l go to the workspace.
// attn_combine_kernel then merges the chunks of a sequence in fixed order with the sink,
// normalises, de-rotates the last 64 dims and stores BF16 (and lse). The chunk count
// depends only on k (CSA) or n (HCA), never on the batch, so results are batch-invariant.
#include "common.cuh"

namespace csa {

constexpr int kAtRows = 64;  // rows per chunk = N of the S MMA
constexpr int kAtThreads = 256;
struct AtSmem {
  uint8_t q[8][128 * 128];      // 8 K-blocks of [128 heads x 64 dims] fp16, 128-B swizzle
  uint8_t v[8][kAtRows * 128];  // 8 dim-blocks of [64 rows x 64 dims] fp16, 128-B swizzle
  uint8_t pm[128 * 128];        // P' [128 heads x 64 rows] fp16, 128-B swizzle
  const uint8_t* row[kAtRows];  // row source
  const float* scl[kAtRows];    // entry rows: address of the entry scale
  int kind[kAtRows];            // 0 invalid, 1 entry, 2 window row
  float scale[kAtRows];         // the row's factor (entry scale; 1 for window rows)
  float mx[2][128], sm[2][128]; // the two column halves' max and sum per head
  float inv_l[128];             // 1 / (chunk sum) per head
  uint64_t q_full, s_done, o_done;
  uint32_t tmem_base;
};

struct AtParams {
  int B, H, k, sparse, C;  // C = chunks per sequence in the workspace
  int64_t Nmax;
  const int32_t* pos;
  const int32_t* idx;
  const int32_t* n_entries;
  const uint8_t* kv;
  const float* kv_scale;
  const uint16_t* swa;
  const float* sink;
  float tau, rope_base;
  int derotate;
  uint16_t* out;
  float* lse;
  __half* part_o;  // [B][C][64][H][8]: chunk output / chunk sum, fp16, 8-dim groups
  float2* part_ml; // [B][C][H]: (chunk max logit, chunk sum)
  float* rot;      // [B][64]: cos, sin of -t theta_j per RoPE pair (chunk 0 writes them)
  int split;       // CTAs per chunk: 2 (each half of the output dims) or 1
  PageMap pm;         // where the entries live (contiguous or paged)
  int32_t* dev_status;
};

__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 v) {
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e)
    w[e] = pack_half2(bf16_bits_to_f32(w[e] & 0xFFFF), bf16_bits_to_f32(w[e] >> 16));
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// 8 BF16 values times f -> 8 FP16 values (one rounding of the fp32 product)
__device__ __forceinline__ uint4 bf16x8_scaled_to_f16x8(uint4 v, float f) {
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e)
    w[e] = pack_half2(bf16_bits_to_f32(w[e] & 0xFFFF) * f, bf16_bits_to_f32(w[e] >> 16) * f);
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// 16 E4M3 codes -> 16 FP16 values, exactly (every E4M3 value is an FP16 value): two packed
// conversions per 32-bit word, the lower code of each pair in the lower half
__device__ __forceinline__ void e4m3x16_codes_to_f16(uint4 raw, uint4* lo, uint4* hi) {
  const uint32_t in[4] = {raw.x, raw.y, raw.z, raw.w};
  uint32_t o[8];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __half2_raw a = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(in[e] & 0xFFFF), __NV_E4M3);
    const __half2_raw b = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(in[e] >> 16), __NV_E4M3);
    o[2 * e] = (uint32_t)a.x | ((uint32_t)a.y << 16);
    o[2 * e + 1] = (uint32_t)b.x | ((uint32_t)b.y << 16);
  }
  *lo = make_uint4(o[0], o[1], o[2], o[3]);
  *hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// 16 E4M3 codes x scale -> two 16-byte chunks of FP16 (one rounding of the fp32 product)
__device__ __forceinline__ void e4m3x16_to_f16(uint4 raw, float scl, uint4* lo, uint4* hi) {
  const uint32_t in[4] = {raw.x, raw.y, raw.z, raw.w};
  uint32_t o[8];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const uint32_t x = in[e];
    o[2 * e] = pack_half2(e4m3_to_f32((uint8_t)(x & 0xFF)) * scl,
                          e4m3_to_f32((uint8_t)((x >> 8) & 0xFF)) * scl);
    o[2 * e + 1] = pack_half2(e4m3_to_f32((uint8_t)((x >> 16) & 0xFF)) * scl,
                              e4m3_to_f32((uint8_t)(x >> 24)) * scl);
  }
  *lo = make_uint4(o[0], o[1], o[2], o[3]);
  *hi = make_uint4(o[4], o[5], o[6], o[7]);
}

__device__ __forceinline__ void store_v_chunk(AtSmem& s, int r, int ch, uint4 v) {
  *reinterpret_cast<uint4*>(&s.v[ch >> 3][r * 128 + (((ch & 7) ^ (r & 7)) << 4)]) = v;
}

__device__ __forceinline__ int at_rows_total(const AtParams& p, int n) {
  return (p.sparse ? p.k : n) + kWin;
}


// O / l of this CTA's NBLK column blocks of 32 (per warp: lane quadrant quad, blocks
// colh * NBLK ..), FP16, heads innermost; the next block loads from TMEM while the current
// one is stored
template <int NBLK>
__device__ __forceinline__ void store_partial(const AtParams& p, const AtSmem& s, uint32_t t_o,
                                              int b, int c, int dh, int quad, int colh,
                                              int tid) {
  const int hh = quad * 32 + (tid & 31);
  const float inv = s.inv_l[hh];
  const uint32_t ta0 = t_o + ((uint32_t)(quad * 32) << 16) + colh * NBLK * 32;
  uint32_t r[2][32];
  tmem_ld32(ta0, r[0]);
  tmem_ld_wait();
#pragma unroll
  for (int i = 0; i < NBLK; ++i) {
    if (i + 1 < NBLK) tmem_ld32(ta0 + (i + 1) * 32, r[(i + 1) & 1]);
    if (hh < p.H) {
      const uint32_t* x = r[i & 1];
      const int g0 = (dh * 8 + colh * NBLK + i) * 4;  // first 8-dim group of this block
#pragma unroll
      for (int e = 0; e < 32; e += 8) {
        uint4 v;
        v.x = pack_half2(__uint_as_float(x[e]) * inv, __uint_as_float(x[e + 1]) * inv);
        v.y = pack_half2(__uint_as_float(x[e + 2]) * inv, __uint_as_float(x[e + 3]) * inv);
        v.z = pack_half2(__uint_as_float(x[e + 4]) * inv, __uint_as_float(x[e + 5]) * inv);
        v.w = pack_half2(__uint_as_float(x[e + 6]) * inv, __uint_as_float(x[e + 7]) * inv);
        // heads innermost: the warp's 32 heads store 512 contiguous bytes
        *reinterpret_cast<uint4*>(
            p.part_o + ((((size_t)b * p.C + c) * 64 + g0 + e / 8) * p.H + hh) * 8) = v;
      }
    }
    tmem_ld_wait();
  }
}

// The staged row of entry r is v'_r = [codes (448 dims, exact in FP16) | rope dims / scale_r]
// with scale_r its entry scale, and a window row is itself with scale 1. Then
//   q . v_r = scale_r (q . v'_r)   and   sum_r p_r v_r = sum_r (p_r scale_r) v'_r,
// so the S product takes v' and the logits are multiplied by scale_r, and the P V product
// takes P' = p * scale_r. The 448 E4M3 dims enter the products exactly; only the 64 rope
// dims of entries are rounded (once, to FP16), where staging v_r itself would round all 448.
__global__ void __launch_bounds__(kAtThreads, 1)
    attn_chunk_kernel(const __grid_constant__ CUtensorMap qmap, AtParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  AtSmem& s = *reinterpret_cast<AtSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  // split = 2: CTA (2c + dh, b) is chunk c of sequence b for output dims [256 dh, +256) (S
  // and the softmax are computed by both CTAs of a chunk, with the same bits); split = 1:
  // CTA (c, b) computes all 512
  const int c = blockIdx.x / p.split, dh = p.split == 2 ? (int)(blockIdx.x & 1) : 0;
  const int b = blockIdx.y, tid = threadIdx.x;
  const int warp = tid >> 5;
  const int row0 = c * kAtRows;
  pdl_wait();
  pdl_trigger();
  // independent loads first: length, position and (CSA) this thread's selected index
  int n = p.n_entries[b];
  const int t = p.pos[b];
  int jsel = -1;
  if (p.sparse && tid < kAtRows && row0 + tid < p.k) jsel = p.idx[(size_t)b * p.k + row0 + tid];
  if (n < 0 || n > p.Nmax) {
    if (tid == 0) report(p.dev_status, CSA_ERR_DEVICE);
    n = n < 0 ? 0 : (int)p.Nmax;
  }
  const int rows_total = at_rows_total(p, n);
  if (row0 >= rows_total) return;  // uniform: this chunk does not exist for this sequence
  if (t < 0 && tid == 0) report(p.dev_status, CSA_ERR_DEVICE);
  const int nwin_first = p.sparse ? p.k : n;  // list index of the first window row

  if (tid == 0) {
    mbar_init(&s.q_full, 1);
    mbar_init(&s.s_done, 1);
    mbar_init(&s.o_done, 1);
    mbar_fence_init();
    prefetch_tensormap(&qmap);
    mbar_arrive_expect_tx(&s.q_full, (uint32_t)p.H * kD * 2);
    for (int blk = 0; blk < 8; ++blk) tma_load_2d(s.q[blk], &qmap, &s.q_full, blk * 64, b * p.H);
  }
  if (warp == 0) tmem_alloc(&s.tmem_base, 512);
  // Q rows H..127 are zero padding (generic-proxy writes, fenced below)
  if (p.H < 128) {
    for (int i = tid; i < 8 * (128 - p.H) * 8; i += kAtThreads) {
      const int blk = i / ((128 - p.H) * 8), rem = i % ((128 - p.H) * 8);
      *reinterpret_cast<uint4*>(&s.q[blk][p.H * 128 + rem * 16]) = make_uint4(0, 0, 0, 0);
    }
  }
  // row sources (the entry scale is fetched with the row data below)
  if (tid < kAtRows) {
    const int r = row0 + tid;
    int kind = 0;
    const uint8_t* src = nullptr;
    if (r < nwin_first) {
      const int j = p.sparse ? jsel : r;
      if (j >= 0 && j < n) {
        const int64_t e = page_entry(p.pm, b, j);
        if (e >= 0) {
          kind = 1;
          src = p.kv + (size_t)e * kRow;
          s.scl[tid] = p.kv_scale + e;
        } else {
          report(p.dev_status, CSA_ERR_DEVICE);
        }
      } else if (j != -1) {
        report(p.dev_status, CSA_ERR_DEVICE);
      }
    } else if (r < rows_total) {
      const int pp = t - (kWin - 1) + (r - nwin_first);
      if (pp >= 0) {
        kind = 2;
        src = reinterpret_cast<const uint8_t*>(p.swa + ((size_t)b * kWin + (pp % kWin)) * kD);
      }
    }
    s.kind[tid] = kind;
    s.row[tid] = src;
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  // gather: four threads per row; every thread issues all of its 16-byte pieces (and the
  // row's scale) before converting any
  {
    const int r = tid >> 2, qd = tid & 3;
    int kind = s.kind[r];
    const uint8_t* src = s.row[r];
    const int units = kind == 1 ? 36 : (kind == 2 ? 64 : 0);  // 16-byte pieces of the row
    float scl = kind == 1 ? __ldg(s.scl[r]) : 1.f;
    uint4 buf[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int u = qd + 4 * i;
      buf[i] = u < units ? __ldg(reinterpret_cast<const uint4*>(src + 16 * u))
                         : make_uint4(0, 0, 0, 0);
    }
    if (kind == 1 && !(scl > 0.f && scl < INFINITY)) {  // the staging divides by the scale
      if (qd == 0) report(p.dev_status, CSA_ERR_DEVICE);
      kind = 0;
      scl = 1.f;
    }
    if (qd == 0) {
      s.scale[r] = scl;
      s.kind[r] = kind;
    }
    if (kind == 1) {
      const float inv = 1.f / scl;
#pragma unroll
      for (int i = 0; i < 9; ++i) {
        const int u = qd + 4 * i;
        if (u < 28) {  // 16 E4M3 codes -> output chunks 2u, 2u+1
          uint4 lo, hi;
          e4m3x16_codes_to_f16(buf[i], &lo, &hi);
          store_v_chunk(s, r, 2 * u, lo);
          store_v_chunk(s, r, 2 * u + 1, hi);
        } else {  // 8 BF16 RoPE dims / scale -> chunk 56 + (u - 28)
          store_v_chunk(s, r, 28 + u, bf16x8_scaled_to_f16x8(buf[i], inv));
        }
      }
    } else if (kind == 2) {
#pragma unroll
      for (int i = 0; i < 16; ++i) store_v_chunk(s, r, qd + 4 * i, bf16x8_to_f16x8(buf[i]));
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) store_v_chunk(s, r, qd + 4 * i, make_uint4(0, 0, 0, 0));
    }
  }
  // widen Q to FP16 in place once the TMA has landed
  bool ok = mbar_wait(&s.q_full, 0, p.dev_status);
  for (int i = tid; i < 8 * p.H * 8; i += kAtThreads) {
    uint4* c16 = reinterpret_cast<uint4*>(&s.q[i / (p.H * 8)][(i % (p.H * 8)) * 16]);
    *c16 = bf16x8_to_f16x8(*c16);
  }
  fence_async_smem();
  ok = __syncthreads_and(ok) != 0;

  // S' = Q V'^T : M = 128 heads, N = 64 rows, K = 512 (32 steps of 16)
  const uint32_t t_o = tmem, t_s = tmem + 256;
  if (tid == 0) {
    if (ok) {
      tc_fence_after();
      const uint32_t id = idesc_f16(128, kAtRows, false);
      const uint64_t qd0 = smem_desc(smem_u32(s.q[0]), 16, 1024, kSwizzle128B);
      const uint64_t vd0 = smem_desc(smem_u32(s.v[0]), 16, 1024, kSwizzle128B);
      for (int kk = 0; kk < 32; ++kk) {  // descriptor start addresses advance in 16-byte units
        const uint64_t qoff = (uint64_t)(((kk >> 2) * 128 * 128 + (kk & 3) * 32) >> 4);
        const uint64_t voff = (uint64_t)(((kk >> 2) * kAtRows * 128 + (kk & 3) * 32) >> 4);
        mma_f16(t_s, qd0 + qoff, vd0 + voff, id, kk > 0);
      }
    }
    mma_commit(&s.s_done);
  }
  // chunk 0's warp 1: the de-rotation table of the sequence, while S is computed
  if (c == 0 && dh == 0 && warp == 1 && p.derotate) {
    float cs, sn;
    rope_cos_sin((double)t, tid & 31, (double)p.rope_base, &cs, &sn);
    *reinterpret_cast<float2*>(p.rot + (size_t)b * 64 + 2 * (tid & 31)) = make_float2(cs, sn);
  }
  {
    const bool waited = mbar_wait(&s.s_done, 0, p.dev_status);
    ok = __syncthreads_and(ok && waited) != 0;
  }
  tc_fence_after();

  // softmax over the chunk's 64 rows, all eight warps: warp w reads TMEM lane quadrant w % 4
  // (heads), columns 32 (w / 4) .. +31 (rows); the two halves exchange max and sum
  const int quad = warp & 3, ch = warp >> 2;
  const int h = quad * 32 + (tid & 31);
  float lg[32];
  float m_c;
  {
    uint32_t r0[32];
    tmem_ld32(t_s + ((uint32_t)(quad * 32) << 16) + 32 * ch, r0);
    tmem_ld_wait();
    float mloc = -INFINITY;
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      const int rr = 32 * ch + r;
      lg[r] = s.kind[rr] ? __uint_as_float(r0[r]) * (p.tau * s.scale[rr]) : -INFINITY;
      mloc = fmaxf(mloc, lg[r]);
    }
    s.mx[ch][h] = mloc;
  }
  __syncthreads();
  m_c = fmaxf(s.mx[0][h], s.mx[1][h]);
  {
    float l_loc = 0.f;
    uint8_t* prow = s.pm + h * 128;
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {  // 16-byte chunks 4 ch + c4 of the P' row
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = c4 * 8 + 2 * e, rr = 32 * ch + r;
        const float p0 = m_c == -INFINITY ? 0.f : expf(lg[r] - m_c);
        const float p1 = m_c == -INFINITY ? 0.f : expf(lg[r + 1] - m_c);
        l_loc += p0;
        l_loc += p1;
        w[e] = pack_half2(p0 * s.scale[rr], p1 * s.scale[rr + 1]);
      }
      const int chunk = 4 * ch + c4;
      *reinterpret_cast<uint4*>(prow + ((chunk ^ (h & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    s.sm[ch][h] = l_loc;
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  if (tid < 128) {  // head tid: the chunk's max and sum (the halves summed in a fixed order)
    const float l_c = s.sm[0][tid] + s.sm[1][tid];
    s.inv_l[tid] = l_c > 0.f ? 1.f / l_c : 0.f;
    if (tid < p.H && dh == 0) {
      const size_t slot = ((size_t)b * p.C + c) * p.H + tid;
      p.part_ml[slot] = ok ? make_float2(fmaxf(s.mx[0][tid], s.mx[1][tid]), l_c)
                           : make_float2(-INFINITY, 0.f);
    }
  }

  // O[:, 256 half .. +256] = P' V'[:, 256 half ..] for this CTA's halves: M = 128, N = 256,
  // K = 64 rows (4 steps of 16); V' read MN-major
  const int nh = 3 - p.split;  // halves of the output this CTA computes
  if (tid == 0) {
    if (ok) {
      tc_fence_after();
      const uint32_t id = idesc_f16(128, 256, true);
      for (int hf = 0; hf < nh; ++hf) {
        for (int kk = 0; kk < 4; ++kk) {
          mma_f16(t_o + hf * 256, smem_desc(smem_u32(s.pm) + kk * 32, 16, 1024, kSwizzle128B),
                  smem_desc(smem_u32(s.v[(dh + hf) * 4]) + kk * 2048, kAtRows * 128, 1024,
                            kSwizzle128B),
                  id, kk > 0);
        }
      }
    }
    mma_commit(&s.o_done);
  }
  mbar_wait(&s.o_done, 0, p.dev_status);
  __syncthreads();  // inv_l written by threads 0-127 above
  tc_fence_after();
  {
    // warp w reads lanes of quadrant w % 4 and the second or first half of this CTA's columns
    if (nh == 2)
      store_partial<8>(p, s, t_o, b, c, dh, quad, warp >> 2, tid);
    else
      store_partial<4>(p, s, t_o, b, c, dh, quad, warp >> 2, tid);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// The merge of the chunk partials: one thread per (8-dim group g, head h) of a sequence,
// CTA (g, b). Every load a thread needs (the C_b chunk statistics of its head and its
// C_b partial groups) is issued before any is used, in batches of kCbBatch chunks. Per
// head: M = max(sink, m_c), e_c = exp(m_c - M) l_c, Z = e_0 + ... + e_{C_b-1} +
// exp(sink - M) in chunk order, out = (sum_c e_c o_c) / Z in chunk order (o_c the chunk's
// normalised output), lse = M + log Z; the RoPE dims are de-rotated by -t theta_j.
constexpr int kCbBatch = 18;

__global__ void __launch_bounds__(128) attn_combine_kernel(AtParams p) {
  const int g = blockIdx.x, b = blockIdx.y, h = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  if (h >= p.H) return;
  int n = p.n_entries[b];
  n = n < 0 ? 0 : (n > p.Nmax ? (int)p.Nmax : n);
  const int C_b = (at_rows_total(p, n) + kAtRows - 1) / kAtRows;
  const float2* ml = p.part_ml + (size_t)b * p.C * p.H + h;
  const __half* src = p.part_o + (((size_t)b * p.C * 64 + g) * p.H + h) * 8;
  const size_t cstride = (size_t)64 * p.H * 8;  // halves from one chunk's partial to the next
  const float sink = p.sink[h];
  float M = sink, Z = 0.f;
  float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (C_b <= kCbBatch) {  // the usual case: one round trip
    float2 st[kCbBatch];
    uint4 v[kCbBatch];
#pragma unroll
    for (int c = 0; c < kCbBatch; ++c) {
      st[c] = c < C_b ? __ldcg(ml + (size_t)c * p.H) : make_float2(-INFINITY, 0.f);
      v[c] = c < C_b ? __ldcg(reinterpret_cast<const uint4*>(src + (size_t)c * cstride))
                     : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int c = 0; c < kCbBatch; ++c) M = fmaxf(M, st[c].x);
#pragma unroll
    for (int c = 0; c < kCbBatch; ++c) {
      if (c >= C_b) break;
      const float e = (M == INFINITY || st[c].x == -INFINITY) ? 0.f
                                                              : __fmul_rn(expf(st[c].x - M), st[c].y);
      Z = __fadd_rn(Z, e);
      const uint32_t x[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&x[q]));
        o[2 * q] = fmaf(e, f.x, o[2 * q]);
        o[2 * q + 1] = fmaf(e, f.y, o[2 * q + 1]);
      }
    }
  } else {  // long HCA rows: the maximum first, then batches of chunks
    for (int c = 0; c < C_b; ++c) M = fmaxf(M, __ldcg(ml + (size_t)c * p.H).x);
    for (int c0 = 0; c0 < C_b; c0 += kCbBatch) {
      float2 st[kCbBatch];
      uint4 v[kCbBatch];
#pragma unroll
      for (int i = 0; i < kCbBatch; ++i) {
        st[i] = c0 + i < C_b ? __ldcg(ml + (size_t)(c0 + i) * p.H) : make_float2(-INFINITY, 0.f);
        v[i] = c0 + i < C_b ? __ldcg(reinterpret_cast<const uint4*>(src + (size_t)(c0 + i) * cstride))
                            : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int i = 0; i < kCbBatch; ++i) {
        if (c0 + i >= C_b) break;
        const float e = (M == INFINITY || st[i].x == -INFINITY) ? 0.f
                                                                : __fmul_rn(expf(st[i].x - M), st[i].y);
        Z = __fadd_rn(Z, e);
        const uint32_t x[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&x[q]));
          o[2 * q] = fmaf(e, f.x, o[2 * q]);
          o[2 * q + 1] = fmaf(e, f.y, o[2 * q + 1]);
        }
      }
    }
  }
  if (M == INFINITY)
    Z = INFINITY;
  else
    Z = __fadd_rn(Z, sink == -INFINITY ? 0.f : expf(sink - M));
  const float iz = (Z > 0.f && Z < INFINITY) ? 1.f / Z : 0.f;
  if (g == 0 && p.lse) p.lse[(size_t)b * p.H + h] = M == INFINITY ? INFINITY : M + logf(Z);
#pragma unroll
  for (int e = 0; e < 8; ++e) o[e] = __fmul_rn(o[e], iz);
  const int d0 = g * 8;
  if (p.derotate && d0 >= kNope) {  // pairs 4(g - 56) .. +3 from chunk 0's table
    const float4* rt = reinterpret_cast<const float4*>(p.rot + (size_t)b * 64 + 2 * (d0 - kNope) / 2);
    const float4 r0 = __ldcg(rt), r1 = __ldcg(rt + 1);
    const float cs[4] = {r0.x, r0.z, r1.x, r1.z}, sn[4] = {r0.y, r0.w, r1.y, r1.w};
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      const float x0 = o[e], x1 = o[e + 1];
      o[e] = fmaf(x0, cs[e / 2], __fmul_rn(x1, sn[e / 2]));
      o[e + 1] = fmaf(-x0, sn[e / 2], __fmul_rn(x1, cs[e / 2]));
    }
  }
  uint4 pk;
  pk.x = (uint32_t)f32_to_bf16_bits(o[0]) | ((uint32_t)f32_to_bf16_bits(o[1]) << 16);
  pk.y = (uint32_t)f32_to_bf16_bits(o[2]) | ((uint32_t)f32_to_bf16_bits(o[3]) << 16);
  pk.z = (uint32_t)f32_to_bf16_bits(o[4]) | ((uint32_t)f32_to_bf16_bits(o[5]) << 16);
  pk.w = (uint32_t)f32_to_bf16_bits(o[6]) | ((uint32_t)f32_to_bf16_bits(o[7]) << 16);
  *reinterpret_cast<uint4*>(p.out + ((size_t)b * p.H + h) * kD + d0) = pk;
}

// ------------------------------------------------------------- prefill attention
// A prefill has many queries over one cache, so each query keeps its Q on chip and walks
// its whole row list: one CTA per (query, half of the 512 output dims). The cache entries
// and the window rows are dequantised to FP16 once per call (prefill_rows16_kernel), so the
// per-query gather is a plain copy. Rows come in chunks of 32 through a triple buffer:
//   warps 0-3  gather the chunk's rows with 16-byte cp.async copies straight into the
//              swizzled layout of the decode kernel (no register staging);
//   warp 4     issues S = Q V^T (M = 128 heads, N = 32, K = 512) into a TMEM buffer, then,
//              once the chunk's P is ready, O[:, half] += P V[:, half] (N = 256, K = 32);
//   warps 5-8  one thread per head: online softmax in the base-2 domain with a lazy
//              rescale (O and the running sum are rescaled in TMEM only when the running
//              maximum grows by more than 2^8); P is written as FP16 into the chunk's own
//              S columns in TMEM, and the P V product reads its A operand from there, so
//              shared memory holds only Q and the three row buffers.
// At the end the softmax threads divide by the running sum plus the sink term, de-rotate
// the RoPE dims and store BF16 (and lse). S is computed by both CTAs of a query (each
// needs all 512 dims of the products); O is split so that it fits TMEM next to S.
constexpr int kPaRows = 32;
constexpr int kPaBufs = 3;
constexpr int kPaThreads = 32 * 9;
constexpr float kLog2e = 1.4426950408889634f;

struct PaSmem {
  uint8_t q[8][128 * 128];             // Q FP16: 8 K-blocks [128 heads x 64 dims], 128-B swizzle
  uint8_t v[kPaBufs][8][kPaRows * 128];  // rows FP16: 8 dim-blocks [32 rows x 64 dims]
  int kind[kPaBufs][kPaRows];
  uint64_t q_full, v_full[kPaBufs], v_free[kPaBufs], s_full[kPaBufs], p_full[kPaBufs],
      o_done[kPaBufs], done;
  uint32_t tmem_base;
  volatile int abort;
};

struct PaParams {
  int H, k;
  int64_t Nmax;
  const int32_t* pos;
  const int32_t* idx;
  const int32_t* n_entries;
  const __half* rows16;  // FP16 rows: entries 0..Nmax-1, then window positions from swa_base
  int64_t swa_base;
  const float* sink;
  float tau, rope_base;
  int derotate;
  uint16_t* out;
  float* lse;
  int32_t* dev_status;
};

__device__ __forceinline__ void pa_store_v(PaSmem& s, int buf, int r, int ch, uint4 v) {
  *reinterpret_cast<uint4*>(&s.v[buf][ch >> 3][r * 128 + (((ch & 7) ^ (r & 7)) << 4)]) = v;
}

__global__ void __launch_bounds__(kPaThreads, 1)
    prefill_attn_kernel(const __grid_constant__ CUtensorMap qmap, PaParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  PaSmem& s = *reinterpret_cast<PaSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int b = blockIdx.x >> 1, hf = blockIdx.x & 1, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  pdl_wait();
  pdl_trigger();
  int n = p.n_entries[b];
  const int t = p.pos[b];
  if (n < 0 || n > p.Nmax) {
    if (tid == 0) report(p.dev_status, CSA_ERR_DEVICE);
    n = n < 0 ? 0 : (int)p.Nmax;
  }
  const int rows_total = p.k + kWin;
  const int nchunks = (rows_total + kPaRows - 1) / kPaRows;
  if (tid == 0) {
    mbar_init(&s.q_full, 1);
    for (int i = 0; i < kPaBufs; ++i) {
      mbar_init(&s.v_full[i], 128);
      mbar_init(&s.v_free[i], 1);
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.p_full[i], 128);
      mbar_init(&s.o_done[i], 1);  // P V of the chunks with this parity
    }
    mbar_init(&s.done, 1);
    s.abort = 0;
    mbar_fence_init();
    prefetch_tensormap(&qmap);
    mbar_arrive_expect_tx(&s.q_full, (uint32_t)p.H * kD * 2);
    for (int blk = 0; blk < 8; ++blk) tma_load_2d(s.q[blk], &qmap, &s.q_full, blk * 64, b * p.H);
  }
  if (warp == 4) tmem_alloc(&s.tmem_base, 512);
  if (p.H < 128) {  // Q rows H..127 are zero padding
    for (int i = tid; i < 8 * (128 - p.H) * 8; i += kPaThreads) {
      const int blk = i / ((128 - p.H) * 8), rem = i % ((128 - p.H) * 8);
      *reinterpret_cast<uint4*>(&s.q[blk][p.H * 128 + rem * 16]) = make_uint4(0, 0, 0, 0);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  const uint32_t t_o = tmem, t_s0 = tmem + 256;

  if (warp < 4) {
    // ---------------------------------------------------------- gather (128 threads)
    const int pt = tid;  // 0..127
    bool ok = mbar_wait(&s.q_full, 0, p.dev_status);
    if (!ok) s.abort = 1;
    for (int i = pt; i < 8 * p.H * 8; i += 128) {  // widen Q to FP16 in place
      uint4* c16 = reinterpret_cast<uint4*>(&s.q[i / (p.H * 8)][(i % (p.H * 8)) * 16]);
      *c16 = bf16x8_to_f16x8(*c16);
    }
    const int r = pt >> 2, qd = pt & 3;
    const int64_t self_row = p.Nmax + (t - p.swa_base);  // always present: stands in for
                                                         // rows that carry no weight
    for (int c = 0; c < nchunks; ++c) {
      const int buf = c % kPaBufs;
      if (s.abort || !mbar_wait(&s.v_free[buf], ((c / kPaBufs) & 1) ^ 1, p.dev_status)) {
        s.abort = 1;
        break;
      }
      const int rl = c * kPaRows + r;  // position in the row list
      int kind = 0;
      int64_t row = self_row;
      if (rl < p.k) {
        const int j = p.idx[(size_t)b * p.k + rl];
        if (j >= 0 && j < n) {
          kind = 1;
          row = j;
        } else if (j != -1 && qd == 0) {
          report(p.dev_status, CSA_ERR_DEVICE);
        }
      } else if (rl < rows_total) {
        const int pp = t - (kWin - 1) + (rl - p.k);
        if (pp >= 0) {
          kind = 2;
          row = p.Nmax + (pp - p.swa_base);
        }
      }
      const __half* src = p.rows16 + row * kD;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int u = qd + 4 * i;  // 16-byte piece = 8 dims
        const uint32_t dst =
            smem_u32(&s.v[buf][u >> 3][r * 128 + (((u & 7) ^ (r & 7)) << 4)]);
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src + 8 * u)
                     : "memory");
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
      if (qd == 0) s.kind[buf][r] = kind;
      asm volatile("cp.async.wait_group 0;" ::: "memory");
      fence_async_smem();  // the copies (and the widened Q) are read by tcgen05.mma
      mbar_arrive(&s.v_full[buf]);
    }
  } else if (warp == 4) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_f16(128, kPaRows, false);
      const uint32_t id_o = idesc_f16(128, 256, true);
      auto issue_pv = [&](int c) -> bool {
        const int cb = c % kPaBufs;
        if (s.abort || !mbar_wait(&s.p_full[cb], (c / kPaBufs) & 1, p.dev_status)) return false;
        tc_fence_after();
        for (int kk = 0; kk < 2; ++kk)  // A = P: 16 rows (8 columns) per step
          mma_f16_ts(t_o, t_s0 + kPaRows * cb + kk * 8,
                     smem_desc(smem_u32(s.v[cb][hf * 4]) + kk * 2048, kPaRows * 128, 1024,
                               kSwizzle128B),
                     id_o, (c > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&s.v_free[cb]);
        mma_commit(&s.o_done[cb]);
        return true;
      };
      bool ok = true;
      for (int c = 0; c < nchunks && ok; ++c) {
        const int buf = c % kPaBufs;
        if (s.abort || !mbar_wait(&s.v_full[buf], (c / kPaBufs) & 1, p.dev_status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t t_s = t_s0 + kPaRows * buf;
        for (int kk = 0; kk < 32; ++kk) {
          const uint32_t off = (kk & 3) * 32;
          mma_f16(t_s, smem_desc(smem_u32(s.q[kk >> 2]) + off, 16, 1024, kSwizzle128B),
                  smem_desc(smem_u32(s.v[buf][kk >> 2]) + off, 16, 1024, kSwizzle128B), id_s,
                  kk > 0 ? 1u : 0u);
        }
        mma_commit(&s.s_full[buf]);
        if (c > 0) ok = issue_pv(c - 1);
      }
      if (ok) ok = issue_pv(nchunks - 1);
      if (!ok) s.abort = 1;
      mma_commit(&s.done);
      mbar_wait(&s.done, 0, p.dev_status);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax (128 threads)
    const int quad = warp & 3, h = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const float scale2 = p.tau * kLog2e;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    // P V of chunk c completes phase c / kPaBufs of o_done[c % kPaBufs]; the next phase of
    // that barrier needs this warp's P of chunk c + kPaBufs, so a wait never trails by two
    auto wait_pv = [&](int c) -> bool {
      bool w = true;
      if (lane == 0) w = mbar_wait(&s.o_done[c % kPaBufs], (c / kPaBufs) & 1, p.dev_status);
      return __shfl_sync(0xffffffffu, w, 0) != 0;
    };
    for (int c = 0; c < nchunks; ++c) {
      const int buf = c % kPaBufs, ph = (c / kPaBufs) & 1;
      bool w = true;
      if (lane == 0)
        w = !s.abort && mbar_wait(&s.s_full[buf], ph, p.dev_status) &&
            mbar_wait(&s.v_full[buf], ph, p.dev_status);
      w = __shfl_sync(0xffffffffu, w, 0) != 0;
      if (!w) {
        s.abort = 1;
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t r[32];
      tmem_ld32(t_s0 + kPaRows * buf + lane_off, r);
      tmem_ld_wait();
      float lg[kPaRows];
      float m_c = -INFINITY;
#pragma unroll
      for (int e = 0; e < kPaRows; ++e) {
        lg[e] = s.kind[buf][e] ? __uint_as_float(r[e]) * scale2 : -INFINITY;
        m_c = fmaxf(m_c, lg[e]);
      }
      // lazy rescale: move the reference maximum only when it grows by more than 2^8
      const bool need = m_c > -INFINITY && (m_run == -INFINITY || m_c > m_run + 8.f);
      if (__any_sync(0xffffffffu, need)) {
        if (c > 0 && !wait_pv(c - 1)) {  // O must hold chunks 0..c-1 before it is rescaled
          s.abort = 1;
          ok = false;
          break;
        }
        const float f = need ? (m_run == -INFINITY ? 0.f : exp2f(m_run - m_c)) : 1.f;
        if (need) {
          l_run *= f;
          m_run = m_c;
        }
        if (c > 0) {
          for (int cc = 0; cc < 8; ++cc) {
            uint32_t o[32];
            tmem_ld32(t_o + lane_off + cc * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
            tmem_st32(t_o + lane_off + cc * 32, o);
          }
          tmem_st_wait();
        }
      }
      // P (FP16) over the chunk's S columns: S was read into registers above, and the
      // previous P in these columns belonged to chunk c - kPaBufs, whose P V completed
      // before S of this chunk was issued
      uint32_t pw[kPaRows / 2];
      float lsum = 0.f;
#pragma unroll
      for (int e2 = 0; e2 < kPaRows / 2; ++e2) {
        const int e = 2 * e2;
        const float p0 = (m_run == -INFINITY || lg[e] == -INFINITY) ? 0.f : exp2f(lg[e] - m_run);
        const float p1 =
            (m_run == -INFINITY || lg[e + 1] == -INFINITY) ? 0.f : exp2f(lg[e + 1] - m_run);
        lsum += p0 + p1;
        pw[e2] = pack_half2(p0, p1);
      }
      tmem_st16(t_s0 + kPaRows * buf + lane_off, pw);
      tmem_st_wait();
      l_run += lsum;
      tc_fence_before();
      mbar_arrive(&s.p_full[buf]);
    }
    // every PV has completed: normalise, de-rotate, store
    const bool fin = ok && wait_pv(nchunks - 1);
    if (fin) {
      tc_fence_after();
      const float sink2 = p.sink[h < p.H ? h : 0] * kLog2e;
      float Z = l_run;
      if (sink2 != -INFINITY) Z += (m_run == -INFINITY) ? (sink2 == INFINITY ? INFINITY : exp2f(sink2))
                                                        : exp2f(sink2 - m_run);
      const float inv = Z > 0.f ? 1.f / Z : 0.f;
      for (int cc = 0; cc < 8; ++cc) {
        uint32_t o[32];
        tmem_ld32(t_o + lane_off + cc * 32, o);
        tmem_ld_wait();
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(o[e]) * inv;
        const int d0 = hf * 256 + cc * 32;
        if (p.derotate && d0 >= kNope) {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float cs, sn;
            rope_cos_sin((double)t, (d0 + e - kNope) >> 1, (double)p.rope_base, &cs, &sn);
            const float x0 = v[e], x1 = v[e + 1];
            v[e] = x0 * cs + x1 * sn;
            v[e + 1] = -x0 * sn + x1 * cs;
          }
        }
        if (h < p.H) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + ((size_t)b * p.H + h) * kD + d0);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w4[e] = (uint32_t)f32_to_bf16_bits(v[q4 * 8 + 2 * e]) |
                      ((uint32_t)f32_to_bf16_bits(v[q4 * 8 + 2 * e + 1]) << 16);
            dst[q4] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
      }
      if (hf == 0 && h < p.H && p.lse) {
        float l;
        if (Z == INFINITY) l = INFINITY;
        else if (Z <= 0.f) l = -INFINITY;
        else l = (m_run == -INFINITY ? log2f(Z) : m_run + log2f(Z)) / kLog2e;
        p.lse[(size_t)b * p.H + h] = l;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Dequantise stored entries 0 .. n-1 to FP16 rows (E4M3 code x entry scale rounded once,
// BF16 RoPE dims widened exactly): the same values the decode gather stages. One warp
// per entry; lanes 0-27 take 16 E4M3 dims each, lanes 28-31 take 16 BF16 dims each.
__global__ void __launch_bounds__(256) prefill_rows16_kernel(const uint8_t* kv, const float* kv_scale,
                                                             int64_t n, __half* rows16) {
  pdl_wait();
  pdl_trigger();
  const int64_t j = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (j >= n) return;
  const uint8_t* row = kv + j * kRow;
  uint4* dst = reinterpret_cast<uint4*>(rows16 + j * kD);
  if (lane < 28) {
    uint4 lo, hi;
    e4m3x16_to_f16(*reinterpret_cast<const uint4*>(row + 16 * lane), __ldg(kv_scale + j), &lo, &hi);
    dst[2 * lane] = lo;
    dst[2 * lane + 1] = hi;
  } else {
    const int q = lane - 28;
    const uint4* src = reinterpret_cast<const uint4*>(row + kNope + 32 * q);
    dst[56 + 2 * q] = bf16x8_to_f16x8(src[0]);
    dst[56 + 2 * q + 1] = bf16x8_to_f16x8(src[1]);
  }
}

cudaError_t launch_prefill_rows16(const uint8_t* kv, const float* kv_scale, int64_t n,
                                  __half* rows16, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  return launch_pdl(prefill_rows16_kernel, dim3((unsigned)((n + 7) / 8)), dim3(256), 0, stream,
                    kv, kv_scale, n, rows16);
}

cudaError_t launch_prefill_attn(const csa_attn_args& a, const __half* rows16, int64_t swa_base,
                                const CUtensorMap& qmap, cudaStream_t stream) {
  PaParams p;
  p.H = a.H;
  p.k = a.k;
  p.Nmax = a.Nmax;
  p.pos = a.pos;
  p.idx = a.idx;
  p.n_entries = a.n_entries;
  p.rows16 = rows16;
  p.swa_base = swa_base;
  p.sink = a.sink;
  p.tau = a.tau > 0.f ? a.tau : 0.044194173824159216f;
  p.rope_base = a.rope_base;
  p.derotate = a.derotate;
  p.out = a.out;
  p.lse = a.lse;
  p.dev_status = a.dev_status;
  const size_t smem = sizeof(PaSmem) + 1024;
  static std::atomic<uint64_t> configured{0};
  if (cudaError_t e = configure_smem_once(prefill_attn_kernel, smem, configured);
      e != cudaSuccess)
    return e;
  return launch_pdl(prefill_attn_kernel, dim3(2 * a.B), dim3(kPaThreads), smem, stream, qmap, p);
}

size_t at_smem_bytes() { return sizeof(AtSmem) + 1024; }

// workspace: partial outputs [B][C][64][H][8] fp16, then (max, sum) [B][C][H], then the
// de-rotation tables [B][64], each 256-byte aligned
static size_t at_align(size_t x) { return (x + 255) & ~(size_t)255; }

size_t at_workspace_size(int B, int H, int rows_max) {
  const size_t C = (size_t)(rows_max + kAtRows - 1) / kAtRows;
  return at_align((size_t)B * C * H * kD * sizeof(__half)) +
         at_align((size_t)B * C * H * sizeof(float2)) + at_align((size_t)B * 64 * sizeof(float));
}

cudaError_t launch_attn(const csa_attn_args& a, int sparse, int rows_max, void* workspace,
                        const CUtensorMap& qmap, cudaStream_t stream) {
  AtParams p;
  p.B = a.B;
  p.H = a.H;
  p.k = sparse ? a.k : 0;
  p.sparse = sparse;
  p.C = (rows_max + kAtRows - 1) / kAtRows;
  p.Nmax = a.Nmax;
  p.pos = a.pos;
  p.idx = a.idx;
  p.n_entries = a.n_entries;
  p.kv = a.kv;
  p.kv_scale = a.kv_scale;
  p.swa = a.swa;
  p.sink = a.sink;
  p.tau = a.tau > 0.f ? a.tau : 0.044194173824159216f;  // 1/sqrt(512)
  p.rope_base = a.rope_base;
  p.derotate = a.derotate;
  p.out = a.out;
  p.lse = a.lse;
  char* ws = reinterpret_cast<char*>(workspace);
  p.part_o = reinterpret_cast<__half*>(ws);
  const size_t o_bytes = at_align((size_t)a.B * p.C * a.H * kD * sizeof(__half));
  p.part_ml = reinterpret_cast<float2*>(ws + o_bytes);
  p.rot = reinterpret_cast<float*>(ws + o_bytes + at_align((size_t)a.B * p.C * a.H * sizeof(float2)));
  p.pm = page_map(a.pages, a.Nmax);
  p.dev_status = a.dev_status;
  const size_t smem = at_smem_bytes();
  static std::atomic<uint64_t> configured{0};
  if (cudaError_t e = configure_smem_once(attn_chunk_kernel, smem, configured);
      e != cudaSuccess)
    return e;
  // two CTAs per chunk (one per half of the output dims) when that still fits one wave
  int sms = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    sms = 0;
  p.split = (int64_t)2 * p.C * a.B <= sms ? 2 : 1;
  cudaError_t e = launch_pdl(attn_chunk_kernel, dim3(p.split * p.C, a.B), dim3(kAtThreads), smem, stream,
                             qmap, p);
  if (e != cudaSuccess) return e;
  return launch_pdl(attn_combine_kernel, dim3(64, a.B), dim3(128), 0, stream, p);
}

}  // namespace csa
