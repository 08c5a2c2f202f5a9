// Lightning indexer + top-k (cyqw.cn DeepSeek-V4 walkthrough §2.2: low-rank, low-precision
// indexer queries score the compressed entries and each query keeps the top-k, one set
// for all heads; §3.4 and chooseai.net §二: the indexer QK path runs in MXFP4).
//
// Kernel 1, indexer_score_kernel: a persistent, warp-specialised stream over the FP4 keys.
//   warp 0      TMA producer: 128-entry key tiles (128 x 64 B, 64-byte swizzle) and the
//               tile's 512-byte scale group, into an 8-stage shared-memory ring;
//   warp 1      tcgen05 issuer: copies the key scales into TMEM (tcgen05.cp), then two
//               kind::mxf4 block-scaled MMAs (K = 64 each) give D[128 entries x 64 heads]
//               in fp32 TMEM, double-buffered; it also stages each sequence's FP4 queries
//               (B operand) and their scales;
//   warps 2..5  epilogue: one thread per entry reads its 64 head sums from TMEM and forms
//               s = sum_h w_h * max(0, acc_h) in fp32, writes it to the score workspace
//               and counts it into a 4096-bin histogram of its order-preserving key.
// Kernel 2, topk_select_kernel: per sequence, the histogram fixes the bin that holds the
//   k-th score; CTAs compact the entries above that bin and the candidates inside it; the
//   last CTA of the sequence (atomic ticket, no spinning) radix-selects the rest by
//   (score desc, index asc), sorts the set by index and clears the workspace it used.
#include "common.cuh"

namespace csa {

constexpr int kIxTile = 128;        // entries per tile = MMA M
constexpr int kIxN = 64;            // MMA N: indexer heads padded to 64
constexpr int kIxStages = 8;
constexpr int kIxKeyBytes = kIxTile * 64;
constexpr int kIxSfBytes = 512;
constexpr int kHistBits = 12;
constexpr int kHist = 1 << kHistBits;
constexpr int kIxMaxB = 1024;
constexpr int kSelChunk = 8192;     // entries per select CTA
constexpr int kSelThreads = 512;

struct IxSmem {
  uint8_t keys[kIxStages][kIxKeyBytes];  // 1024-byte aligned tiles
  uint8_t q[2][kIxN * 64];               // queries, 64-byte swizzle, two sequence slots
  uint8_t ksf[kIxStages][kIxSfBytes];
  uint8_t qsf[2][512];
  float w[kIxN];
  uint32_t hist[kHist];
  int32_t prefix[kIxMaxB + 1];
  uint64_t full[kIxStages], empty[kIxStages];
  uint64_t acc_full[2], acc_empty[2], q_free[2], done;
  uint32_t tmem_base;
  volatile int abort;
};

// Workspace layout of csa_indexer_topk (all regions 256-byte aligned).
struct IxWs {
  float* scores;       // [B][Nmax]
  uint32_t* hist;      // [B][kHist]
  uint32_t* counters;  // [B][4]: selected-above count, candidate count, ticket, spare
  int32_t* sel;        // [B][k]
  uint64_t* cand;      // [B][Nmax]
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

__host__ __device__ inline size_t ix_ws_layout(int B, int64_t Nmax, int k, char* base,
                                               IxWs* ws) {
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off += align256(bytes);
    return p;
  };
  char* p0 = take((size_t)B * Nmax * 4);
  char* p1 = take((size_t)B * kHist * 4);
  char* p2 = take((size_t)B * 16);
  char* p3 = take((size_t)B * k * 4);
  char* p4 = take((size_t)B * Nmax * 8);
  if (ws) {
    ws->scores = (float*)p0;
    ws->hist = (uint32_t*)p1;
    ws->counters = (uint32_t*)p2;
    ws->sel = (int32_t*)p3;
    ws->cand = (uint64_t*)p4;
  }
  return off;
}

size_t ix_workspace_size(int B, int64_t Nmax, int k) {
  return ix_ws_layout(B, Nmax, k, nullptr, nullptr);
}

struct IxParams {
  int B, H_I;
  int64_t Nmax;
  const int32_t* n_entries;
  const uint8_t* q_fp4;
  const uint8_t* q_sf;
  const float* w;
  const uint8_t* k_sf;
  IxWs ws;
  int32_t* dev_status;
};

__device__ __forceinline__ int clamp_n(int n, int64_t Nmax, int32_t* st) {
  if (n < 0 || n > Nmax) {
    report(st, CSA_ERR_DEVICE);
    return n < 0 ? 0 : (int)Nmax;
  }
  return n;
}

__global__ void __launch_bounds__(192, 1)
    indexer_score_kernel(const __grid_constant__ CUtensorMap kmap, IxParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  IxSmem& s = *reinterpret_cast<IxSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Tile schedule: sequence b owns ceil(n_b / 128) tiles; CTA c takes a contiguous range.
  if (warp == 0) {
    int carry = 0;
    if (lane == 0) s.prefix[0] = 0;
    for (int base = 0; base < p.B; base += 32) {
      const int bb = base + lane;
      int v = 0;
      if (bb < p.B) v = (clamp_n(p.n_entries[bb], p.Nmax, p.dev_status) + kIxTile - 1) / kIxTile;
      int incl = v;
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (bb < p.B) s.prefix[bb + 1] = carry + incl;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  if (threadIdx.x == 32) {
    for (int i = 0; i < kIxStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.acc_full[i], 1);
      mbar_init(&s.acc_empty[i], 4);
      mbar_init(&s.q_free[i], 1);
    }
    mbar_init(&s.done, 1);
    s.abort = 0;
    mbar_fence_init();
  }
  for (int i = threadIdx.x; i < kHist; i += blockDim.x) s.hist[i] = 0;
  __syncthreads();
  const int total = s.prefix[p.B];
  const int g0 = (int)((int64_t)total * blockIdx.x / gridDim.x);
  const int g1 = (int)((int64_t)total * (blockIdx.x + 1) / gridDim.x);
  if (g0 >= g1) return;  // uniform across the CTA
  if (warp == 1) tmem_alloc(&s.tmem_base, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  const uint32_t t_sfa = tmem + 128, t_sfb = tmem + 136;

  // first sequence of this CTA
  int b0 = 0;
  while (s.prefix[b0 + 1] <= g0) ++b0;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tensormap(&kmap);
      int b = b0, it = 0;
      for (int g = g0; g < g1; ++g, ++it) {
        while (s.prefix[b + 1] <= g) ++b;
        const int t = g - s.prefix[b];
        const int st = it % kIxStages;
        if (s.abort || !mbar_wait(&s.empty[st], ((it / kIxStages) & 1) ^ 1, p.dev_status)) {
          s.abort = 1;
          break;
        }
        mbar_arrive_expect_tx(&s.full[st], kIxKeyBytes + kIxSfBytes);
        tma_load_3d(s.keys[st], &kmap, &s.full[st], 0, t * kIxTile, b);
        bulk_load(s.ksf[st], p.k_sf + ((size_t)b * (p.Nmax / kIxTile) + t) * kIxSfBytes,
                  kIxSfBytes, &s.full[st]);
      }
      // drain: every copy this warp issued has landed before the CTA winds down
      const int issued = it;
      for (int i = issued - kIxStages < 0 ? 0 : issued - kIxStages; i < issued; ++i)
        mbar_wait(&s.full[i % kIxStages], (i / kIxStages) & 1, p.dev_status);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    int b = -1, nseq = -1, it = 0;
    uint32_t qslot = 0;
    for (int g = g0; g < g1; ++g, ++it) {
      int nb = b < 0 ? b0 : b;
      while (s.prefix[nb + 1] <= g) ++nb;
      if (nb != b) {  // stage this sequence's queries (B operand) and their scales
        if (b >= 0 && lane == 0) mma_commit(&s.q_free[qslot]);
        b = nb;
        ++nseq;
        qslot = nseq & 1;
        bool ok = true;
        if (lane == 0) ok = !s.abort && mbar_wait(&s.q_free[qslot], ((nseq >> 1) & 1) ^ 1,
                                                  p.dev_status);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) { s.abort = 1; break; }
        const uint8_t* qsrc = p.q_fp4 + (size_t)b * p.H_I * 64;
        for (int c = lane; c < kIxN * 4; c += 32) {  // 16-byte chunks, 64-byte swizzle
          const int r = c >> 2, ch = c & 3;
          uint4 v = make_uint4(0, 0, 0, 0);
          if (r < p.H_I) v = *reinterpret_cast<const uint4*>(qsrc + r * 64 + ch * 16);
          *reinterpret_cast<uint4*>(&s.q[qslot][r * 64 + ((ch ^ ((r >> 1) & 3)) << 4)]) = v;
        }
        {  // scale atom: lane r0 holds the 4 scales of heads r0, r0+32, r0+64, r0+96
          uint32_t wv[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int n = lane + 32 * j;
            wv[j] = n < p.H_I
                        ? *reinterpret_cast<const uint32_t*>(p.q_sf + ((size_t)b * p.H_I + n) * 4)
                        : 0x7F7F7F7Fu;
          }
          *reinterpret_cast<uint4*>(&s.qsf[qslot][lane * 16]) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tc_fence_after();
          tmem_cp_32x128b_x4(t_sfb, smem_desc(smem_u32(s.qsf[qslot]), 0, 128, kSwizzleNone));
        }
      }
      if (lane == 0) {
        const int st = it % kIxStages, a = it & 1;
        bool ok = !s.abort && mbar_wait(&s.acc_empty[a], ((it >> 1) & 1) ^ 1, p.dev_status) &&
                  mbar_wait(&s.full[st], (it / kIxStages) & 1, p.dev_status);
        if (!ok) {
          s.abort = 1;
        } else {
          tc_fence_after();
          tmem_cp_32x128b_x4(t_sfa, smem_desc(smem_u32(s.ksf[st]), 0, 128, kSwizzleNone));
          const uint32_t ka = smem_u32(s.keys[st]), qa = smem_u32(s.q[qslot]);
#pragma unroll
          for (int kh = 0; kh < 2; ++kh) {
            mma_mxf4(tmem + a * kIxN, smem_desc(ka + 32 * kh, 16, 512, kSwizzle64B),
                     smem_desc(qa + 32 * kh, 16, 512, kSwizzle64B),
                     idesc_mxf4(kIxTile, kIxN, 2 * kh), t_sfa, t_sfb, kh);
          }
          mma_commit(&s.empty[st]);
          mma_commit(&s.acc_full[a]);
        }
      }
      if (__shfl_sync(0xffffffffu, s.abort, 0)) break;
    }
    if (lane == 0) {  // every tcgen05 operation of this CTA has completed
      mma_commit(&s.done);
      mbar_wait(&s.done, 0, p.dev_status);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    int b = -1, n_b = 0, it = 0;
    auto flush = [&](int bb) {
      asm volatile("bar.sync 1, 128;" ::: "memory");
      uint32_t* gh = p.ws.hist + (size_t)bb * kHist;
      for (int i = threadIdx.x - 64; i < kHist; i += 128) {
        const uint32_t v = s.hist[i];
        if (v) {
          atomicAdd(gh + i, v);
          s.hist[i] = 0;
        }
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
    };
    for (int g = g0; g < g1; ++g, ++it) {
      int nb = b < 0 ? b0 : b;
      while (s.prefix[nb + 1] <= g) ++nb;
      if (nb != b) {
        if (b >= 0) flush(b);
        b = nb;
        n_b = clamp_n(p.n_entries[b], p.Nmax, nullptr);
        if (threadIdx.x - 64 < kIxN) {
          const int h = threadIdx.x - 64;
          s.w[h] = h < p.H_I ? p.w[(size_t)b * p.H_I + h] : 0.f;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
      }
      const int t = g - s.prefix[b], a = it & 1;
      // one thread waits for the accumulator; the named barrier hands the outcome to the
      // other 127, so every epilogue thread takes the same path (no divergent barriers)
      bool fail = false;
      if (threadIdx.x == 64) fail = s.abort || !mbar_wait(&s.acc_full[a], (it >> 1) & 1, p.dev_status);
      if (named_bar_or(1, 128, fail)) {
        s.abort = 1;
        break;
      }
      tc_fence_after();
      uint32_t r0[32], r1[32];
      const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + a * kIxN;
      tmem_ld32(taddr, r0);
      tmem_ld32(taddr + 32, r1);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.acc_empty[a]);
      float sc = 0.f;
#pragma unroll
      for (int h = 0; h < 32; ++h) sc = fmaf(s.w[h], fmaxf(__uint_as_float(r0[h]), 0.f), sc);
#pragma unroll
      for (int h = 0; h < 32; ++h) sc = fmaf(s.w[32 + h], fmaxf(__uint_as_float(r1[h]), 0.f), sc);
      const int j = t * kIxTile + row;
      if (j < n_b) {
        p.ws.scores[(size_t)b * p.Nmax + j] = sc;
        atomicAdd(&s.hist[float_key(sc) >> (32 - kHistBits)], 1u);
      }
    }
    if (b >= 0) flush(b);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ------------------------------------------------------------------- select
struct SelParams {
  int B, k;
  int64_t Nmax;
  const int32_t* n_entries;
  IxWs ws;
  int32_t* idx;
  float* scores_out;
  int32_t* dev_status;
};

__device__ __forceinline__ void warp_append(bool pred, uint32_t* counter, uint32_t* slot_out) {
  const uint32_t m = __ballot_sync(0xffffffffu, pred);
  uint32_t base = 0;
  const int lane = threadIdx.x & 31;
  if (m) {
    const int leader = __ffs(m) - 1;
    if (lane == leader) base = atomicAdd(counter, __popc(m));
    base = __shfl_sync(0xffffffffu, base, leader);
  }
  *slot_out = base + __popc(m & ((1u << lane) - 1));
}

__global__ void __launch_bounds__(kSelThreads) topk_select_kernel(SelParams p) {
  __shared__ uint32_t sh_hist[kHist];
  __shared__ uint32_t part[kSelThreads];
  __shared__ int sh_tbin, sh_last;
  __shared__ uint64_t sh_prefix;
  __shared__ uint32_t sh_remaining;
  __shared__ int32_t list[2048];
  __shared__ uint32_t list_n;
  const int b = blockIdx.y, sblk = blockIdx.x, tid = threadIdx.x;
  const int n = clamp_n(p.n_entries[b], p.Nmax, p.dev_status);
  const int k_eff = n < p.k ? n : p.k;
  const int S_b = n == 0 ? 1 : (n + kSelChunk - 1) / kSelChunk;
  if (sblk >= S_b) return;
  uint32_t* cnt = p.ws.counters + (size_t)b * 4;
  const float* sc = p.ws.scores + (size_t)b * p.Nmax;

  // 1. threshold bin: the highest bin whose suffix count reaches k
  if (n > p.k) {
    const uint32_t* gh = p.ws.hist + (size_t)b * kHist;
    for (int i = tid; i < kHist; i += kSelThreads) sh_hist[i] = __ldcg(gh + i);
    __syncthreads();
    constexpr int per = kHist / kSelThreads;  // 8 bins per thread, thread 0 = top bins
    uint32_t mine = 0;
    for (int i = 0; i < per; ++i) mine += sh_hist[kHist - 1 - (tid * per + i)];
    part[tid] = mine;
    __syncthreads();
    if (tid == 0) {
      uint32_t cum = 0;
      int tb = 0;
      for (int t = 0; t < kSelThreads; ++t) {
        if (cum + part[t] >= (uint32_t)p.k) {
          for (int i = 0; i < per; ++i) {
            const int bin = kHist - 1 - (t * per + i);
            if (cum + sh_hist[bin] >= (uint32_t)p.k) { tb = bin; break; }
            cum += sh_hist[bin];
          }
          break;
        }
        cum += part[t];
      }
      sh_tbin = tb;
    }
  } else if (tid == 0) {
    sh_tbin = -1;  // everything is selected
  }
  __syncthreads();
  const int tbin = sh_tbin;

  // 2. compaction of this CTA's slice
  const int j0 = sblk * kSelChunk, j1 = min(n, j0 + kSelChunk);
  for (int base = j0; base < j1; base += kSelThreads) {
    const int j = base + tid;
    const bool in = j < j1;
    uint32_t key = 0;
    int bin = -2;
    if (in) {
      key = float_key(__ldcg(sc + j));
      bin = (int)(key >> (32 - kHistBits));
    }
    uint32_t slot;
    const bool above = in && bin > tbin;
    warp_append(above, &cnt[0], &slot);
    if (above) {
      if (slot < (uint32_t)p.k) p.ws.sel[(size_t)b * p.k + slot] = j;
      else report(p.dev_status, CSA_ERR_DEVICE);  // histogram and scores disagree
    }
    const bool eq = in && bin == tbin;
    warp_append(eq, &cnt[1], &slot);
    if (eq) {
      if (slot < (uint32_t)p.Nmax)
        p.ws.cand[(size_t)b * p.Nmax + slot] = ((uint64_t)key << 32) | (0xFFFFFFFFu - (uint32_t)j);
      else report(p.dev_status, CSA_ERR_DEVICE);
    }
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    sh_last = atomicAdd(&cnt[2], 1u) == (uint32_t)(S_b - 1);
  }
  __syncthreads();
  if (!sh_last) return;
  __threadfence();

  // 3. the last CTA of the sequence finishes the selection
  uint32_t n_sel = __ldcg(&cnt[0]), n_cand = __ldcg(&cnt[1]);
  if (n_sel > (uint32_t)p.k) n_sel = (uint32_t)p.k;
  if (n_cand > (uint32_t)p.Nmax) n_cand = (uint32_t)p.Nmax;
  const uint32_t need = (uint32_t)k_eff > n_sel ? (uint32_t)k_eff - n_sel : 0u;
  const uint64_t* cand = p.ws.cand + (size_t)b * p.Nmax;
  if (n_sel > (uint32_t)k_eff || need > n_cand) report(p.dev_status, CSA_ERR_DEVICE);
  uint64_t thr = 0;  // composites >= thr are kept
  if (need > 0 && need < n_cand) {
    if (tid == 0) { sh_prefix = 0; sh_remaining = need; }
    uint64_t mask = 0;
    for (int pass = 7; pass >= 0; --pass) {
      for (int i = tid; i < 256; i += kSelThreads) sh_hist[i] = 0;
      __syncthreads();
      const uint64_t pre = sh_prefix;
      for (uint32_t i = tid; i < n_cand; i += kSelThreads) {
        const uint64_t c = __ldcg(cand + i);
        if ((c & mask) == pre) atomicAdd(&sh_hist[(c >> (8 * pass)) & 255], 1u);
      }
      __syncthreads();
      if (tid == 0) {
        uint32_t cum = 0, rem = sh_remaining;
        int d = 255;
        for (; d > 0; --d) {
          if (cum + sh_hist[d] >= rem) break;
          cum += sh_hist[d];
        }
        sh_prefix = pre | ((uint64_t)d << (8 * pass));
        sh_remaining = rem - cum;
      }
      mask |= (uint64_t)255 << (8 * pass);
      __syncthreads();
    }
    thr = sh_prefix;
  }
  if (tid == 0) list_n = 0;
  __syncthreads();
  for (uint32_t i = tid; i < n_sel && i < (uint32_t)k_eff; i += kSelThreads)
    list[i] = __ldcg(p.ws.sel + (size_t)b * p.k + i);
  if (tid == 0) list_n = n_sel < (uint32_t)k_eff ? n_sel : (uint32_t)k_eff;
  __syncthreads();
  if (need > 0) {
    for (uint32_t i = tid; i < n_cand; i += kSelThreads) {
      const uint64_t c = __ldcg(cand + i);
      if (c >= thr) {
        const uint32_t slot = atomicAdd(&list_n, 1u);
        if (slot < 2048) list[slot] = (int32_t)(0xFFFFFFFFu - (uint32_t)(c & 0xFFFFFFFFu));
      }
    }
  }
  __syncthreads();
  const int cnt_sel = list_n < 2048u ? (int)list_n : 2048;
  int P2 = 1;
  while (P2 < p.k) P2 <<= 1;
  for (int i = cnt_sel + tid; i < P2; i += kSelThreads) list[i] = 0x7FFFFFFF;
  __syncthreads();
  for (int size = 2; size <= P2; size <<= 1) {  // bitonic sort, ascending
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < P2; i += kSelThreads) {
        const int jx = i ^ stride;
        if (jx > i) {
          const bool up = (i & size) == 0;
          const int x = list[i], y = list[jx];
          if ((x > y) == up) { list[i] = y; list[jx] = x; }
        }
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < p.k; i += kSelThreads) {
    const int v = i < cnt_sel ? list[i] : -1;
    p.idx[(size_t)b * p.k + i] = v;
    if (p.scores_out) p.scores_out[(size_t)b * p.k + i] = v >= 0 ? __ldcg(sc + v) : __int_as_float(0x7fc00000);
  }
  // 4. leave the workspace zeroed for the next call
  uint32_t* gh = p.ws.hist + (size_t)b * kHist;
  for (int i = tid; i < kHist; i += kSelThreads) gh[i] = 0;
  if (tid < 4) cnt[tid] = 0;
}

// ------------------------------------------------------------------- launch
cudaError_t launch_indexer_topk(const csa_topk_args& a, void* workspace, int num_sms,
                                const CUtensorMap& kmap, cudaStream_t stream) {
  IxWs ws;
  ix_ws_layout(a.B, a.Nmax, a.k, (char*)workspace, &ws);
  IxParams p{a.B, a.H_I, a.Nmax, a.n_entries, a.q_fp4, a.q_sf, a.w, a.k_sf, ws, a.dev_status};
  const size_t smem = sizeof(IxSmem) + 1024;
  static int configured = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured != dev) {
    cudaError_t e = cudaFuncSetAttribute(indexer_score_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = dev;
  }
  const int64_t tiles_max = (int64_t)a.B * (a.Nmax / kIxTile);
  int grid = 2 * num_sms;
  if (tiles_max < grid) grid = (int)(tiles_max > 0 ? tiles_max : 1);
  indexer_score_kernel<<<grid, 192, smem, stream>>>(kmap, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  SelParams sp{a.B, a.k, a.Nmax, a.n_entries, ws, a.idx, a.scores, a.dev_status};
  const int64_t chunks = (a.Nmax + kSelChunk - 1) / kSelChunk;
  dim3 g2((unsigned)(chunks > 0 ? chunks : 1), a.B);
  topk_select_kernel<<<g2, kSelThreads, 0, stream>>>(sp);
  return cudaGetLastError();
}

size_t ix_smem_bytes() { return sizeof(IxSmem) + 1024; }

}  // namespace csa
