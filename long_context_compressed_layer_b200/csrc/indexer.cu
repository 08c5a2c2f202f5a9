// Lightning indexer + top-k (cyqw.cn DeepSeek-V4 walkthrough §2.2: low-rank, low-precision
// indexer queries score the compressed entries and each query keeps the top-k, one set
// for all heads; §3.4 and chooseai.net §二: the indexer QK path runs in MXFP4).
//
// Kernel 1, indexer_score_kernel: a persistent (one CTA per SM), warp-specialised stream
// over the FP4 keys.
//   warp 0      TMA producer: 128-entry key tiles (128 x 64 B, 64-byte swizzle) and the
//               tile's 512-byte scale group, into a 12-stage shared-memory ring;
//   warp 1      tcgen05 issuer: copies the key scales into TMEM (tcgen05.cp), then two
//               kind::mxf4 block-scaled MMAs (K = 64 each) give D[128 entries x 64 heads]
//               in fp32 TMEM, four accumulators deep; it also stages each sequence's FP4
//               queries (B operand) and their scales;
//   warps 2..9  epilogue, two groups of four (one warp per TMEM lane quadrant) taking
//               alternate tiles: one thread per entry reads its 64 head sums from TMEM and
//               forms s = sum_h w_h * max(0, acc_h) in fp32 (w held in registers), writes it
//               to the score workspace and counts its order-preserving key into the warp's
//               own 4096-bin histogram (16-bit counters), flushed to the sequence's global
//               histogram when the warp moves to another sequence.
// Kernels 2-3, the selection (no sorting anywhere):
//   topk_threshold_kernel: per sequence and 8192-entry slice, the histogram fixes the bin
//     that holds the k-th score (a parallel suffix scan); each CTA counts its entries above
//     that bin and appends the in-bin candidates. The last CTA of a sequence (atomic ticket,
//     no spinning) resolves the exact cut inside the bin by a radix select on the remaining
//     20 key bits (ties broken by the smaller index), then turns the per-slice counts into
//     output offsets and clears the histogram and counters for the next call;
//   topk_write_kernel: every slice writes its selected entries in index order at its offset,
//     so the output comes out ascending without a sort.
#include "common.cuh"

namespace csa {

constexpr int kIxTile = 128;        // entries per tile = MMA M
constexpr int kIxN = 64;            // MMA N: indexer heads padded to 64
#ifndef CSA_IX_CTAS_PER_SM
#define CSA_IX_CTAS_PER_SM 2
#endif
constexpr int kIxCtasPerSm = CSA_IX_CTAS_PER_SM;
// Two CTAs per SM give every SM two independent TMA producers and tcgen05 issuers; each
// CTA then owns half of TMEM (256 columns) and about half of shared memory.
constexpr int kIxStages = kIxCtasPerSm == 2 ? 7 : 12;
constexpr int kIxBatch = kIxCtasPerSm == 2 ? 1 : 3;  // tiles per accumulator handshake
constexpr int kIxNbuf = kIxCtasPerSm == 2 ? 3 : 2;   // accumulator batches in flight
constexpr int kIxAcc = kIxNbuf * kIxBatch;           // TMEM accumulators of 64 columns
constexpr int kIxEpiWarps = kIxCtasPerSm == 2 ? 4 : 8;  // groups of four (one per quadrant)
constexpr int kIxGroups = kIxEpiWarps / 4;
constexpr int kIxTmemCols = kIxCtasPerSm == 2 ? 256 : 512;
constexpr int kIxThreads = 64 + 32 * kIxEpiWarps;
static_assert(kIxAcc * 64 + 16 <= kIxTmemCols, "accumulators and scale factors fit TMEM");
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
  uint32_t hist[kIxEpiWarps][kHist / 2]; // per-warp histograms, two 16-bit bins per word
  uint8_t ksf[kIxStages][kIxSfBytes];
  uint8_t qsf[2][512];
  int32_t prefix[kIxMaxB + 1];
  uint64_t full[kIxStages], empty[kIxStages];
  uint64_t acc_full[kIxNbuf], acc_empty[kIxNbuf], q_free[2], done;
  uint32_t tmem_base;
  volatile int abort;
};

// Workspace layout of csa_indexer_topk (all regions 256-byte aligned).
struct IxWs {
  float* scores;        // [B][Nmax]
  uint32_t* hist;       // [B][kHist]
  uint32_t* counters;   // [B][4]: candidate count, ticket
  uint32_t* slice_cnt;  // [B][S]: above-bin count per slice, then the slice's output offset
  uint32_t* rule;       // [B][4]: cut key, cut index, selected count
  uint64_t* cand;       // [B][Nmax]: (key << 32) | index of the in-bin candidates
  int S;                // slices per sequence
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

__host__ __device__ inline int ix_slices(int64_t Nmax) {
  const int64_t s = (Nmax + kSelChunk - 1) / kSelChunk;
  return s > 0 ? (int)s : 1;
}

__host__ __device__ inline size_t ix_ws_layout(int B, int64_t Nmax, int k, char* base,
                                               IxWs* ws) {
  (void)k;
  const int S = ix_slices(Nmax);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off += align256(bytes);
    return p;
  };
  char* p0 = take((size_t)B * Nmax * 4);
  char* p1 = take((size_t)B * kHist * 4);
  char* p2 = take((size_t)B * 16);
  char* p3 = take((size_t)B * S * 4);
  char* p4 = take((size_t)B * 16);
  char* p5 = take((size_t)B * Nmax * 8);
  if (ws) {
    ws->scores = (float*)p0;
    ws->hist = (uint32_t*)p1;
    ws->counters = (uint32_t*)p2;
    ws->slice_cnt = (uint32_t*)p3;
    ws->rule = (uint32_t*)p4;
    ws->cand = (uint64_t*)p5;
    ws->S = S;
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

__global__ void __launch_bounds__(kIxThreads, kIxCtasPerSm)
    indexer_score_kernel(const __grid_constant__ CUtensorMap kmap, IxParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  IxSmem& s = *reinterpret_cast<IxSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // set-up that touches no global memory overlaps the previous kernel's tail
  if (threadIdx.x == 32) {
    for (int i = 0; i < kIxStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < kIxNbuf; ++i) {
      mbar_init(&s.acc_full[i], 1);
      mbar_init(&s.acc_empty[i], 4);
    }
    for (int i = 0; i < 2; ++i) mbar_init(&s.q_free[i], 1);
    mbar_init(&s.done, 1);
    s.abort = 0;
    mbar_fence_init();
  }
  if (threadIdx.x == 0) prefetch_tensormap(&kmap);
  {
    uint32_t* hz = &s.hist[0][0];
    for (int i = threadIdx.x; i < kIxEpiWarps * kHist / 2; i += blockDim.x) hz[i] = 0;
  }
  if (warp == 1) tmem_alloc(&s.tmem_base, kIxTmemCols);
  pdl_wait();
  pdl_trigger();

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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int total = s.prefix[p.B];
  const int g0 = (int)((int64_t)total * blockIdx.x / gridDim.x);
  const int g1 = (int)((int64_t)total * (blockIdx.x + 1) / gridDim.x);
  const uint32_t tmem = s.tmem_base;
  if (g0 >= g1) {  // uniform across the CTA: nothing to score
    if (warp == 1) tmem_dealloc(tmem, kIxTmemCols);
    return;
  }
  const uint32_t t_sfa = tmem + kIxAcc * kIxN, t_sfb = t_sfa + 8;

  // first sequence of this CTA
  int b0 = 0;
  while (s.prefix[b0 + 1] <= g0) ++b0;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
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
        // tile it goes to accumulator a of batch bt = it / kIxBatch, buffer bb
        const int st = it % kIxStages, bt = it / kIxBatch, bb = bt % kIxNbuf;
        const int a = bb * kIxBatch + it % kIxBatch;
        bool ok = !s.abort;
        if (ok && it % kIxBatch == 0) {  // first tile of a batch: its buffer must be free
          ok = mbar_wait(&s.acc_empty[bb], ((bt / kIxNbuf) & 1) ^ 1, p.dev_status);
          // the epilogue's TMEM reads of this buffer happen before our MMAs overwrite it
          tc_fence_after();
        }
        // (the key tile arrives through the async proxy: the barrier alone orders it)
        ok = ok && mbar_wait(&s.full[st], (it / kIxStages) & 1, p.dev_status);
        if (!ok) {
          s.abort = 1;
        } else {
          tmem_cp_32x128b_x4(t_sfa, smem_desc(smem_u32(s.ksf[st]), 0, 128, kSwizzleNone));
          const uint32_t ka = smem_u32(s.keys[st]), qa = smem_u32(s.q[qslot]);
#pragma unroll
          for (int kh = 0; kh < 2; ++kh) {
            mma_mxf4(tmem + a * kIxN, smem_desc(ka + 32 * kh, 16, 512, kSwizzle64B),
                     smem_desc(qa + 32 * kh, 16, 512, kSwizzle64B),
                     idesc_mxf4(kIxTile, kIxN, 2 * kh), t_sfa, t_sfb, kh);
          }
          mma_commit(&s.empty[st]);
          // last tile of the batch (or of this CTA): hand the batch to the epilogue
          if (it % kIxBatch == kIxBatch - 1 || g + 1 == g1) mma_commit(&s.acc_full[bb]);
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
    const int ew = warp - 2;            // 0..7
    const int grp = ew >> 2;            // takes the batches bt with bt % kIxGroups == grp
    const int quad = warp & 3;          // TMEM lane quadrant
    const int row = quad * 32 + lane;   // entry within the tile
    uint32_t* hist = s.hist[ew];
    int b = -1, n_b = 0, since_flush = 0;
    float w[kIxN];
    auto flush = [&](int bb) {  // warp-local: add the warp's counts to the global histogram
      __syncwarp();
      uint32_t* gh = p.ws.hist + (size_t)bb * kHist;
      for (int i = lane; i < kHist / 2; i += 32) {
        const uint32_t v = hist[i];
        if (v) {
          if (v & 0xFFFFu) atomicAdd(gh + 2 * i, v & 0xFFFFu);
          if (v >> 16) atomicAdd(gh + 2 * i + 1, v >> 16);
          hist[i] = 0;
        }
      }
      __syncwarp();
    };
    // batch bt holds tiles kIxBatch*bt .. of this CTA; group grp takes bt % kIxGroups == grp
    const int ntiles = g1 - g0;
    int bseq = b0;
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    for (int bt = grp; bt * kIxBatch < ntiles; bt += kIxGroups) {
      const int bb = bt % kIxNbuf;
      bool ok = true;
      if (lane == 0) ok = !s.abort && mbar_wait(&s.acc_full[bb], (bt / kIxNbuf) & 1, p.dev_status);
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        s.abort = 1;
        break;
      }
      tc_fence_after();
      const int it0 = bt * kIxBatch, it_end = min(ntiles, it0 + kIxBatch);
      for (int it = it0; it < it_end; ++it) {
        const int g = g0 + it;
        while (s.prefix[bseq + 1] <= g) ++bseq;
        // 16-bit counters: a warp adds at most 32 counts per tile, so flush every 2000
        // tiles (< 65536 counts) as well as whenever the sequence changes
        if (bseq != b || since_flush == 2000) {
          if (b >= 0) flush(b);
          since_flush = 0;
          b = bseq;
          n_b = clamp_n(p.n_entries[b], p.Nmax, nullptr);
#pragma unroll
          for (int h = 0; h < kIxN; ++h) w[h] = h < p.H_I ? __ldg(p.w + (size_t)b * p.H_I + h) : 0.f;
        }
        ++since_flush;
        uint32_t r[2][32];
        const uint32_t ta = lane_base + (bb * kIxBatch + (it - it0)) * kIxN;
        tmem_ld32(ta, r[0]);
        tmem_ld32(ta + 32, r[1]);
        tmem_ld_wait();
        // s = sum_h w_h * max(0, acc_h): eight independent partial sums (heads h = k mod 8)
        // combined in a fixed tree, so the FMA latency chain is 8 deep instead of 64
        float part[8];
#pragma unroll
        for (int k8 = 0; k8 < 8; ++k8) part[k8] = 0.f;
#pragma unroll
        for (int h = 0; h < kIxN; ++h)
          part[h & 7] = fmaf(w[h], fmaxf(__uint_as_float(r[h >> 5][h & 31]), 0.f), part[h & 7]);
        const float sc = ((part[0] + part[1]) + (part[2] + part[3])) +
                         ((part[4] + part[5]) + (part[6] + part[7]));
        const int j = (g - s.prefix[b]) * kIxTile + row;
        if (j < n_b) {
          p.ws.scores[(size_t)b * p.Nmax + j] = sc;
          const uint32_t bin = float_key(sc) >> (32 - kHistBits);
          atomicAdd(&hist[bin >> 1], 1u << (16 * (bin & 1)));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.acc_empty[bb]);
    }
    if (b >= 0) flush(b);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kIxTmemCols);
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

// Inclusive scan over the 512 threads of a CTA (16 warps); `tmp` holds 16 words.
__device__ __forceinline__ uint32_t block_incl_scan(uint32_t v, uint32_t* tmp, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  __syncthreads();
  if (lane == 31) tmp[warp] = v;
  __syncthreads();
  uint32_t before = 0, all = 0;
  for (int w = 0; w < kSelThreads / 32; ++w) {
    const uint32_t t = tmp[w];
    if (w < warp) before += t;
    all += t;
  }
  if (total) *total = all;
  return v + before;
}

constexpr int kSelPer = kSelChunk / kSelThreads;  // 16 entries per thread

// scores[j .. j+15] (entries at or past `end` read as 0, never touched in memory)
__device__ __forceinline__ void load_scores16(const float* sc, int j, int end, float (&v)[kSelPer]) {
  if (j + kSelPer <= end) {
#pragma unroll
    for (int q = 0; q < kSelPer / 4; ++q) {
      const float4 f = __ldcg(reinterpret_cast<const float4*>(sc + j) + q);
      v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
    }
  } else {
#pragma unroll
    for (int e = 0; e < kSelPer; ++e) v[e] = j + e < end ? __ldcg(sc + j + e) : 0.f;
  }
}

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

// Radix-select step over the candidates: among those whose field matches `prefix` under
// `mask`, histogram the digit (field >> shift) & (2^bits - 1) and find the digit where the
// running count (from the top when `descending`, else from the bottom) reaches *remaining.
// Updates *prefix / *remaining (shared). Field: key = cand >> 32 (hi) or index (lo).
// Candidates come from shared memory (staged) or, past its capacity, from global memory.
__device__ __forceinline__ uint64_t cand_at(const uint64_t* cand, uint32_t i, bool staged) {
  return staged ? cand[i] : __ldcg(cand + i);
}

constexpr uint32_t kCandStage = 2048;

__device__ void radix_step(const uint64_t* cand, bool staged, uint32_t n_cand, bool hi, uint32_t key_eq,
                           bool need_key_eq, uint32_t mask, int shift, int bits,
                           bool descending, uint32_t* prefix, uint32_t* remaining,
                           uint32_t* h, uint32_t* digit_pop = nullptr) {
  const int tid = threadIdx.x;
  const uint32_t nd = 1u << bits;
  for (uint32_t i = tid; i < 256; i += kSelThreads) h[i] = 0;
  __syncthreads();
  const uint32_t pre = *prefix;
  for (uint32_t i = tid; i < n_cand; i += kSelThreads) {
    const uint64_t c = cand_at(cand, i, staged);
    const uint32_t key = (uint32_t)(c >> 32), ix = (uint32_t)c;
    if (need_key_eq && key != key_eq) continue;
    const uint32_t f = hi ? key : ix;
    if ((f & mask) == pre) atomicAdd(&h[(f >> shift) & (nd - 1)], 1u);
  }
  __syncthreads();
  if (threadIdx.x < 32) {  // one warp: 8 digits per lane, walked in the chosen direction
    const int lane = threadIdx.x;
    const int per = (int)(nd + 31) / 32;
    uint32_t mine = 0;
    for (int i = 0; i < per; ++i) {
      const int r = lane * per + i;
      if (r < (int)nd) mine += h[descending ? nd - 1 - r : r];
    }
    uint32_t incl = mine;
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const uint32_t rem = *remaining;
    const bool cross = incl >= rem && incl - mine < rem;
    if (cross) {
      uint32_t cum = incl - mine;
      for (int i = 0; i < per; ++i) {
        const int r = lane * per + i;
        const uint32_t d = descending ? nd - 1 - r : r;
        if (cum + h[d] >= rem) {
          *prefix = pre | (d << shift);
          *remaining = rem - cum;
          if (digit_pop) *digit_pop = h[d];
          break;
        }
        cum += h[d];
      }
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kSelThreads) topk_threshold_kernel(SelParams p) {
  __shared__ uint32_t h[kHist];
  __shared__ uint32_t tmp[kSelThreads / 32];
  __shared__ int sh_tbin, sh_last;
  __shared__ uint32_t sh_above, sh_prefix, sh_rem, sh_sum, sh_pop;
  __shared__ uint64_t cand_s[kCandStage];
  const int b = blockIdx.y, sblk = blockIdx.x, tid = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  const int n = clamp_n(p.n_entries[b], p.Nmax, p.dev_status);
  const int k_eff = n < p.k ? n : p.k;
  const int S_b = n == 0 ? 1 : (n + kSelChunk - 1) / kSelChunk;
  if (sblk >= S_b) return;
  uint32_t* cnt = p.ws.counters + (size_t)b * 4;
  uint32_t* scnt = p.ws.slice_cnt + (size_t)b * p.ws.S;
  const float* sc = p.ws.scores + (size_t)b * p.Nmax;

  // 1. threshold bin: highest bin whose suffix count reaches k (parallel suffix scan)
  if (tid == 0) { sh_tbin = -1; sh_above = 0; }
  if (n > p.k) {
    const uint32_t* gh = p.ws.hist + (size_t)b * kHist;
    for (int i = tid; i < kHist; i += kSelThreads) h[i] = __ldcg(gh + i);
    __syncthreads();
    constexpr int per = kHist / kSelThreads;  // thread 0 holds the top bins
    uint32_t mine = 0;
    for (int i = 0; i < per; ++i) mine += h[kHist - 1 - (tid * per + i)];
    const uint32_t incl = block_incl_scan(mine, tmp, nullptr);
    if (incl >= (uint32_t)p.k && incl - mine < (uint32_t)p.k) {
      uint32_t cum = incl - mine;
      for (int i = 0; i < per; ++i) {
        const int bin = kHist - 1 - (tid * per + i);
        if (cum + h[bin] >= (uint32_t)p.k) { sh_tbin = bin; break; }
        cum += h[bin];
      }
    }
  }
  __syncthreads();
  const int tbin = sh_tbin;

  // 2. this slice: count entries above the bin, append the in-bin candidates. Each thread
  // owns 16 consecutive entries, loaded as four float4 before any is used.
  const int j0 = sblk * kSelChunk, j1 = min(n, j0 + kSelChunk);
  const int jt = j0 + tid * kSelPer;
  float v[kSelPer];
  load_scores16(sc, jt, j1, v);
  uint32_t above = 0;
#pragma unroll
  for (int e = 0; e < kSelPer; ++e) {
    const int j = jt + e;
    const bool in = j < j1;
    const uint32_t key = float_key(v[e]);
    const int bin = in ? (int)(key >> (32 - kHistBits)) : -2;
    above += (in && bin > tbin) ? 1u : 0u;
    const bool eq = in && bin == tbin;
    uint32_t slot;
    warp_append(eq, &cnt[0], &slot);
    if (eq) {
      if (slot < (uint32_t)p.Nmax) p.ws.cand[(size_t)b * p.Nmax + slot] = ((uint64_t)key << 32) | (uint32_t)j;
      else report(p.dev_status, CSA_ERR_DEVICE);
    }
  }
  for (int o = 16; o > 0; o >>= 1) above += __shfl_xor_sync(0xffffffffu, above, o);
  if ((tid & 31) == 0 && above) atomicAdd(&sh_above, above);
  __syncthreads();
  if (tid == 0) {
    scnt[sblk] = sh_above;
    __threadfence();
    sh_last = atomicAdd(&cnt[1], 1u) == (uint32_t)(S_b - 1);
  }
  __syncthreads();
  if (!sh_last) return;
  __threadfence();

  // 3. the last CTA of the sequence: exact cut inside the bin
  uint32_t part = 0;
  for (int s2 = tid; s2 < S_b; s2 += kSelThreads) part += __ldcg(scnt + s2);
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if (tid == 0) sh_sum = 0;
  __syncthreads();
  if ((tid & 31) == 0 && part) atomicAdd(&sh_sum, part);
  __syncthreads();
  const uint32_t above_total = sh_sum;
  uint32_t n_cand = __ldcg(&cnt[0]);
  if (n_cand > (uint32_t)p.Nmax) n_cand = (uint32_t)p.Nmax;
  const uint64_t* cand = p.ws.cand + (size_t)b * p.Nmax;
  const bool staged = n_cand <= kCandStage;
  if (staged) {
    for (uint32_t i = tid; i < n_cand; i += kSelThreads) cand_s[i] = __ldcg(cand + i);
    cand = cand_s;
    __syncthreads();
  }
  // rule: entry j with key is selected iff key > cut_key, or key == cut_key and
  // j <= cut_idx (a signed index; -1 takes none of the entries at the cut key)
  uint32_t cut_key;
  int32_t cut_idx;
  if (tbin < 0) {  // every entry is selected
    cut_key = 0u;
    cut_idx = 0x7FFFFFFF;
  } else {
    const uint32_t need = (uint32_t)k_eff > above_total ? (uint32_t)k_eff - above_total : 0u;
    if (need == 0) {  // the bin contributes nothing
      cut_key = ((uint32_t)(tbin + 1) << (32 - kHistBits)) - 1u;
      cut_idx = -1;
    } else if (need >= n_cand) {  // the whole bin (need > n_cand means inconsistent data)
      if (need > n_cand) report(p.dev_status, CSA_ERR_DEVICE);
      cut_key = (uint32_t)tbin << (32 - kHistBits);
      cut_idx = 0x7FFFFFFF;
    } else {
      // key: the need-th largest among the candidates (20 bits below the bin)
      if (tid == 0) { sh_prefix = (uint32_t)tbin << (32 - kHistBits); sh_rem = need; }
      __syncthreads();
      const uint32_t top = ~0u << (32 - kHistBits);
      radix_step(cand, staged, n_cand, true, 0, false, top, 12, 8, true, &sh_prefix, &sh_rem, h);
      radix_step(cand, staged, n_cand, true, 0, false, top | (0xFFu << 12), 4, 8, true, &sh_prefix,
                 &sh_rem, h);
      radix_step(cand, staged, n_cand, true, 0, false, top | (0xFFFu << 8) | 0xF0u, 0, 4, true,
                 &sh_prefix, &sh_rem, h, &sh_pop);
      cut_key = sh_prefix;
      // sh_rem entries with key == cut_key are taken, sh_pop exist
      if (sh_pop == sh_rem) {
        cut_idx = 0x7FFFFFFF;
      } else {  // a tie at the cut: the sh_rem smallest indices (4 ascending 8-bit passes)
        __syncthreads();
        if (tid == 0) sh_prefix = 0;
        __syncthreads();
        radix_step(cand, staged, n_cand, false, cut_key, true, 0u, 24, 8, false, &sh_prefix, &sh_rem, h);
        radix_step(cand, staged, n_cand, false, cut_key, true, 0xFF000000u, 16, 8, false, &sh_prefix,
                   &sh_rem, h);
        radix_step(cand, staged, n_cand, false, cut_key, true, 0xFFFF0000u, 8, 8, false, &sh_prefix,
                   &sh_rem, h);
        radix_step(cand, staged, n_cand, false, cut_key, true, 0xFFFFFF00u, 0, 8, false, &sh_prefix,
                   &sh_rem, h);
        cut_idx = (int32_t)sh_prefix;
      }
    }
  }
  // selected count per slice: above-bin entries plus the candidates that pass the cut
  for (uint32_t i = tid; i < n_cand; i += kSelThreads) {
    const uint64_t c = cand_at(cand, i, staged);
    const uint32_t key = (uint32_t)(c >> 32), j = (uint32_t)c;
    if (tbin >= 0 && (key > cut_key || (key == cut_key && (int32_t)j <= cut_idx)))
      atomicAdd(scnt + j / kSelChunk, 1u);
  }
  __threadfence();
  __syncthreads();
  // exclusive scan of the slice counts -> output offsets
  uint32_t carry = 0;
  for (int base = 0; base < S_b; base += kSelThreads) {
    const int s2 = base + tid;
    const uint32_t v = s2 < S_b ? __ldcg(scnt + s2) : 0u;
    uint32_t tot;
    const uint32_t incl = block_incl_scan(v, tmp, &tot);
    if (s2 < S_b) scnt[s2] = carry + incl - v;
    carry += tot;
    __syncthreads();
  }
  if (tid == 0) {
    uint32_t* r = p.ws.rule + (size_t)b * 4;
    r[0] = cut_key;
    r[1] = (uint32_t)cut_idx;
    r[2] = (uint32_t)k_eff;
    if (carry != (uint32_t)k_eff) report(p.dev_status, CSA_ERR_DEVICE);
    cnt[0] = 0;
    cnt[1] = 0;
  }
  uint32_t* gh = p.ws.hist + (size_t)b * kHist;
  for (int i = tid; i < kHist; i += kSelThreads) gh[i] = 0;
}

__global__ void __launch_bounds__(kSelThreads) topk_write_kernel(SelParams p) {
  __shared__ uint32_t tmp[kSelThreads / 32];
  const int b = blockIdx.y, sblk = blockIdx.x, tid = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  int n = p.n_entries[b];
  n = n < 0 ? 0 : (n > p.Nmax ? (int)p.Nmax : n);
  const int S_b = n == 0 ? 1 : (n + kSelChunk - 1) / kSelChunk;
  if (sblk >= S_b) return;
  const uint32_t* r = p.ws.rule + (size_t)b * 4;
  const uint32_t cut_key = __ldcg(r), k_eff = __ldcg(r + 2);
  const int32_t cut_idx = (int32_t)__ldcg(r + 1);
  const uint32_t off = __ldcg(p.ws.slice_cnt + (size_t)b * p.ws.S + sblk);
  const float* sc = p.ws.scores + (size_t)b * p.Nmax;
  int32_t* out = p.idx + (size_t)b * p.k;
  const int j0 = sblk * kSelChunk, j1 = min(n, j0 + kSelChunk);
  const int jt = j0 + tid * kSelPer;  // 16 consecutive entries per thread
  float v[kSelPer];
  load_scores16(sc, jt, j1, v);
  uint32_t mask = 0;
#pragma unroll
  for (int e = 0; e < kSelPer; ++e) {
    const int j = jt + e;
    const uint32_t key = float_key(v[e]);
    if (j < j1 && (key > cut_key || (key == cut_key && j <= cut_idx))) mask |= 1u << e;
  }
  const uint32_t mine = __popc(mask);
  const uint32_t incl = block_incl_scan(mine, tmp, nullptr);
  uint32_t slot = off + incl - mine;
#pragma unroll
  for (int e = 0; e < kSelPer; ++e) {
    if (mask & (1u << e)) {
      if (slot < (uint32_t)p.k) {
        out[slot] = jt + e;
        if (p.scores_out) p.scores_out[(size_t)b * p.k + slot] = v[e];
      } else {
        report(p.dev_status, CSA_ERR_DEVICE);
      }
      ++slot;
    }
  }
  if (sblk == 0) {
    for (int i = (int)k_eff + tid; i < p.k; i += kSelThreads) {
      out[i] = -1;
      if (p.scores_out) p.scores_out[(size_t)b * p.k + i] = __int_as_float(0x7fc00000);
    }
  }
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
  int grid = kIxCtasPerSm * num_sms;
  if (tiles_max < grid) grid = (int)(tiles_max > 0 ? tiles_max : 1);
  cudaError_t e = launch_pdl(indexer_score_kernel, dim3(grid), dim3(kIxThreads), smem, stream,
                             kmap, p);
  if (e != cudaSuccess) return e;
  SelParams sp{a.B, a.k, a.Nmax, a.n_entries, ws, a.idx, a.scores, a.dev_status};
  dim3 g2((unsigned)ws.S, a.B);
  e = launch_pdl(topk_threshold_kernel, g2, dim3(kSelThreads), 0, stream, sp);
  if (e != cudaSuccess) return e;
  return launch_pdl(topk_write_kernel, g2, dim3(kSelThreads), 0, stream, sp);
}

size_t ix_smem_bytes() { return sizeof(IxSmem) + 1024; }

}  // namespace csa
