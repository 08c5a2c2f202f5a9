// Lightning indexer + top-k (cyqw.cn DeepSeek-V4 walkthrough §2.2: low-rank, low-precision
// indexer queries score the compressed entries and each query keeps the top-k, one set
// for all heads; §3.4 and chooseai.net §二: the indexer QK path runs in MXFP4).
//
// indexer_score_kernel: a persistent, warp-specialised stream over the FP4 keys, launched
// cooperatively with one CTA per SM. Each CTA runs two independent pipelines over two
// halves of its contiguous range of (sequence, 128-entry tile) work items, each pipeline
// with its own warps, shared-memory ring and half of TMEM:
//   producer warp  TMA loads of the 128 x 64-byte key tile (64-byte swizzle) and the
//                  tile's 512-byte scale group into a 6-stage ring;
//   issuer warp    copies the key scales into TMEM (tcgen05.cp), issues two kind::mxf4
//                  block-scaled MMAs (K = 64 each) giving D[128 entries x 64 heads] in fp32
//                  TMEM, three accumulators deep, and stages each sequence's FP4 queries
//                  (B operand) and their scales;
//   4 epilogue warps  one per TMEM lane quadrant, one thread per entry: reads its 64 head
//                  sums, forms s = sum_h w_h * max(0, acc_h) in fp32 (w in registers, head
//                  pairs in packed FMAs; rounded to BF16 when asked), writes the score to
//                  the workspace and counts its order-preserving key into the warp's own
//                  2048-bin histogram (16-bit counters), flushed to the sequence's global
//                  histogram when the warp moves to another sequence.
// After a grid barrier the same CTAs select (no sorting anywhere):
//   select_threshold: per sequence and 12,288-entry slice, the histogram fixes the bin
//     that holds the k-th score (a parallel suffix scan); each CTA counts its entries above
//     that bin and appends the in-bin candidates. The last CTA of a sequence (atomic ticket,
//     no spinning) resolves the exact cut inside the bin by a radix select on the remaining
//     21 key bits (ties broken by the smaller index), turns the per-slice counts into output
//     offsets, clears the histogram and counters for the next call and publishes the cut;
//   select_write: every slice writes its selected entries in index order at its offset, so
//     the output comes out ascending without a sort.
// If the cooperative launch is refused, scoring runs as an ordinary launch followed by the
// same two steps as stand-alone kernels (topk_threshold_kernel, topk_write_kernel). The
// prefill variant (prefill_score_kernel, topk_query_kernel) is described further down.
#include "common.cuh"

namespace csa {

constexpr int kIxTile = 128;        // entries per tile = MMA M
constexpr int kIxN = 64;            // MMA N: indexer heads padded to 64
// The decode kernel: one CTA per SM (cooperative launch), one producer filling a ring of
// key-tile quads, and three pipelines taking the tiles in turn, each an MMA issuer warp and
// a group of four epilogue warps (see the file head).
constexpr int kDxQuad = 4;          // key tiles per copy: one 32 KB tensor copy + 2 KB scales
constexpr int kDxStages = 4;        // quads in flight per SM (136 KB)
constexpr int kDxScTiles = 64;      // a CTA range of up to 64 tiles keeps its scores on chip
constexpr int kDxGroups = 3;        // pipelines: issuer warp + epilogue warp group
constexpr int kDxBufs = 2;          // accumulators per pipeline
constexpr int kDxAcc = kDxGroups * kDxBufs;
constexpr int kDxWarps = 1 + 5 * kDxGroups;
constexpr int kDxThreads = 32 * kDxWarps;
constexpr int kDxTmemCols = 512;
constexpr int kDxMaxCtas = 256;     // grid limit (per-CTA counts in the workspace)
constexpr int kDxCand = 2048;       // in-bin candidates staged in shared memory
static_assert(kDxAcc * 64 + 16 * kDxGroups <= kDxTmemCols,
              "accumulators and scale factors fit TMEM");
constexpr int kIxKeyBytes = kIxTile * 64;
constexpr int kIxSfBytes = 512;
constexpr int kHistBits = 11;       // histogram of the top key bits (sign, exponent, 2 mantissa)
constexpr int kLowBits = 32 - kHistBits;
constexpr int kHist = 1 << kHistBits;
constexpr int kIxMaxB = 1024;
constexpr int kSelThreads = 384;            // threads of the stand-alone selection kernels
constexpr int kSelPer = 32;                 // consecutive entries per thread
constexpr int kSelChunk = kSelThreads * kSelPer;  // entries per slice

// Workspace layout of csa_indexer_topk (all regions 256-byte aligned). Everything that must
// be zero when a call starts sits at the front at offsets that do not depend on B: the
// grid barriers, then one fixed-size block per sequence (counters, rule, histogram). A call
// with fewer sequences therefore finds its blocks where a larger call left them zeroed.
constexpr int kSeqWords = 8 + kHist;  // per-sequence block: counters[4], rule[4], hist

struct IxWs {
  uint32_t* grid_bar;   // the two grid barriers' 64-bit counters, at words 0 and 32
  uint32_t* seq;        // [B][kSeqWords]
  uint32_t* slice_cnt;  // [B][S]: above-bin count per slice, then the slice's output offset
  float* scores;        // [B][Nmax]
  uint64_t* cand;       // [B][Nmax]: (key << 32) | index of the in-bin candidates
  uint4* cta_cnt;       // [B][kDxMaxCtas]: per CTA (above-bin count, in-bin count, bin)
  uint64_t* cand_slots; // [B][kDxMaxCtas][32]: per CTA its first in-bin candidates
  int S;                // slices per sequence
  // counters: candidate count, ticket; rule: cut key, cut index, selected count, ready flag
  __device__ uint32_t* counters(int b) const { return seq + (size_t)b * kSeqWords; }
  __device__ uint32_t* rule(int b) const { return seq + (size_t)b * kSeqWords + 4; }
  __device__ uint32_t* hist(int b) const { return seq + (size_t)b * kSeqWords + 8; }
};
static_assert((kSeqWords * 4) % 16 == 0, "histograms stay 16-byte aligned");

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
  char* p0 = take(512);
  char* p1 = take((size_t)B * kSeqWords * 4);
  char* p2 = take((size_t)B * S * 4);
  char* p3 = take((size_t)B * Nmax * 4);
  char* p4 = take((size_t)B * Nmax * 8);
  char* p5 = take((size_t)B * kDxMaxCtas * sizeof(uint4));
  char* p6 = take((size_t)B * kDxMaxCtas * 32 * sizeof(uint64_t));
  if (ws) {
    ws->grid_bar = (uint32_t*)p0;
    ws->seq = (uint32_t*)p1;
    ws->slice_cnt = (uint32_t*)p2;
    ws->scores = (float*)p3;
    ws->cand = (uint64_t*)p4;
    ws->cta_cnt = (uint4*)p5;
    ws->cand_slots = (uint64_t*)p6;
    ws->S = S;
  }
  return off;
}

size_t ix_workspace_size(int B, int64_t Nmax, int k) {
  return ix_ws_layout(B, Nmax, k, nullptr, nullptr);
}

struct IxParams {
  int B, H_I, k;
  int fused;  // 1: the selection follows in this (cooperative) launch
  int bf16;   // 1: scores are rounded to BF16 before they are stored and selected
  uint64_t wait_ns;  // limit of the selection's grid-barrier waits
  int64_t Nmax;
  const int32_t* n_entries;
  const uint8_t* q_fp4;
  const uint8_t* q_sf;
  const float* w;
  const uint8_t* k_sf;
  IxWs ws;
  int32_t* idx;
  float* scores_out;
  int32_t* dev_status;
  PageMap pm;  // where the keys live (contiguous, or paged)
  int tpl;     // paged keys: key tiles per copy (min(4, tiles per page))
};

__device__ __forceinline__ int clamp_n(int n, int64_t Nmax, int32_t* st) {
  if (n < 0 || n > Nmax) {
    report(st, CSA_ERR_DEVICE);
    return n < 0 ? 0 : (int)Nmax;
  }
  return n;
}

struct alignas(1024) DxSmem {
  uint8_t keys[kDxStages][kDxQuad][kIxKeyBytes];  // quads of key tiles (64-byte swizzle)
  uint8_t q[kDxGroups][2][kIxN * 64];     // queries (B operand) per pipeline, two slots
  float sc[kDxScTiles * kIxTile];         // the CTA's scores (fused path, small ranges)
  uint8_t ksf[kDxStages][kDxQuad][kIxSfBytes];  // key scale groups
  uint8_t qsf[kDxGroups][2][512];         // query scale atoms
  uint32_t hist[kDxGroups][kHist / 2];    // per-group histograms, two 16-bit bins per word
  alignas(16) float w[kDxGroups][2][kIxN];  // head weights of each group's sequence (read
                                            // as float4)
  int32_t qprefix[kIxMaxB + 1];           // quads of sequences 0 .. b-1
  int32_t tiles[kIxMaxB];                 // tiles of sequence b: ceil(n_b / 128)
  uint64_t full[kDxStages], empty[kDxStages];
  uint64_t acc_full[kDxAcc], acc_empty[kDxAcc], q_free[kDxGroups][2], done[kDxGroups];
  uint64_t grp_bar[kDxGroups];            // the four warps of a group meet around a flush
  uint64_t roles_bar;                     // every warp has finished its role
  int32_t grp_seq[kDxGroups];             // sequence whose counts a group histogram holds
  uint32_t tmem_base;
  volatile int abort;
};
// dynamic shared memory (+1 KB for alignment) and the static kilobyte of the helpers fit
// the 227 KB a CTA may hold
static_assert(sizeof(DxSmem) + 2048 <= 232448, "decode kernel shared memory");
static_assert(offsetof(DxSmem, w) % 16 == 0 && offsetof(DxSmem, q) % 1024 == 0 &&
                  offsetof(DxSmem, keys) % 1024 == 0 && offsetof(DxSmem, ksf) % 16 == 0 &&
                  offsetof(DxSmem, qsf) % 16 == 0 && offsetof(DxSmem, hist) % 16 == 0 &&
                  offsetof(DxSmem, sc) % 16 == 0,
              "vector and bulk-copy fields of the decode kernel's shared memory are aligned");

__device__ void select_decode(const IxParams& p, uint8_t* scratch, const DxSmem& s, int q0,
                              int q1, bool on_chip, bool ok);

// Adds a histogram of two 16-bit bins per word to sequence bb's global histogram: lanes
// [from, from + stride) of the calling threads take every stride-th word.
__device__ __forceinline__ void hist_flush(uint32_t* h, uint32_t* gh, int from, int stride) {
  for (int i = from; i < kHist / 2; i += stride) {
    const uint32_t v = h[i];
    if (v) {
      if (v & 0xFFFFu) atomicAdd(gh + 2 * i, v & 0xFFFFu);
      if (v >> 16) atomicAdd(gh + 2 * i + 1, v >> 16);
      h[i] = 0;
    }
  }
}

// The four warps of an epilogue group meet on an mbarrier (bounded wait): lane 0 of each
// warp arrives, then waits for the phase to complete. The warp synchronises first, so the
// shared-memory writes of all its lanes are ordered before lane 0's arrival (a release)
// and visible to the warps that return from the wait (an acquire).
__device__ __forceinline__ bool group_meet(uint64_t* bar, uint32_t& phase, int32_t* st) {
  bool ok = true;
  __syncwarp();
  if ((threadIdx.x & 31) == 0) {
    mbar_arrive(bar);
    ok = mbar_wait(bar, phase, st);
  }
  phase ^= 1;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// The CTA's tiles in order: quads q0 .. q1-1 (quad q of sequence b = the tiles 4(q - qprefix[b])
// .. +3 that exist), numbered it = 0, 1, ... over the CTA. Calls f(b, t, it, qq, sub, nt):
// sequence, tile within the sequence, CTA tile index, CTA quad index, slot in the quad,
// tiles in the quad. Stops early when f returns false.
template <typename F>
__device__ __forceinline__ void for_each_tile(const DxSmem& s, int q0, int q1, int b0, F&& f) {
  int b = b0, it = 0;
  for (int q = q0, qq = 0; q < q1; ++q, ++qq) {
    while (s.qprefix[b + 1] <= q) ++b;
    const int t0 = kDxQuad * (q - s.qprefix[b]);
    const int nt = min(kDxQuad, s.tiles[b] - t0);
    for (int sub = 0; sub < nt; ++sub, ++it)
      if (!f(b, t0 + sub, it, qq, sub, nt)) return;
  }
}

__global__ void __launch_bounds__(kDxThreads, 1)
    indexer_decode_kernel(const __grid_constant__ CUtensorMap kmap, IxParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  DxSmem& s = *reinterpret_cast<DxSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // set-up that touches no global memory overlaps the previous kernel's tail
  if (warp == 1 && lane == 0) {
    for (int i = 0; i < kDxStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], kDxQuad);  // one MMA commit per tile of the quad
    }
    for (int i = 0; i < kDxAcc; ++i) {
      mbar_init(&s.acc_full[i], 1);
      mbar_init(&s.acc_empty[i], 4);
    }
    for (int i = 0; i < kDxGroups; ++i) {
      mbar_init(&s.q_free[i][0], 1);
      mbar_init(&s.q_free[i][1], 1);
      mbar_init(&s.grp_bar[i], 4);
      mbar_init(&s.done[i], 1);
    }
    mbar_init(&s.roles_bar, kDxWarps);
    s.abort = 0;
    mbar_fence_init();
  }
  if (threadIdx.x == 0) prefetch_tensormap(&kmap);
  for (int i = threadIdx.x; i < kDxGroups * kHist / 2; i += kDxThreads) (&s.hist[0][0])[i] = 0;
  if (threadIdx.x < kDxGroups) s.grp_seq[threadIdx.x] = -1;
  if (warp == 1) tmem_alloc(&s.tmem_base, kDxTmemCols);
  pdl_wait();
  pdl_trigger();

  // Schedule: sequence b owns ceil(n_b / 128) tiles in ceil(tiles / 4) quads; CTA c takes a
  // contiguous range of quads.
  if (warp == 0) {
    int carry = 0;
    if (lane == 0) s.qprefix[0] = 0;
    for (int base = 0; base < p.B; base += 32) {
      const int bb = base + lane;
      int v = 0;
      if (bb < p.B) {
        const int t = (clamp_n(p.n_entries[bb], p.Nmax, p.dev_status) + kIxTile - 1) / kIxTile;
        s.tiles[bb] = t;
        v = (t + kDxQuad - 1) / kDxQuad;
      }
      int incl = v;
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (bb < p.B) s.qprefix[bb + 1] = carry + incl;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int total = s.qprefix[p.B];
  const int q0 = (int)((int64_t)total * blockIdx.x / gridDim.x);
  const int q1 = (int)((int64_t)total * (blockIdx.x + 1) / gridDim.x);
  const uint32_t tmem = s.tmem_base;
  // fused path with a short range: scores stay in shared memory
  const bool on_chip = p.fused && (q1 - q0) * kDxQuad <= kDxScTiles;
  int b0 = 0;  // first sequence of this CTA
  while (b0 < p.B && s.qprefix[b0 + 1] <= q0) ++b0;

  if (q0 < q1 && warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int b = b0, qq = 0;
      const int groups = (int)(p.Nmax / kIxTile);
      const uint64_t stream_policy = l2_evict_first_policy();  // keys are read once
      for (int q = q0; q < q1; ++q, ++qq) {
        while (s.qprefix[b + 1] <= q) ++b;
        const int t0 = kDxQuad * (q - s.qprefix[b]);
        const int st = qq % kDxStages;
        if (s.abort || !mbar_wait(&s.empty[st], ((qq / kDxStages) & 1) ^ 1, p.dev_status)) {
          s.abort = 1;
          break;
        }
        if (!p.pm.table) {
          // the quad's four key tiles in one tensor copy (tiles past Nmax read as zeros;
          // tiles past n_b are read but not scored) and the scale groups that exist
          const uint32_t sf_bytes = (uint32_t)min(kDxQuad, groups - t0) * kIxSfBytes;
          mbar_arrive_expect_tx(&s.full[st], kDxQuad * kIxKeyBytes + sf_bytes);
          tma_load_4d_hint(&s.keys[st][0][0], &kmap, &s.full[st], 0, 0, t0, b, stream_policy);
          bulk_load_hint(&s.ksf[st][0][0], p.k_sf + ((size_t)b * groups + t0) * kIxSfBytes,
                         sf_bytes, &s.full[st], stream_policy);
        } else {
          // paged keys: copies of tpl tiles from the page of each (a page holds whole
          // copies); tiles past n_b that lie in another page are not read (their slots
          // keep stale keys, which are not scored)
          int64_t e[kDxQuad];
          int nl = 0;
          for (int t = t0; t < t0 + kDxQuad && t < s.tiles[b]; t += p.tpl)
            e[nl++] = page_entry(p.pm, b, (int64_t)t * kIxTile);
          mbar_arrive_expect_tx(&s.full[st], (uint32_t)(nl * p.tpl) * (kIxKeyBytes + kIxSfBytes));
          const int64_t tiles_pp = ((int64_t)1 << p.pm.shift) / kIxTile;
          for (int l = 0; l < nl; ++l) {
            int64_t el = e[l];
            if (el < 0) {  // a page outside the pool: reported; the first page is read instead
              report(p.dev_status, CSA_ERR_DEVICE);
              el = 0;
            }
            const int64_t g = el / kIxTile;  // the copy's first key group in the pool
            tma_load_4d_hint(&s.keys[st][l * p.tpl][0], &kmap, &s.full[st], 0, 0,
                             (int)(g % tiles_pp), (int)(g / tiles_pp), stream_policy);
            bulk_load_hint(&s.ksf[st][l * p.tpl][0], p.k_sf + (size_t)g * kIxSfBytes,
                           (uint32_t)p.tpl * kIxSfBytes, &s.full[st], stream_policy);
          }
        }
      }
      // drain: every copy this warp issued has landed before the CTA winds down
      const int issued = qq;
      for (int i = issued - kDxStages < 0 ? 0 : issued - kDxStages; i < issued; ++i)
        mbar_wait(&s.full[i % kDxStages], (i / kDxStages) & 1, p.dev_status);
    }
    __syncwarp();  // the warp reaches the CTA barrier below converged
  } else if (q0 < q1 && warp <= kDxGroups) {
    // ---------------------------------------------------------------- MMA issuers
    // issuer pi takes the tiles it = pi, pi + 3, ... into its pipeline's two accumulators;
    // its key and query scale factors have TMEM columns of their own
    const int pi = warp - 1;
    const uint32_t t_sfa = tmem + kDxAcc * kIxN + 16 * pi, t_sfb = t_sfa + 8;
    int cur = -1, nseq = -1;
    uint32_t qslot = 0;
    for_each_tile(s, q0, q1, b0, [&](int b, int t, int it, int qq, int sub, int nt) -> bool {
      (void)t;
      if (it % kDxGroups != pi) return true;
      const int u = it / kDxGroups;
      if (b != cur) {  // stage this sequence's queries (B operand) and their scales
        if (cur >= 0 && lane == 0) mma_commit(&s.q_free[pi][qslot]);
        cur = b;
        ++nseq;
        qslot = nseq & 1;
        bool ok = true;
        if (lane == 0) ok = !s.abort && mbar_wait(&s.q_free[pi][qslot], ((nseq >> 1) & 1) ^ 1,
                                                  p.dev_status);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) { s.abort = 1; return false; }
        const uint8_t* qsrc = p.q_fp4 + (size_t)b * p.H_I * 64;
        uint8_t* qdst = s.q[pi][qslot];
        for (int c = lane; c < kIxN * 4; c += 32) {  // 16-byte chunks, 64-byte swizzle
          const int r = c >> 2, ch = c & 3;
          uint4 v = make_uint4(0, 0, 0, 0);
          if (r < p.H_I) v = *reinterpret_cast<const uint4*>(qsrc + r * 64 + ch * 16);
          *reinterpret_cast<uint4*>(&qdst[r * 64 + ((ch ^ ((r >> 1) & 3)) << 4)]) = v;
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
          *reinterpret_cast<uint4*>(&s.qsf[pi][qslot][lane * 16]) =
              make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tc_fence_after();
          tmem_cp_32x128b_x4(t_sfb, smem_desc(smem_u32(s.qsf[pi][qslot]), 0, 128, kSwizzleNone));
        }
      }
      if (lane == 0) {
        const int st = qq % kDxStages, buf = pi * kDxBufs + (u & 1);
        bool ok = !s.abort;
        if (ok) {
          ok = mbar_wait(&s.acc_empty[buf], ((u >> 1) & 1) ^ 1, p.dev_status);
          // the epilogue's TMEM reads of this buffer happen before our MMAs overwrite it
          tc_fence_after();
        }
        // (the key tile arrives through the async proxy: the barrier alone orders it)
        ok = ok && mbar_wait(&s.full[st], (qq / kDxStages) & 1, p.dev_status);
        if (!ok) {
          s.abort = 1;
        } else {
          tmem_cp_32x128b_x4(t_sfa, smem_desc(smem_u32(s.ksf[st][sub]), 0, 128, kSwizzleNone));
          const uint32_t ka = smem_u32(s.keys[st][sub]), qa = smem_u32(s.q[pi][qslot]);
#pragma unroll
          for (int kh = 0; kh < 2; ++kh) {
            mma_mxf4(tmem + buf * kIxN, smem_desc(ka + 32 * kh, 16, 512, kSwizzle64B),
                     smem_desc(qa + 32 * kh, 16, 512, kSwizzle64B),
                     idesc_mxf4(kIxTile, kIxN, 2 * kh), t_sfa, t_sfb, kh);
          }
          // the stage is free once the MMAs of all its tiles have read it: one arrival per
          // tile, and the last tile of a short quad also stands in for the missing ones
          const int arrivals = sub == nt - 1 ? 1 + kDxQuad - nt : 1;
          for (int a = 0; a < arrivals; ++a) mma_commit(&s.empty[st]);
          mma_commit(&s.acc_full[buf]);
        }
      }
      return __shfl_sync(0xffffffffu, s.abort, 0) == 0;
    });
    if (lane == 0) {  // every tcgen05 operation of this issuer has completed
      mma_commit(&s.done[pi]);
      mbar_wait(&s.done[pi], 0, p.dev_status);
    }
    __syncwarp();
  } else if (q0 < q1) {
    // ---------------------------------------------------------------- epilogue
    const int ew = warp - 1 - kDxGroups, gi = ew >> 2;  // epilogue warp, its pipeline
    const int quad = warp & 3;              // TMEM lane quadrant
    const int row = quad * 32 + lane;       // entry within the tile
    uint32_t* hist = s.hist[gi];
    uint32_t meet_phase = 0;
    int cur = -1, n_b = 0, since_flush = 0, wsl = 1;
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    for_each_tile(s, q0, q1, b0, [&](int b, int t, int it, int qq, int sub, int nt) -> bool {
      (void)qq; (void)sub; (void)nt;
      if (it % kDxGroups != gi) return true;
      const int u = it / kDxGroups;
      const int buf = gi * kDxBufs + (u & 1);
      bool ok = true;
      if (lane == 0) ok = !s.abort && mbar_wait(&s.acc_full[buf], (u >> 1) & 1, p.dev_status);
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        s.abort = 1;
        return false;
      }
      tc_fence_after();
      // 16-bit counters: a group adds 128 counts per tile, so flush every 400 tiles
      // (< 65536 counts) as well as whenever the sequence changes; the group's four warps
      // meet before the flush (all counts added) and after it (bins cleared). The head
      // weights of a new sequence go to the other weight slot, which no warp of the group
      // still reads once the first meeting has passed.
      if (b != cur || since_flush == 400) {
        if (cur >= 0) {
          if (!group_meet(&s.grp_bar[gi], meet_phase, p.dev_status)) { s.abort = 1; return false; }
          hist_flush(hist, p.ws.hist(cur), (ew & 3) * 32 + lane, 128);
        }
        if (b != cur) {
          wsl ^= 1;
          if ((ew & 3) == 0)
            for (int h = lane; h < kIxN; h += 32)
              s.w[gi][wsl][h] = h < p.H_I ? __ldg(p.w + (size_t)b * p.H_I + h) : 0.f;
        }
        if (!group_meet(&s.grp_bar[gi], meet_phase, p.dev_status)) { s.abort = 1; return false; }
        since_flush = 0;
        cur = b;
        n_b = clamp_n(p.n_entries[cur], p.Nmax, nullptr);
      }
      ++since_flush;
      // s = sum_h w_h * max(0, acc_h): eight independent partial sums (heads h = k mod 8)
      // combined in a fixed tree; all 64 columns are read before one wait
      uint32_t r[2][32];
      const uint32_t ta = lane_base + buf * kIxN;
      tmem_ld32(ta, r[0]);
      tmem_ld32(ta + 32, r[1]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.acc_empty[buf]);  // TMEM reads done: buffer free
      const float4* w4 = reinterpret_cast<const float4*>(s.w[gi][wsl]);
      float part[8];
#pragma unroll
      for (int k8 = 0; k8 < 8; ++k8) part[k8] = 0.f;
#pragma unroll
      for (int h4 = 0; h4 < kIxN / 4; ++h4) {
        const float4 wv = w4[h4];
        const int h = 4 * h4;
        fma2(part[h & 7], part[(h + 1) & 7], wv.x, wv.y,
             fmaxf(__uint_as_float(r[h >> 5][h & 31]), 0.f),
             fmaxf(__uint_as_float(r[(h + 1) >> 5][(h + 1) & 31]), 0.f));
        fma2(part[(h + 2) & 7], part[(h + 3) & 7], wv.z, wv.w,
             fmaxf(__uint_as_float(r[(h + 2) >> 5][(h + 2) & 31]), 0.f),
             fmaxf(__uint_as_float(r[(h + 3) >> 5][(h + 3) & 31]), 0.f));
      }
      float sc = ((part[0] + part[1]) + (part[2] + part[3])) +
                 ((part[4] + part[5]) + (part[6] + part[7]));
      if (p.bf16) sc = bf16_bits_to_f32(f32_to_bf16_bits(sc));
      const int j = t * kIxTile + row;
      if (j < n_b) {
        if (on_chip) s.sc[it * kIxTile + row] = sc;
        else p.ws.scores[(size_t)cur * p.Nmax + j] = sc;
        const uint32_t bin = float_key(sc) >> (32 - kHistBits);
        atomicAdd(&hist[bin >> 1], 1u << (16 * (bin & 1)));
      }
      return true;
    });
    if ((ew & 3) == 0 && lane == 0) s.grp_seq[gi] = cur;
  }
  // Every warp has finished its role: a bounded meeting on an mbarrier first. (The CTA
  // barrier alone, right after the roles, was seen to let thread 0 through while epilogue
  // warps were still scoring their last tiles, and the histogram sum below must see all of
  // their counts.)
  tc_fence_before();
  {
    uint32_t roles_phase = 0;
    if (!group_meet(&s.roles_bar, roles_phase, p.dev_status)) s.abort = 1;
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kDxTmemCols);
  }
  // the groups' last histograms: counts of groups holding the same sequence are summed
  // here, so each bin costs one global atomic per CTA
  for (int gi = 0; gi < kDxGroups; ++gi) {
    const int b = s.grp_seq[gi];
    bool first = b >= 0;
    for (int gj = 0; gj < gi; ++gj) first = first && s.grp_seq[gj] != b;
    if (!first) continue;
    uint32_t* gh = p.ws.hist(b);
    for (int bin = threadIdx.x; bin < kHist; bin += kDxThreads) {
      uint32_t c = 0;
      for (int gj = gi; gj < kDxGroups; ++gj)
        if (s.grp_seq[gj] == b) c += (s.hist[gj][bin >> 1] >> (16 * (bin & 1))) & 0xFFFFu;
      if (c) atomicAdd(gh + bin, c);
    }
  }
  const bool ok = !__syncthreads_or(s.abort);
  if (p.fused)
    select_decode(p, reinterpret_cast<uint8_t*>(&s.keys[0][0][0]), s, q0, q1, on_chip, ok);
}

// ------------------------------------------------------------------- select
// Static shared-memory scratch of the stand-alone selection kernels.
struct SelScratch {
  uint32_t h[kHist];
  uint64_t cand[2048];
  uint32_t tmp[32];
  int tbin, last;
  uint32_t above, prefix, rem, sum, pop;
};
constexpr uint32_t kCandStage = 2048;

// Inclusive scan over the CTA (NT threads); tmp holds one word per warp.
template <int NT = kSelThreads>
__device__ __forceinline__ uint32_t block_incl_scan(uint32_t v, uint32_t* tmp, uint32_t* total) {
  constexpr int nw = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  __syncthreads();
  if (lane == 31) tmp[warp] = v;
  __syncthreads();
  uint32_t before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < nw; ++w) {
    const uint32_t t = tmp[w];
    if (w < warp) before += t;
    all += t;
  }
  if (total) *total = all;
  return v + before;
}

// scores[j .. j+31] (entries at or past `end` read as 0 and are never used)
__device__ __forceinline__ void load_scores(const float* sc, int j, int end,
                                            float (&v)[kSelPer]) {
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

// Candidates come from shared memory (staged) or, past its capacity, from global memory.
__device__ __forceinline__ uint64_t cand_at(const uint64_t* cand, uint32_t i, bool staged) {
  return staged ? cand[i] : __ldcg(cand + i);
}

// Radix-select step over the candidates: among those whose field matches `prefix` under
// `mask`, histogram the digit (field >> shift) & (2^bits - 1) and find the digit where the
// running count (from the top when `descending`, else from the bottom) reaches *remaining.
// Updates *prefix / *remaining (shared). Field: key = cand >> 32 (hi) or index (lo).
// Candidates are read through `get(i)` (the staged or global list).
template <int NT, typename Get>
__device__ void radix_step_g(const Get& get, uint32_t n_cand, bool hi, uint32_t key_eq,
                             bool need_key_eq, uint32_t mask, int shift, int bits,
                             bool descending, uint32_t* prefix, uint32_t* remaining, uint32_t* h,
                             uint32_t* digit_pop = nullptr) {
  const int tid = threadIdx.x;
  const uint32_t nd = 1u << bits;
  for (uint32_t i = tid; i < nd; i += NT) h[i] = 0;
  __syncthreads();
  const uint32_t pre = *prefix;
  for (uint32_t i = tid; i < n_cand; i += NT) {
    const uint64_t c = get(i);
    const uint32_t key = (uint32_t)(c >> 32), ix = (uint32_t)c;
    if (need_key_eq && key != key_eq) continue;
    const uint32_t f = hi ? key : ix;
    if ((f & mask) == pre) atomicAdd(&h[(f >> shift) & (nd - 1)], 1u);
  }
  __syncthreads();
  if (threadIdx.x < 32) {  // one warp: nd/32 digits per lane, walked in the chosen direction
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
    if (incl >= rem && incl - mine < rem) {
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

__device__ void radix_step(const uint64_t* cand, bool staged, uint32_t n_cand, bool hi,
                           uint32_t key_eq, bool need_key_eq, uint32_t mask, int shift,
                           int bits, bool descending, uint32_t* prefix, uint32_t* remaining,
                           uint32_t* h, uint32_t* digit_pop = nullptr) {
  radix_step_g<kSelThreads>([&](uint32_t i) { return cand_at(cand, i, staged); }, n_cand, hi,
                            key_eq, need_key_eq, mask, shift, bits, descending, prefix,
                            remaining, h, digit_pop);
}

__device__ __forceinline__ int slices_of(int n) {
  return n == 0 ? 1 : (n + kSelChunk - 1) / kSelChunk;
}

// Phase 1 of the selection for slice sb of sequence b: the threshold bin (highest bin whose
// suffix count reaches k), the slice's count above it and its in-bin candidates. The last
// slice of the sequence to finish resolves the exact cut (finalize).
__device__ void select_threshold(const IxParams& p, SelScratch& x, int b, int sb) {
  const int tid = threadIdx.x;
  const int n = clamp_n(p.n_entries[b], p.Nmax, p.dev_status);
  const int k_eff = n < p.k ? n : p.k;
  const int S_b = slices_of(n);
  uint32_t* cnt = p.ws.counters(b);
  uint32_t* scnt = p.ws.slice_cnt + (size_t)b * p.ws.S;
  const float* sc = p.ws.scores + (size_t)b * p.Nmax;

  if (tid == 0) { x.tbin = -1; x.above = 0; }
  if (n > p.k) {
    const uint4* gh = reinterpret_cast<const uint4*>(p.ws.hist(b));
    constexpr int nv = kHist / 4, vper = (nv + kSelThreads - 1) / kSelThreads;
    uint4 hv[vper];  // every load in flight before any is stored
#pragma unroll
    for (int i = 0; i < vper; ++i) {
      const int q = tid + i * kSelThreads;
      hv[i] = q < nv ? __ldcg(gh + q) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < vper; ++i) {
      const int q = tid + i * kSelThreads;
      if (q < nv) reinterpret_cast<uint4*>(x.h)[q] = hv[i];
    }
    __syncthreads();
    constexpr int per = (kHist + kSelThreads - 1) / kSelThreads;  // thread 0 holds the top
    uint32_t mine = 0;
    for (int i = 0; i < per; ++i) {
      const int r = tid * per + i;
      if (r < kHist) mine += x.h[kHist - 1 - r];
    }
    const uint32_t incl = block_incl_scan(mine, x.tmp, nullptr);
    if (incl >= (uint32_t)p.k && incl - mine < (uint32_t)p.k) {
      uint32_t cum = incl - mine;
      for (int i = 0; i < per; ++i) {
        const int r = tid * per + i;
        if (r >= kHist) break;
        const int bin = kHist - 1 - r;
        if (cum + x.h[bin] >= (uint32_t)p.k) { x.tbin = bin; break; }
        cum += x.h[bin];
      }
    }
  }
  __syncthreads();
  const int tbin = x.tbin;

  const int j0 = sb * kSelChunk, j1 = min(n, j0 + kSelChunk);
  const int jt = j0 + tid * kSelPer;
  float v[kSelPer];
  load_scores(sc, jt, j1, v);
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
  if ((tid & 31) == 0 && above) atomicAdd(&x.above, above);
  __syncthreads();
  if (tid == 0) {
    scnt[sb] = x.above;
    __threadfence();
    x.last = atomicAdd(&cnt[1], 1u) == (uint32_t)(S_b - 1);
  }
  __syncthreads();
  if (!x.last) return;
  __threadfence();

  // ---- finalize: the exact cut inside the bin, per-slice output offsets, workspace reset
  uint32_t part = 0;
  for (int s2 = tid; s2 < S_b; s2 += kSelThreads) part += __ldcg(scnt + s2);
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if (tid == 0) x.sum = 0;
  __syncthreads();
  if ((tid & 31) == 0 && part) atomicAdd(&x.sum, part);
  __syncthreads();
  const uint32_t above_total = x.sum;
  uint32_t n_cand = __ldcg(&cnt[0]);
  if (n_cand > (uint32_t)p.Nmax) n_cand = (uint32_t)p.Nmax;
  const uint64_t* cand = p.ws.cand + (size_t)b * p.Nmax;
  const bool staged = n_cand <= kCandStage;
  if (staged) {
    for (uint32_t base = 0; base < n_cand; base += 8 * kSelThreads) {
      uint64_t cv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t i = base + tid + u * kSelThreads;
        cv[u] = i < n_cand ? __ldcg(cand + i) : 0ull;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t i = base + tid + u * kSelThreads;
        if (i < n_cand) x.cand[i] = cv[u];
      }
    }
    cand = x.cand;
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
      cut_key = ((uint32_t)(tbin + 1) << kLowBits) - 1u;
      cut_idx = -1;
    } else if (need >= n_cand) {  // the whole bin (need > n_cand means inconsistent data)
      if (need > n_cand) report(p.dev_status, CSA_ERR_DEVICE);
      cut_key = (uint32_t)tbin << kLowBits;
      cut_idx = 0x7FFFFFFF;
    } else {
      // key: the need-th largest among the candidates (the kLowBits below the bin), in
      // digits of 8, 8 and kLowBits - 16 bits
      if (tid == 0) { x.prefix = (uint32_t)tbin << kLowBits; x.rem = need; }
      __syncthreads();
      const uint32_t top = ~0u << kLowBits;
      radix_step(cand, staged, n_cand, true, 0, false, top, kLowBits - 8, 8, true, &x.prefix,
                 &x.rem, x.h);
      radix_step(cand, staged, n_cand, true, 0, false, ~0u << (kLowBits - 8), kLowBits - 16, 8,
                 true, &x.prefix, &x.rem, x.h);
      radix_step(cand, staged, n_cand, true, 0, false, ~0u << (kLowBits - 16), 0, kLowBits - 16,
                 true, &x.prefix, &x.rem, x.h, &x.pop);
      cut_key = x.prefix;
      if (x.pop == x.rem) {  // x.rem entries with key == cut_key are taken, x.pop exist
        cut_idx = 0x7FFFFFFF;
      } else {  // a tie at the cut: the x.rem smallest indices (4 ascending 8-bit passes)
        __syncthreads();
        if (tid == 0) x.prefix = 0;
        __syncthreads();
        radix_step(cand, staged, n_cand, false, cut_key, true, 0u, 24, 8, false, &x.prefix,
                   &x.rem, x.h);
        radix_step(cand, staged, n_cand, false, cut_key, true, 0xFF000000u, 16, 8, false,
                   &x.prefix, &x.rem, x.h);
        radix_step(cand, staged, n_cand, false, cut_key, true, 0xFFFF0000u, 8, 8, false,
                   &x.prefix, &x.rem, x.h);
        radix_step(cand, staged, n_cand, false, cut_key, true, 0xFFFFFF00u, 0, 8, false,
                   &x.prefix, &x.rem, x.h);
        cut_idx = (int32_t)x.prefix;
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
    const uint32_t vv = s2 < S_b ? __ldcg(scnt + s2) : 0u;
    uint32_t tot;
    const uint32_t incl = block_incl_scan(vv, x.tmp, &tot);
    if (s2 < S_b) scnt[s2] = carry + incl - vv;
    carry += tot;
    __syncthreads();
  }
  if (tid == 0) {
    uint32_t* r = p.ws.rule(b);
    r[0] = cut_key;
    r[1] = (uint32_t)cut_idx;
    r[2] = (uint32_t)k_eff;
    if (carry != (uint32_t)k_eff) report(p.dev_status, CSA_ERR_DEVICE);
    cnt[0] = 0;
    cnt[1] = 0;
  }
  uint32_t* gh = p.ws.hist(b);
  for (int i = tid; i < kHist; i += kSelThreads) gh[i] = 0;
  __syncthreads();
  __threadfence();
  __syncthreads();
}

// Phase 2: slice sb of sequence b writes its selected entries, in index order, at its offset.
__device__ void select_write(const IxParams& p, SelScratch& x, int b, int sb) {
  const int tid = threadIdx.x;
  int n = p.n_entries[b];
  n = n < 0 ? 0 : (n > p.Nmax ? (int)p.Nmax : n);
  const uint32_t* r = p.ws.rule(b);
  const uint32_t cut_key = __ldcg(r), k_eff = __ldcg(r + 2);
  const int32_t cut_idx = (int32_t)__ldcg(r + 1);
  const uint32_t off = __ldcg(p.ws.slice_cnt + (size_t)b * p.ws.S + sb);
  const float* sc = p.ws.scores + (size_t)b * p.Nmax;
  int32_t* out = p.idx + (size_t)b * p.k;
  const int j0 = sb * kSelChunk, j1 = min(n, j0 + kSelChunk);
  const int jt = j0 + tid * kSelPer;
  float v[kSelPer];
  load_scores(sc, jt, j1, v);
  uint32_t mask = 0;
#pragma unroll
  for (int e = 0; e < kSelPer; ++e) {
    const int j = jt + e;
    const uint32_t key = float_key(v[e]);
    if (j < j1 && (key > cut_key || (key == cut_key && j <= cut_idx))) mask |= 1u << e;
  }
  const uint32_t mine = __popc(mask);
  const uint32_t incl = block_incl_scan(mine, x.tmp, nullptr);
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
  if (sb == 0) {
    for (int i = (int)k_eff + tid; i < p.k; i += kSelThreads) {
      out[i] = -1;
      if (p.scores_out) p.scores_out[(size_t)b * p.k + i] = __int_as_float(0x7fc00000);
    }
  }
  __syncthreads();
}

// ------------------------------------------------------- decode selection (fused)
// Grid-wide barrier of the cooperative decode launch on a 64-bit arrival counter that only
// grows: a CTA's arrival returns the count before it, which fixes the barrier instance it
// belongs to (all CTAs of a launch arrive once per instance), and it waits until the count
// reaches the end of that instance. Every CTA arrives, also one that has already given
// up, so later instances stay aligned; a CTA with ok == false does not wait. The wait is
// bounded by limit_ns. Returns ok && the wait completed.
// Grid barrier of the cooperative launch on a monotone 64-bit counter of the workspace.
// Every barrier adds exactly 2^20 to it whatever the grid size G: CTA c adds
// floor(2^20 (c+1) / G) - floor(2^20 c / G), so the counter is a multiple of 2^20 whenever no
// barrier is in progress, and a CTA waits (at most limit_ns, then CSA_ERR_TIMEOUT) for the
// next multiple above the value it found. Calls of any grid size can share the workspace.
__device__ bool grid_sync(unsigned long long* ctr, bool ok, uint64_t limit_ns,
                          int32_t* dev_status) {
  __shared__ int sh_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    constexpr unsigned long long kRound = 1ull << 20;
    const unsigned long long G = gridDim.x, c = blockIdx.x;
    const unsigned long long w = (kRound * (c + 1)) / G - (kRound * c) / G;
    unsigned long long old;
    asm volatile("atom.add.release.gpu.global.u64 %0, [%1], %2;" : "=l"(old) : "l"(ctr), "l"(w) : "memory");
    const unsigned long long target = ((old >> 20) + 1) << 20;
    if (ok) {
      const uint64_t t0 = globaltimer();
      while (true) {
        unsigned long long v;
        asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(ctr) : "memory");
        if (v >= target) break;
        if (globaltimer() - t0 > limit_ns) {
          report(dev_status, CSA_ERR_TIMEOUT);
          ok = false;
          break;
        }
      }
    }
    sh_ok = ok;
  }
  __syncthreads();
  return sh_ok != 0;
}

constexpr int kDxSlot = 32;  // in-bin candidates a CTA publishes in its slot

struct DxSel {
  uint64_t cand[kDxCand];             // the sequence's in-bin candidates (key << 32 | index)
  uint64_t dc[1024];                  // the candidates of the digit holding the cut
  uint16_t seg[kDxCand];              // the covering CTA each candidate came from
  uint32_t h[256];                    // digit histogram of the cut search
  uint32_t seg_off[kDxMaxCtas + 1];   // candidate offsets of the covering CTAs
  uint32_t nin[kDxMaxCtas];           // their in-bin counts
  uint32_t above[kDxMaxCtas];         // their above-bin counts
  uint32_t pass[kDxMaxCtas];          // their in-bin candidates that pass the cut
  uint32_t sub[kDxMaxCtas * 32];      // BF16 keys: their in-bin counts by the next 5 key bits
  uint32_t tmp[32];
  int32_t n[kIxMaxB];                 // eligible entries of the covered sequences
  int tbin;
  uint32_t cnt, above_total, off, prefix, rem, pop, spill;
  uint64_t v_cut;
};
static_assert(sizeof(DxSel) <= sizeof(uint8_t[kDxStages][kDxQuad][kIxKeyBytes]),
              "selection scratch fits the key ring");

// c_lo: the first CTA whose range ends after quad P; c_hi: the last CTA whose range starts
// before quad Q (CTA c covers quads [total*c/G, total*(c+1)/G)).
__device__ __forceinline__ int cta_ending_after(int64_t total, int G, int64_t P) {
  return (int)(((int64_t)G * (P + 1) + total - 1) / total) - 1;
}
__device__ __forceinline__ int cta_starting_before(int64_t total, int G, int64_t Q) {
  return (int)(((int64_t)G * Q + total - 1) / total) - 1;
}
__device__ __forceinline__ int64_t cta_q0(int64_t total, int c, int G) { return total * c / G; }

__device__ __forceinline__ uint64_t cand_value(uint32_t key, int j) {
  // larger value = earlier in the (score descending, index ascending) order
  return ((uint64_t)key << 32) | (uint32_t)(0xFFFFFFFFu - (uint32_t)j);
}

// The entries [ja, jb) of sequence b that a CTA with quads [q0, q1) owns (ja == jb: none).
struct SeqPart {
  int ja, jb, tiles;  // entry range, tiles it spans
  int t_lo;           // its first tile within the sequence
};
__device__ __forceinline__ SeqPart seq_part(const DxSmem& s, int b, int n, int q0, int q1) {
  SeqPart r;
  const int qa = max(q0, s.qprefix[b]) - s.qprefix[b];
  const int qb = min(q1, s.qprefix[b + 1]) - s.qprefix[b];
  r.t_lo = kDxQuad * qa;
  const int t_hi = min(kDxQuad * qb, s.tiles[b]);
  r.tiles = qa < qb ? t_hi - r.t_lo : 0;
  r.ja = r.t_lo * kIxTile;
  r.jb = r.tiles > 0 ? min(t_hi * kIxTile, n) : r.ja;
  return r;
}

// The selection inside the cooperative decode launch, after every CTA has added its
// histogram counts and holds its scores (in shared memory, or for long ranges in the
// workspace):
//  barrier 1;
//  B: for each sequence it covers (n > k), the CTA finds the threshold bin from the
//     sequence's histogram (the highest bin whose count from the top reaches k), counts
//     its own entries above that bin and publishes (above, in-bin count, bin) and its
//     in-bin entries in index order (the first kDxSlot in its slot, the rest in its own part
//     of the sequence's candidate array);
//  barrier 2;
//  C: every CTA of the sequence gathers all counts and candidates in one round trip and
//     resolves the same exact cut: a 256-bin histogram of the next 8 key bits finds the
//     digit holding it, and the candidates of that digit are ranked by (key, index) in
//     full. The CTA counts the earlier CTAs' passing candidates, so it knows its output
//     offset, and writes its selected entries in index order there. The first CTA of a
//     sequence clears the sequence's histogram for the next call.
// Each thread owns a contiguous run of the CTA's entries, so one block scan orders a pass.
// ok == false (a wait of this CTA gave up) skips the work but still arrives at both
// barriers. Sequences with n <= k select every entry in place.
__device__ void select_decode(const IxParams& p, uint8_t* scratch, const DxSmem& s, int q0,
                              int q1, bool on_chip, bool ok) {
  DxSel& x = *reinterpret_cast<DxSel*>(scratch);
  constexpr int NT = kDxThreads;
  const int tid = threadIdx.x, c = blockIdx.x, G = gridDim.x;
  const int64_t total = s.qprefix[p.B];
  int bf = 0;  // covered sequences: bf .. bl (some may own no tile of this CTA)
  while (bf < p.B && s.qprefix[bf + 1] <= q0) ++bf;
  int bl = bf - 1;
  if (q0 < q1) {
    bl = bf;
    while (bl + 1 < p.B && s.qprefix[bl + 1] < q1) ++bl;
  }
  for (int b = bf + tid; b <= bl; b += NT) x.n[b - bf] = clamp_n(p.n_entries[b], p.Nmax, nullptr);
  ok = grid_sync(reinterpret_cast<unsigned long long*>(p.ws.grid_bar), ok, p.wait_ns,
                 p.dev_status);
  // scores of sequence b by entry index (the CTA's own entries only)
  auto seq_scores = [&](int b, const SeqPart& r, int it_b0) -> const float* {
    return on_chip ? s.sc + (int64_t)(it_b0 - r.t_lo) * kIxTile
                   : p.ws.scores + (size_t)b * p.Nmax;
  };

  // ---- B: threshold bin, above-bin count and in-bin candidates per covered sequence
  for (int b = bf, it_b0 = 0; ok && b <= bl; ++b) {
    const int n = x.n[b - bf];
    const SeqPart r = seq_part(s, b, n, q0, q1);
    const int itb = it_b0;
    it_b0 += r.tiles;
    if (n <= p.k || r.tiles == 0) continue;
    {  // the threshold bin from the complete histogram: thread t holds the bins
       // 2047 - 4 kQ t down to 2048 - 4 kQ (t + 1), kQ = quads per thread
      constexpr int kQ = (kHist / 4 + NT - 1) / NT;
      uint32_t hb[4 * kQ];
#pragma unroll
      for (int q = 0; q < kQ; ++q) {
        const int hq = kHist / 4 - 1 - (tid * kQ + q);
        const uint4 hv = hq >= 0 ? __ldcg(reinterpret_cast<const uint4*>(p.ws.hist(b)) + hq)
                                 : make_uint4(0u, 0u, 0u, 0u);
        hb[4 * q] = hv.w; hb[4 * q + 1] = hv.z; hb[4 * q + 2] = hv.y; hb[4 * q + 3] = hv.x;
      }
      if (tid == 0) x.tbin = -1;
      uint32_t mine = 0;
#pragma unroll
      for (int i = 0; i < 4 * kQ; ++i) mine += hb[i];
      const uint32_t incl = block_incl_scan<NT>(mine, x.tmp, nullptr);
      if (incl >= (uint32_t)p.k && incl - mine < (uint32_t)p.k) {
        uint32_t cum = incl - mine;
        for (int i = 0; i < 4 * kQ; ++i) {
          if (cum + hb[i] >= (uint32_t)p.k) { x.tbin = kHist - 1 - 4 * kQ * tid - i; break; }
          cum += hb[i];
        }
      }
      __syncthreads();
    }
    const int tbin = x.tbin;
    const float* sc = seq_scores(b, r, itb);
    const int per = (r.jb - r.ja + NT - 1) / NT;
    const int j0 = min(r.jb, r.ja + tid * per), j1 = min(r.jb, j0 + per);
    uint32_t above = 0, in = 0;
    for (int j = j0; j < j1; ++j) {
      const int bin = (int)(float_key(sc[j]) >> kLowBits);
      above += bin > tbin ? 1u : 0u;
      in += bin == tbin ? 1u : 0u;
    }
    uint32_t nin_tot, above_tot;
    if (p.bf16) {
      // 16-bit keys: the bin's 11 bits and the next 5 are the whole key, so the counts of
      // the in-bin entries by those 5 bits (the CTA's slot, as 32 words) fix the cut
      for (int i = tid; i < 32; i += NT) x.h[i] = 0;
      __syncthreads();
      for (int j = j0; j < j1; ++j) {
        const uint32_t key = float_key(sc[j]);
        if ((int)(key >> kLowBits) == tbin) atomicAdd(&x.h[(key >> 16) & 31u], 1u);
      }
      block_incl_scan<NT>(in, x.tmp, &nin_tot);
      block_incl_scan<NT>(above, x.tmp, &above_tot);
      if (tid < 32)
        reinterpret_cast<uint32_t*>(p.ws.cand_slots + ((size_t)b * kDxMaxCtas + c) * kDxSlot)[tid] =
            x.h[tid];
      if (tid == 0)
        p.ws.cta_cnt[(size_t)b * kDxMaxCtas + c] =
            make_uint4(above_tot, nin_tot, (uint32_t)tbin, 0u);
      continue;
    }
    const uint32_t pos0 = block_incl_scan<NT>(in, x.tmp, &nin_tot) - in;
    block_incl_scan<NT>(above, x.tmp, &above_tot);
    if (in) {  // this thread's in-bin entries, in index order
      uint64_t* slot = p.ws.cand_slots + ((size_t)b * kDxMaxCtas + c) * kDxSlot;
      uint64_t* spill = p.ws.cand + (size_t)b * p.Nmax + r.ja;
      uint32_t pos = pos0;
      for (int j = j0; j < j1; ++j) {
        const uint32_t key = float_key(sc[j]);
        if ((int)(key >> kLowBits) != tbin) continue;
        const uint64_t cv = ((uint64_t)key << 32) | (uint32_t)j;
        if (pos < (uint32_t)kDxSlot) slot[pos] = cv; else spill[pos] = cv;
        ++pos;
      }
    }
    if (tid == 0)
      p.ws.cta_cnt[(size_t)b * kDxMaxCtas + c] = make_uint4(above_tot, nin_tot, (uint32_t)tbin, 0u);
  }
  ok = grid_sync(reinterpret_cast<unsigned long long*>(p.ws.grid_bar + 32), ok, p.wait_ns,
                 p.dev_status);
  if (!ok) return;

  // ---- C: the exact cut, this CTA's output offset, the ordered write
  for (int b = c; b < p.B; b += G)  // sequences with no entry at all: padding only
    if (s.qprefix[b + 1] == s.qprefix[b])
      for (int i = tid; i < p.k; i += NT) {
        p.idx[(size_t)b * p.k + i] = -1;
        if (p.scores_out) p.scores_out[(size_t)b * p.k + i] = __int_as_float(0x7fc00000);
      }
  for (int b = bf, it_b0 = 0; b <= bl; ++b) {
    const int n = x.n[b - bf];
    const SeqPart r = seq_part(s, b, n, q0, q1);
    const int itb = it_b0;
    it_b0 += r.tiles;
    if (r.tiles == 0) continue;
    const int k_eff = n < p.k ? n : p.k;
    const int c_lo = cta_ending_after(total, G, s.qprefix[b]);
    const int c_hi = cta_starting_before(total, G, s.qprefix[b + 1]);
    const float* sc = seq_scores(b, r, itb);
    int32_t* out = p.idx + (size_t)b * p.k;
    float* sout = p.scores_out ? p.scores_out + (size_t)b * p.k : nullptr;
    uint64_t v_cut = 0;  // n <= k: every entry (every value is >= 0), at its own index
    uint32_t base = (uint32_t)r.ja;
    // BF16 keys: entries above the cut value cut16 (the key's top 16 bits) and entries at
    // it with index <= cut_idx are selected (cut16 = -1: use v_cut)
    int cut16 = -1;
    int32_t cut_idx = -1;
    if (n > p.k && p.bf16) {
      const int nseg = c_hi - c_lo + 1;
      const int myseg = c - c_lo;
      uint32_t* sub = x.sub;  // [nseg][32]
      // one round trip: every covering CTA's counts and its 32 sub-bin counts
      for (int i = tid; i < nseg; i += NT) {
        const int cc = c_lo + i;
        const bool has = cta_q0(total, cc, G) < cta_q0(total, cc + 1, G);
        const uint4 v = has ? __ldcg(p.ws.cta_cnt + (size_t)b * kDxMaxCtas + cc)
                            : make_uint4(0u, 0u, 0u, 0u);
        x.above[i] = v.x;
        x.nin[i] = v.y;
        if (cc == c) x.tbin = (int)v.z;
      }
      for (int e = tid; e < nseg * 32; e += NT) {
        const int cc = c_lo + e / 32;
        const bool has = cta_q0(total, cc, G) < cta_q0(total, cc + 1, G);
        sub[e] = has ? __ldcg(reinterpret_cast<const uint32_t*>(
                                  p.ws.cand_slots + ((size_t)b * kDxMaxCtas + cc) * kDxSlot) +
                              (e & 31))
                     : 0u;
      }
      if (tid < 32) x.h[tid] = 0;
      __syncthreads();
      uint32_t above_total, nin_total;
      {
        const uint32_t av = tid < nseg ? x.above[tid] : 0u;
        const uint32_t nv = tid < nseg ? x.nin[tid] : 0u;
        block_incl_scan<NT>(av, x.tmp, &above_total);
        block_incl_scan<NT>(nv, x.tmp, &nin_total);
      }
      for (int e = tid; e < nseg * 32; e += NT)
        if (sub[e]) atomicAdd(&x.h[e & 31], sub[e]);
      __syncthreads();
      const int tbin = x.tbin;
      const int64_t need = (int64_t)k_eff - above_total;
      if (need <= 0) {  // nothing from the bin (as in the fp32 path)
        if (need < 0) report(p.dev_status, CSA_ERR_DEVICE);
        v_cut = cand_value((uint32_t)(tbin + 1) << kLowBits, -1);
      } else if (need >= (int64_t)nin_total) {  // the whole bin
        if (need > (int64_t)nin_total) report(p.dev_status, CSA_ERR_DEVICE);
        v_cut = cand_value((uint32_t)tbin << kLowBits, 0x7FFFFFFF);
      } else {
        if (tid == 0) {  // the sub-bin holding the need-th largest key, from the top
          uint32_t cum = 0;
          int sb = 31;
          for (; sb > 0 && cum + x.h[sb] < (uint32_t)need; --sb) cum += x.h[sb];
          x.off = (uint32_t)sb;
          x.rem = (uint32_t)need - cum;  // entries wanted at the cut value, from 1
        }
        __syncthreads();
        const uint32_t sb = x.off, need_in = x.rem;
        cut16 = (tbin << 5) | (int)sb;
        // per covering CTA: entries above the cut value, entries at it; the ties go to the
        // smallest indices, i.e. to the CTAs in order
        if (tid < 32) {
          uint32_t before_gt = 0, before_tie = 0, my_tie = 0;
          for (int i = tid; i < nseg; i += 32) {
            uint32_t gt = 0;
            for (int q = (int)sb + 1; q < 32; ++q) gt += sub[i * 32 + q];
            const uint32_t tie = sub[i * 32 + sb];
            if (i < myseg) { before_gt += x.above[i] + gt; before_tie += tie; }
            if (i == myseg) my_tie = tie;
          }
          for (int o = 16; o > 0; o >>= 1) {
            before_gt += __shfl_xor_sync(0xffffffffu, before_gt, o);
            before_tie += __shfl_xor_sync(0xffffffffu, before_tie, o);
            my_tie += __shfl_xor_sync(0xffffffffu, my_tie, o);
          }
          if (tid == 0) {
            const uint32_t take_before = before_tie < need_in ? before_tie : need_in;
            const uint32_t left = need_in - take_before;
            const uint32_t take = my_tie < left ? my_tie : left;
            x.off = before_gt + take_before;  // this CTA's output offset
            x.pop = take;
            x.cnt = my_tie;
          }
        }
        __syncthreads();
        base = x.off;
        const uint32_t take = x.pop, my_tie = x.cnt;
        if (take == 0) {
          cut_idx = -1;
        } else if (take == my_tie) {
          cut_idx = 0x7FFFFFFF;
        } else {  // the CTA where the cut falls: the index of its take-th entry at the cut
          const float* scb = seq_scores(b, r, itb);
          const int per = (r.jb - r.ja + NT - 1) / NT;
          const int j0 = min(r.jb, r.ja + tid * per), j1 = min(r.jb, j0 + per);
          uint32_t mt = 0;
          for (int j = j0; j < j1; ++j) mt += (int)(float_key(scb[j]) >> 16) == cut16 ? 1u : 0u;
          const uint32_t incl = block_incl_scan<NT>(mt, x.tmp, nullptr);
          if (incl >= take && incl - mt < take) {
            uint32_t cum = incl - mt;
            for (int j = j0; j < j1; ++j)
              if ((int)(float_key(scb[j]) >> 16) == cut16 && ++cum == take) { x.prefix = (uint32_t)j; break; }
          }
          __syncthreads();
          cut_idx = (int32_t)x.prefix;
        }
      }
    } else if (n > p.k) {
      const int nseg = c_hi - c_lo + 1;
      // one round trip: every covering CTA's counts and slot
      for (int i = tid; i < nseg; i += NT) {
        const int cc = c_lo + i;
        const bool has = cta_q0(total, cc, G) < cta_q0(total, cc + 1, G);
        const uint4 v = has ? __ldcg(p.ws.cta_cnt + (size_t)b * kDxMaxCtas + cc)
                            : make_uint4(0u, 0u, 0u, 0u);
        x.above[i] = v.x;
        x.nin[i] = v.y;
        x.pass[i] = 0;
        if (cc == c) x.tbin = (int)v.z;
      }
      constexpr int kSlotLoads = (kDxMaxCtas * kDxSlot + NT - 1) / NT;
      uint64_t sv[kSlotLoads];
#pragma unroll
      for (int u = 0; u < kSlotLoads; ++u) {
        const int e = tid + u * NT;
        sv[u] = e < nseg * kDxSlot
                    ? __ldcg(p.ws.cand_slots + ((size_t)b * kDxMaxCtas + c_lo) * kDxSlot + e)
                    : 0ull;
      }
      if (tid == 0) x.spill = 0;
      __syncthreads();
      {  // offsets of the candidates by covering CTA (nseg <= kDxMaxCtas < NT), totals
        const uint32_t vv = tid < nseg ? x.nin[tid] : 0u;
        const uint32_t av = tid < nseg ? x.above[tid] : 0u;
        if (vv > (uint32_t)kDxSlot) x.spill = 1;
        uint32_t tot, atot;
        const uint32_t incl = block_incl_scan<NT>(vv, x.tmp, &tot);
        if (tid < nseg) x.seg_off[tid + 1] = incl;
        if (tid == 0) x.seg_off[0] = 0;
        block_incl_scan<NT>(av, x.tmp, &atot);
        if (tid == 0) x.above_total = atot;
        __syncthreads();
      }
      const uint32_t ntot = x.seg_off[nseg], above_total = x.above_total;
      const int tbin = x.tbin;
      const int64_t need = (int64_t)k_eff - above_total;
      const bool staged = ntot <= (uint32_t)kDxCand;
      auto spill_src = [&](int sgi) {  // spill part of covering CTA c_lo + sgi
        const int64_t sq0 = cta_q0(total, c_lo + sgi, G);
        const int64_t ja_s = (sq0 > s.qprefix[b] ? sq0 - s.qprefix[b] : 0) * kDxQuad * kIxTile;
        return p.ws.cand + (size_t)b * p.Nmax + ja_s;
      };
      if (staged) {  // the candidate list: the slots (already in registers), then any spill
#pragma unroll
        for (int u = 0; u < kSlotLoads; ++u) {
          const int e = tid + u * NT;
          if (e < nseg * kDxSlot) {
            const int sgi = e / kDxSlot, i = e % kDxSlot;
            if ((uint32_t)i < x.nin[sgi]) {
              x.cand[x.seg_off[sgi] + i] = sv[u];
              x.seg[x.seg_off[sgi] + i] = (uint16_t)sgi;
            }
          }
        }
        if (x.spill) {
          for (int sgi = 0; sgi < nseg; ++sgi) {
            if (x.nin[sgi] <= (uint32_t)kDxSlot) continue;
            const uint64_t* src = spill_src(sgi);
            for (uint32_t i = kDxSlot + tid; i < x.nin[sgi]; i += NT) {
              x.cand[x.seg_off[sgi] + i] = __ldcg(src + i);
              x.seg[x.seg_off[sgi] + i] = (uint16_t)sgi;
            }
          }
        }
        __syncthreads();
      }
      // candidate i of the concatenation (from shared memory, or for a very large bin from
      // the slots and spill parts in global memory)
      auto seg_of = [&](uint32_t i) {
        int lo = 0, hi = nseg - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (x.seg_off[mid] <= i) lo = mid; else hi = mid - 1;
        }
        return lo;
      };
      auto get = [&](uint32_t i) -> uint64_t {
        if (staged) return x.cand[i];
        const int sgi = seg_of(i);
        const uint32_t ri = i - x.seg_off[sgi];
        return ri < (uint32_t)kDxSlot
                   ? __ldcg(p.ws.cand_slots + ((size_t)b * kDxMaxCtas + c_lo + sgi) * kDxSlot + ri)
                   : __ldcg(spill_src(sgi) + ri);
      };
      auto value_of = [&](uint64_t cv) { return cand_value((uint32_t)(cv >> 32), (int)(uint32_t)cv); };
      if (need <= 0) {  // the bin contributes nothing: the cut sits just above it (tbin is
                        // below the top bin here, as the top bin has nothing above it)
        if (need < 0) report(p.dev_status, CSA_ERR_DEVICE);
        v_cut = cand_value((uint32_t)(tbin + 1) << kLowBits, -1);
      } else if (need >= (int64_t)ntot) {  // the whole bin
        if (need > (int64_t)ntot) report(p.dev_status, CSA_ERR_DEVICE);
        v_cut = cand_value((uint32_t)tbin << kLowBits, 0x7FFFFFFF);
      } else {
        // the digit of key bits 13..20 that holds the need-th largest candidate
        for (int i = tid; i < 256; i += NT) x.h[i] = 0;
        if (tid == 0) x.cnt = 0;
        __syncthreads();
        for (uint32_t i = tid; i < ntot; i += NT)
          atomicAdd(&x.h[(uint32_t)(get(i) >> 32 >> (kLowBits - 8)) & 255u], 1u);
        __syncthreads();
        const uint32_t hd = tid < 256 ? x.h[255 - tid] : 0u;  // descending digits
        const uint32_t incl = block_incl_scan<NT>(hd, x.tmp, nullptr);
        if (tid < 256 && incl >= (uint32_t)need && incl - hd < (uint32_t)need) {
          x.tbin = 255 - tid;  // (reused) the digit
          x.off = (uint32_t)need - (incl - hd);  // rank wanted inside the digit, from 1
        }
        __syncthreads();
        const uint32_t digit = (uint32_t)x.tbin, want = x.off, m = x.h[digit];
        auto digit_of = [&](uint64_t cv) { return ((uint32_t)(cv >> 32) >> (kLowBits - 8)) & 255u; };
        if (staged && m <= 1024u) {
          // the digit's candidates, each ranked by one warp: the one with want - 1 larger
          // values in the digit is the cut (larger digits are all above it)
          for (uint32_t i = tid; i < ntot; i += NT) {
            const uint64_t cv = x.cand[i];
            if (digit_of(cv) == digit) x.dc[atomicAdd(&x.cnt, 1u)] = value_of(cv);
          }
          __syncthreads();
          const int warp = tid >> 5, lane = tid & 31;
          for (uint32_t i = warp; i < m; i += NT / 32) {
            const uint64_t v = x.dc[i];
            uint32_t rank = 0;
            for (uint32_t j2 = lane; j2 < m; j2 += 32) rank += x.dc[j2] > v ? 1u : 0u;
            for (int o = 16; o > 0; o >>= 1) rank += __shfl_xor_sync(0xffffffffu, rank, o);
            if (lane == 0 && rank == want - 1) x.v_cut = v;
          }
          __syncthreads();
          v_cut = x.v_cut;
        } else {
          // many candidates in one digit (heavy ties): radix select on the remaining 13
          // key bits, then the smallest indices among equal keys
          if (tid == 0) {
            x.prefix = ((uint32_t)tbin << kLowBits) | (digit << (kLowBits - 8));
            x.rem = want;
          }
          __syncthreads();
          radix_step_g<NT>(get, ntot, true, 0, false, ~0u << (kLowBits - 8), 5, 8, true,
                           &x.prefix, &x.rem, x.h);
          radix_step_g<NT>(get, ntot, true, 0, false, ~0u << 5, 0, 5, true, &x.prefix, &x.rem,
                           x.h, &x.pop);
          const uint32_t cut_key = x.prefix;
          int32_t cut_idx = 0x7FFFFFFF;
          if (x.pop != x.rem) {
            __syncthreads();
            if (tid == 0) x.prefix = 0;
            __syncthreads();
            radix_step_g<NT>(get, ntot, false, cut_key, true, 0u, 24, 8, false, &x.prefix,
                             &x.rem, x.h);
            radix_step_g<NT>(get, ntot, false, cut_key, true, 0xFF000000u, 16, 8, false,
                             &x.prefix, &x.rem, x.h);
            radix_step_g<NT>(get, ntot, false, cut_key, true, 0xFFFF0000u, 8, 8, false,
                             &x.prefix, &x.rem, x.h);
            radix_step_g<NT>(get, ntot, false, cut_key, true, 0xFFFFFF00u, 0, 8, false,
                             &x.prefix, &x.rem, x.h);
            cut_idx = (int32_t)x.prefix;
          }
          v_cut = cand_value(cut_key, cut_idx);
        }
      }
      // output offset: above-bin entries and passing candidates of the earlier CTAs
      const int myseg = c - c_lo;
      for (uint32_t i = tid; i < x.seg_off[myseg]; i += NT)
        if (value_of(get(i)) >= v_cut) atomicAdd(&x.pass[staged ? x.seg[i] : seg_of(i)], 1u);
      __syncthreads();
      if (tid < 32) {
        uint32_t off = 0;
        for (int i = tid; i < myseg; i += 32) off += x.above[i] + x.pass[i];
        for (int o = 16; o > 0; o >>= 1) off += __shfl_xor_sync(0xffffffffu, off, o);
        if (tid == 0) x.off = off;
      }
      __syncthreads();
      base = x.off;
    }
    {  // ordered write of this CTA's selected entries: each thread its contiguous run
      auto selected = [&](float v, int j) {
        if (cut16 < 0) return cand_value(float_key(v), j) >= v_cut;
        const int k16 = (int)(float_key(v) >> 16);
        return k16 > cut16 || (k16 == cut16 && j <= cut_idx);
      };
      const int per = (r.jb - r.ja + NT - 1) / NT;
      const int j0 = min(r.jb, r.ja + tid * per), j1 = min(r.jb, j0 + per);
      uint32_t mine = 0;
      for (int j = j0; j < j1; ++j) mine += selected(sc[j], j) ? 1u : 0u;
      uint32_t tot;
      uint32_t pos = base + block_incl_scan<NT>(mine, x.tmp, &tot) - mine;
      if (mine) {
        for (int j = j0; j < j1; ++j) {
          const float v = sc[j];
          if (!selected(v, j)) continue;
          if (pos < (uint32_t)p.k) {
            out[pos] = j;
            if (sout) sout[pos] = v;
          } else {
            report(p.dev_status, CSA_ERR_DEVICE);
          }
          ++pos;
        }
      }
      base += tot;
    }
    if (c == c_hi) {  // the last CTA of the sequence: its end is the selection's end
      if (base != (uint32_t)k_eff && tid == 0) report(p.dev_status, CSA_ERR_DEVICE);
      for (int i = k_eff + tid; i < p.k; i += NT) {
        out[i] = -1;
        if (sout) sout[i] = __int_as_float(0x7fc00000);
      }
    }
    if (c == c_lo)  // every CTA read this histogram before barrier 2
      for (int i = tid; i < kHist; i += NT) p.ws.hist(b)[i] = 0;
    __syncthreads();
  }
}

// Stand-alone selection kernels (when a cooperative launch is not available): one CTA per
// (slice, sequence).
__global__ void __launch_bounds__(kSelThreads) topk_threshold_kernel(IxParams p) {
  __shared__ __align__(16) uint8_t raw[sizeof(SelScratch)];
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.y, sb = blockIdx.x;
  int n = p.n_entries[b];
  n = n < 0 ? 0 : (n > p.Nmax ? (int)p.Nmax : n);
  if (sb < slices_of(n)) select_threshold(p, *reinterpret_cast<SelScratch*>(raw), b, sb);
}

__global__ void __launch_bounds__(kSelThreads) topk_write_kernel(IxParams p) {
  __shared__ __align__(16) uint8_t raw[sizeof(SelScratch)];
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.y, sb = blockIdx.x;
  int n = p.n_entries[b];
  n = n < 0 ? 0 : (n > p.Nmax ? (int)p.Nmax : n);
  if (sb < slices_of(n)) select_write(p, *reinterpret_cast<SelScratch*>(raw), b, sb);
}

// ------------------------------------------------------------- prefill scoring
// In a prefill every query of the call scores the same key array (one sequence), so the
// key stream is shared: a 128-entry key tile is loaded once for a group of kPxQ
// consecutive queries and meets their kPxQ x 64 heads in kPxQ block-scaled MMAs
// (D[128 entries x 64 heads] each, 2 x K = 64), instead of once per query. The roles are
// those of the decode kernel with one pipeline per CTA: a TMA producer warp, a tcgen05
// issuer warp that also stages each group's queries and scales, and eight epilogue warps
// in two groups of four taking alternate tiles (accumulator buffer = tile parity). An
// epilogue thread owns one entry and forms its kPxQ scores, masked by each query's own
// eligible count, and counts them into per-warp, per-query histograms. The selection then
// runs as topk_query_kernel, one CTA per query.
constexpr int kPxQ = 3;                     // queries per group
constexpr int kPxStages = 6;
constexpr int kPxNbuf = 2;                  // accumulator buffers (one per epilogue group)
constexpr int kPxEpiWarps = 8;
constexpr int kPxThreads = 32 * (2 + kPxEpiWarps);
constexpr int kPxGroupCols = kPxQ * kIxN;   // TMEM columns of one buffer
constexpr int kPxTmemCols = 512;
constexpr int kPxMaxG = (kIxMaxB + kPxQ - 1) / kPxQ;
static_assert(kPxNbuf * kPxGroupCols + 8 + 8 * kPxQ <= kPxTmemCols, "TMEM budget");

struct alignas(1024) PxSmem {
  uint8_t keys[kPxStages][kIxKeyBytes];
  uint8_t q[2][kPxQ][kIxN * 64];
  uint32_t hist[kPxEpiWarps][kPxQ][kHist / 2];
  uint8_t ksf[kPxStages][kIxSfBytes];
  uint8_t qsf[2][kPxQ][512];
  float w[kPxEpiWarps][kPxQ][kIxN];
  int32_t prefix[kPxMaxG + 1];
  uint64_t full[kPxStages], empty[kPxStages];
  uint64_t acc_full[kPxNbuf], acc_empty[kPxNbuf], q_free[2], done;
  uint32_t tmem_base;
  volatile int abort;
};

__global__ void __launch_bounds__(kPxThreads, 1)
    prefill_score_kernel(const __grid_constant__ CUtensorMap kmap, IxParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  PxSmem& s = *reinterpret_cast<PxSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = (p.B + kPxQ - 1) / kPxQ;
  if (warp == 1 && lane == 0) {
    for (int i = 0; i < kPxStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < kPxNbuf; ++i) {
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
    uint32_t* hz = &s.hist[0][0][0];
    for (int i = threadIdx.x; i < kPxEpiWarps * kPxQ * kHist / 2; i += kPxThreads) hz[i] = 0;
  }
  if (warp == 1) tmem_alloc(&s.tmem_base, kPxTmemCols);
  pdl_wait();
  pdl_trigger();
  // group g holds queries kPxQ*g .. kPxQ*g + kPxQ - 1 and ceil(max n / 128) key tiles
  if (warp == 0) {
    int carry = 0;
    if (lane == 0) s.prefix[0] = 0;
    for (int base = 0; base < G; base += 32) {
      const int g = base + lane;
      int v = 0;
      if (g < G) {
        int nmax = 0;
        for (int qq = 0; qq < kPxQ; ++qq) {
          const int qi = kPxQ * g + qq;
          if (qi < p.B) nmax = max(nmax, clamp_n(p.n_entries[qi], p.Nmax, p.dev_status));
        }
        v = (nmax + kIxTile - 1) / kIxTile;
      }
      int incl = v;
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (g < G) s.prefix[g + 1] = carry + incl;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int total = s.prefix[G];
  const int g0 = (int)((int64_t)total * blockIdx.x / gridDim.x);
  const int g1 = (int)((int64_t)total * (blockIdx.x + 1) / gridDim.x);
  const uint32_t tmem = s.tmem_base;
  const uint32_t t_sfa = tmem + kPxNbuf * kPxGroupCols;
  int gr0 = 0;  // first group of this CTA
  if (g0 < g1)
    while (s.prefix[gr0 + 1] <= g0) ++gr0;

  if (g0 < g1 && warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int gr = gr0, it = 0;
      for (int g = g0; g < g1; ++g, ++it) {
        while (s.prefix[gr + 1] <= g) ++gr;
        const int t = g - s.prefix[gr];
        const int st = it % kPxStages;
        if (s.abort || !mbar_wait(&s.empty[st], ((it / kPxStages) & 1) ^ 1, p.dev_status)) {
          s.abort = 1;
          break;
        }
        mbar_arrive_expect_tx(&s.full[st], kIxKeyBytes + kIxSfBytes);
        tma_load_3d(s.keys[st], &kmap, &s.full[st], 0, t * kIxTile, 0);
        bulk_load(s.ksf[st], p.k_sf + (size_t)t * kIxSfBytes, kIxSfBytes, &s.full[st]);
      }
      const int issued = it;
      for (int i = issued - kPxStages < 0 ? 0 : issued - kPxStages; i < issued; ++i)
        mbar_wait(&s.full[i % kPxStages], (i / kPxStages) & 1, p.dev_status);
    }
  } else if (g0 < g1 && warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    int gr = -1, ngr = -1, it = 0;
    uint32_t qslot = 0;
    for (int g = g0; g < g1; ++g, ++it) {
      int nb = gr < 0 ? gr0 : gr;
      while (s.prefix[nb + 1] <= g) ++nb;
      if (nb != gr) {  // stage the group's queries (B operands) and their scales
        if (gr >= 0 && lane == 0) mma_commit(&s.q_free[qslot]);
        gr = nb;
        ++ngr;
        qslot = ngr & 1;
        bool ok = true;
        if (lane == 0)
          ok = !s.abort && mbar_wait(&s.q_free[qslot], ((ngr >> 1) & 1) ^ 1, p.dev_status);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) { s.abort = 1; break; }
        for (int qq = 0; qq < kPxQ; ++qq) {
          const int qi = kPxQ * gr + qq;
          const bool has = qi < p.B;
          const uint8_t* qsrc = p.q_fp4 + (size_t)(has ? qi : 0) * p.H_I * 64;
          for (int c = lane; c < kIxN * 4; c += 32) {  // 16-byte chunks, 64-byte swizzle
            const int r = c >> 2, ch = c & 3;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (has && r < p.H_I) v = *reinterpret_cast<const uint4*>(qsrc + r * 64 + ch * 16);
            *reinterpret_cast<uint4*>(&s.q[qslot][qq][r * 64 + ((ch ^ ((r >> 1) & 3)) << 4)]) = v;
          }
          uint32_t wv[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int n = lane + 32 * j;
            wv[j] = (has && n < p.H_I)
                        ? *reinterpret_cast<const uint32_t*>(p.q_sf + ((size_t)qi * p.H_I + n) * 4)
                        : 0x7F7F7F7Fu;
          }
          *reinterpret_cast<uint4*>(&s.qsf[qslot][qq][lane * 16]) =
              make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tc_fence_after();
          for (int qq = 0; qq < kPxQ; ++qq)
            tmem_cp_32x128b_x4(t_sfa + 8 + 8 * qq,
                               smem_desc(smem_u32(s.qsf[qslot][qq]), 0, 128, kSwizzleNone));
        }
      }
      if (lane == 0) {
        const int st = it % kPxStages, bb = it % kPxNbuf;
        bool ok = !s.abort;
        if (ok) {
          ok = mbar_wait(&s.acc_empty[bb], ((it / kPxNbuf) & 1) ^ 1, p.dev_status);
          tc_fence_after();
        }
        ok = ok && mbar_wait(&s.full[st], (it / kPxStages) & 1, p.dev_status);
        if (!ok) {
          s.abort = 1;
        } else {
          tmem_cp_32x128b_x4(t_sfa, smem_desc(smem_u32(s.ksf[st]), 0, 128, kSwizzleNone));
          const uint32_t ka = smem_u32(s.keys[st]);
          for (int qq = 0; qq < kPxQ; ++qq) {
            const uint32_t qa = smem_u32(s.q[qslot][qq]);
#pragma unroll
            for (int kh = 0; kh < 2; ++kh)
              mma_mxf4(tmem + bb * kPxGroupCols + qq * kIxN,
                       smem_desc(ka + 32 * kh, 16, 512, kSwizzle64B),
                       smem_desc(qa + 32 * kh, 16, 512, kSwizzle64B),
                       idesc_mxf4(kIxTile, kIxN, 2 * kh), t_sfa, t_sfa + 8 + 8 * qq, kh);
          }
          mma_commit(&s.empty[st]);
          mma_commit(&s.acc_full[bb]);
        }
      }
      if (__shfl_sync(0xffffffffu, s.abort, 0)) break;
    }
    if (lane == 0) {
      mma_commit(&s.done);
      mbar_wait(&s.done, 0, p.dev_status);
    }
    __syncwarp();
  } else if (g0 < g1) {
    // ---------------------------------------------------------------- epilogue
    const int ew = warp - 2, grp = ew >> 2, quad = warp & 3, row = quad * 32 + lane;
    const int ntiles = g1 - g0;
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    float* wq = &s.w[ew][0][0];
    int gr = -1, since_flush = 0, gseq = gr0;
    int nq[kPxQ];
    auto flush = [&](int gg) {
      __syncwarp();
      for (int qq = 0; qq < kPxQ; ++qq) {
        const int qi = kPxQ * gg + qq;
        uint32_t* hist = s.hist[ew][qq];
        uint32_t* gh = qi < p.B ? p.ws.hist(qi) : nullptr;
        for (int i = lane; i < kHist / 2; i += 32) {
          const uint32_t v = hist[i];
          if (v) {
            if (gh) {
              if (v & 0xFFFFu) atomicAdd(gh + 2 * i, v & 0xFFFFu);
              if (v >> 16) atomicAdd(gh + 2 * i + 1, v >> 16);
            }
            hist[i] = 0;
          }
        }
      }
      __syncwarp();
    };
    for (int it = grp; it < ntiles; it += kPxNbuf) {
      const int bb = it % kPxNbuf;
      bool ok = true;
      if (lane == 0)
        ok = !s.abort && mbar_wait(&s.acc_full[bb], (it / kPxNbuf) & 1, p.dev_status);
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        s.abort = 1;
        break;
      }
      tc_fence_after();
      const int g = g0 + it;
      while (s.prefix[gseq + 1] <= g) ++gseq;
      if (gseq != gr || since_flush >= 2000) {
        if (gr >= 0) flush(gr);
        since_flush = 0;
        gr = gseq;
        for (int qq = 0; qq < kPxQ; ++qq) {
          const int qi = kPxQ * gr + qq;
          nq[qq] = qi < p.B ? clamp_n(p.n_entries[qi], p.Nmax, nullptr) : 0;
          for (int h = lane; h < kIxN; h += 32)
            wq[qq * kIxN + h] = (qi < p.B && h < p.H_I) ? __ldg(p.w + (size_t)qi * p.H_I + h) : 0.f;
        }
        __syncwarp();
      }
      ++since_flush;
      const int j = (g - s.prefix[gr]) * kIxTile + row;
      for (int qq = 0; qq < kPxQ; ++qq) {
        uint32_t r[2][32];
        const uint32_t ta = lane_base + bb * kPxGroupCols + qq * kIxN;
        tmem_ld32(ta, r[0]);
        tmem_ld32(ta + 32, r[1]);
        tmem_ld_wait();
        const float4* w4 = reinterpret_cast<const float4*>(wq + qq * kIxN);
        float part[8];
#pragma unroll
        for (int k8 = 0; k8 < 8; ++k8) part[k8] = 0.f;
#pragma unroll
        for (int h4 = 0; h4 < kIxN / 4; ++h4) {
          const float4 wv = w4[h4];
          const int h = 4 * h4;
          fma2(part[h & 7], part[(h + 1) & 7], wv.x, wv.y,
               fmaxf(__uint_as_float(r[h >> 5][h & 31]), 0.f),
               fmaxf(__uint_as_float(r[(h + 1) >> 5][(h + 1) & 31]), 0.f));
          fma2(part[(h + 2) & 7], part[(h + 3) & 7], wv.z, wv.w,
               fmaxf(__uint_as_float(r[(h + 2) >> 5][(h + 2) & 31]), 0.f),
               fmaxf(__uint_as_float(r[(h + 3) >> 5][(h + 3) & 31]), 0.f));
        }
        const float sc = ((part[0] + part[1]) + (part[2] + part[3])) +
                         ((part[4] + part[5]) + (part[6] + part[7]));
        if (j < nq[qq]) {
          const int qi = kPxQ * gr + qq;
          p.ws.scores[(size_t)qi * p.Nmax + j] = sc;
          const uint32_t bin = float_key(sc) >> kLowBits;
          atomicAdd(&s.hist[ew][qq][bin >> 1], 1u << (16 * (bin & 1)));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.acc_empty[bb]);
    }
    if (gr >= 0) flush(gr);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kPxTmemCols);
  }
}

// One CTA per query: the whole selection of a query whose eligible count is small enough
// for one CTA to scan (the queries of a prefill). The histogram gives the threshold bin;
// pass 1 reads the scores in 1536-entry tiles (one float4 per thread), counts the entries
// above the bin and collects the in-bin candidates in shared memory; the radix select of
// the decode path fixes the exact cut; pass 2 reads the tiles again in index order and
// writes the selected indices at offsets from a block scan, so the output is ascending.
// It leaves the query's histogram zeroed.
constexpr int kQsTile = kSelThreads * 4;

__global__ void __launch_bounds__(kSelThreads) topk_query_kernel(IxParams p) {
  __shared__ __align__(16) uint8_t raw[sizeof(SelScratch)];
  SelScratch& x = *reinterpret_cast<SelScratch*>(raw);
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x, tid = threadIdx.x;
  const int n = clamp_n(p.n_entries[b], p.Nmax, p.dev_status);
  const int k_eff = n < p.k ? n : p.k;
  const float* sc = p.ws.scores + (size_t)b * p.Nmax;
  uint32_t* gh = p.ws.hist(b);
  if (tid == 0) { x.tbin = -1; x.above = 0; x.pop = 0; }
  if (n > p.k) {
    for (int i = tid; i < kHist; i += kSelThreads) x.h[i] = __ldcg(gh + i);
    __syncthreads();
    constexpr int per = (kHist + kSelThreads - 1) / kSelThreads;
    uint32_t mine = 0;
    for (int i = 0; i < per; ++i) {
      const int r = tid * per + i;
      if (r < kHist) mine += x.h[kHist - 1 - r];
    }
    const uint32_t incl = block_incl_scan(mine, x.tmp, nullptr);
    if (incl >= (uint32_t)p.k && incl - mine < (uint32_t)p.k) {
      uint32_t cum = incl - mine;
      for (int i = 0; i < per; ++i) {
        const int r = tid * per + i;
        if (r >= kHist) break;
        const int bin = kHist - 1 - r;
        if (cum + x.h[bin] >= (uint32_t)p.k) { x.tbin = bin; break; }
        cum += x.h[bin];
      }
    }
  }
  __syncthreads();
  const int tbin = x.tbin;
  uint32_t cut_key = 0u;
  int32_t cut_idx = 0x7FFFFFFF;  // tbin < 0: every eligible entry is selected
  if (tbin >= 0) {
    // pass 1: count above the bin, collect the bin's candidates (x.pop counts them; past
    // the shared capacity they go to the global candidate list)
    uint64_t* gcand = p.ws.cand + (size_t)b * p.Nmax;
    uint32_t above = 0;
    for (int j0 = 0; j0 < n; j0 += kQsTile) {
      const int j = j0 + 4 * tid;
      float v[4] = {0.f, 0.f, 0.f, 0.f};
      if (j + 4 <= n) {
        const float4 f = __ldcg(reinterpret_cast<const float4*>(sc + j));
        v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
      } else {
        for (int e = 0; e < 4; ++e) v[e] = j + e < n ? __ldcg(sc + j + e) : 0.f;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (j + e >= n) continue;
        const uint32_t key = float_key(v[e]);
        const int bin = (int)(key >> kLowBits);
        above += bin > tbin ? 1u : 0u;
        if (bin == tbin) {
          const uint32_t slot = atomicAdd(&x.pop, 1u);
          const uint64_t c = ((uint64_t)key << 32) | (uint32_t)(j + e);
          if (slot < kCandStage) x.cand[slot] = c;
          if (slot < (uint32_t)p.Nmax) gcand[slot] = c;  // complete list for overflow
        }
      }
    }
    for (int o = 16; o > 0; o >>= 1) above += __shfl_xor_sync(0xffffffffu, above, o);
    if ((tid & 31) == 0 && above) atomicAdd(&x.above, above);
    __syncthreads();
    const uint32_t above_total = x.above;
    uint32_t n_cand = x.pop;
    if (n_cand > (uint32_t)p.Nmax) n_cand = (uint32_t)p.Nmax;
    const bool staged = n_cand <= kCandStage;
    const uint64_t* cand = staged ? x.cand : gcand;
    if (!staged) __threadfence_block();
    const uint32_t need = (uint32_t)k_eff > above_total ? (uint32_t)k_eff - above_total : 0u;
    if (need == 0) {
      cut_key = ((uint32_t)(tbin + 1) << kLowBits) - 1u;
      cut_idx = -1;
    } else if (need >= n_cand) {
      if (need > n_cand) report(p.dev_status, CSA_ERR_DEVICE);
      cut_key = (uint32_t)tbin << kLowBits;
      cut_idx = 0x7FFFFFFF;
    } else {
      __syncthreads();
      if (tid == 0) { x.prefix = (uint32_t)tbin << kLowBits; x.rem = need; }
      __syncthreads();
      radix_step(cand, staged, n_cand, true, 0, false, ~0u << kLowBits, kLowBits - 8, 8, true,
                 &x.prefix, &x.rem, x.h);
      radix_step(cand, staged, n_cand, true, 0, false, ~0u << (kLowBits - 8), kLowBits - 16, 8,
                 true, &x.prefix, &x.rem, x.h);
      radix_step(cand, staged, n_cand, true, 0, false, ~0u << (kLowBits - 16), 0, kLowBits - 16,
                 true, &x.prefix, &x.rem, x.h, &x.sum);
      cut_key = x.prefix;
      if (x.sum == x.rem) {
        cut_idx = 0x7FFFFFFF;
      } else {
        __syncthreads();
        if (tid == 0) x.prefix = 0;
        __syncthreads();
        radix_step(cand, staged, n_cand, false, cut_key, true, 0u, 24, 8, false, &x.prefix,
                   &x.rem, x.h);
        radix_step(cand, staged, n_cand, false, cut_key, true, 0xFF000000u, 16, 8, false,
                   &x.prefix, &x.rem, x.h);
        radix_step(cand, staged, n_cand, false, cut_key, true, 0xFFFF0000u, 8, 8, false,
                   &x.prefix, &x.rem, x.h);
        radix_step(cand, staged, n_cand, false, cut_key, true, 0xFFFFFF00u, 0, 8, false,
                   &x.prefix, &x.rem, x.h);
        cut_idx = (int32_t)x.prefix;
      }
    }
  }
  // pass 2: ordered write
  int32_t* out = p.idx + (size_t)b * p.k;
  uint32_t base = 0;
  for (int j0 = 0; j0 < n; j0 += kQsTile) {
    const int j = j0 + 4 * tid;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (j + 4 <= n) {
      const float4 f = __ldcg(reinterpret_cast<const float4*>(sc + j));
      v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
    } else {
      for (int e = 0; e < 4; ++e) v[e] = j + e < n ? __ldcg(sc + j + e) : 0.f;
    }
    uint32_t mask = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t key = float_key(v[e]);
      if (j + e < n && (key > cut_key || (key == cut_key && j + e <= cut_idx))) mask |= 1u << e;
    }
    const uint32_t mine = __popc(mask);
    uint32_t tot;
    const uint32_t incl = block_incl_scan(mine, x.tmp, &tot);
    uint32_t slot = base + incl - mine;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (mask & (1u << e)) {
        if (slot < (uint32_t)p.k) {
          out[slot] = j + e;
          if (p.scores_out) p.scores_out[(size_t)b * p.k + slot] = v[e];
        } else {
          report(p.dev_status, CSA_ERR_DEVICE);
        }
        ++slot;
      }
    }
    base += tot;
    __syncthreads();  // x.tmp is reused by the next tile's scan
  }
  if (base != (uint32_t)k_eff && tid == 0) report(p.dev_status, CSA_ERR_DEVICE);
  for (int i = k_eff + tid; i < p.k; i += kSelThreads) {
    out[i] = -1;
    if (p.scores_out) p.scores_out[(size_t)b * p.k + i] = __int_as_float(0x7fc00000);
  }
  for (int i = tid; i < kHist; i += kSelThreads) gh[i] = 0;
}

// ------------------------------------------------------------------- launch
cudaError_t launch_indexer_topk(const csa_topk_args& a, void* workspace, int num_sms,
                                const CUtensorMap& kmap, cudaStream_t stream, int bf16) {
  IxWs ws;
  ix_ws_layout(a.B, a.Nmax, a.k, (char*)workspace, &ws);
  const uint64_t wait_ns = a.select_wait_ns > 0 ? (uint64_t)a.select_wait_ns : kWaitLimitNs;
  IxParams p{a.B, a.H_I, a.k, 1, bf16, wait_ns, a.Nmax, a.n_entries, a.q_fp4, a.q_sf, a.w,
             a.k_sf, ws, a.idx, a.scores, a.dev_status, PageMap{}, kDxQuad};
  p.pm = page_map(a.pages, a.Nmax);
  p.tpl = a.pages.block_table ? (a.pages.page_entries / kIxTile < kDxQuad
                                     ? a.pages.page_entries / kIxTile : kDxQuad)
                              : kDxQuad;
  const size_t smem = sizeof(DxSmem) + 1024;
  static std::atomic<uint64_t> configured{0};
  if (cudaError_t e = configure_smem_once(indexer_decode_kernel, smem, configured, 100);
      e != cudaSuccess)
    return e;
  // no more CTAs than the largest number of key quads the call can have (a short context
  // then pays its grid barriers across a few CTAs, not across every SM)
  const int64_t quads_max = (int64_t)a.B * ((a.Nmax + kDxQuad * kIxTile - 1) / (kDxQuad * kIxTile));
  int grid_max = num_sms < kDxMaxCtas ? num_sms : kDxMaxCtas;
  if (quads_max < grid_max) grid_max = quads_max > 0 ? (int)quads_max : 1;
  cudaError_t e = cudaSuccess;
  if (!(a.flags & CSA_TOPK_SEPARATE_SELECT)) {
    // Scoring and selection in one cooperative launch (every CTA resident, so the grid
    // barriers between the phases always complete); the runtime refuses a grid that
    // cannot be resident, and the selection then runs as two further kernels.
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kDxThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cfg.gridDim = dim3(grid_max);
    e = cudaLaunchKernelEx(&cfg, indexer_decode_kernel, kmap, p);
    if (e == cudaSuccess) return cudaSuccess;
    (void)cudaGetLastError();
  }
  p.fused = 0;
  const int64_t tiles_max = (int64_t)a.B * (a.Nmax / kIxTile);
  int grid = grid_max;
  if (tiles_max < grid) grid = (int)(tiles_max > 0 ? tiles_max : 1);
  e = launch_pdl(indexer_decode_kernel, dim3(grid), dim3(kDxThreads), smem, stream, kmap, p);
  if (e != cudaSuccess) return e;
  dim3 g2((unsigned)ws.S, a.B);
  e = launch_pdl(topk_threshold_kernel, g2, dim3(kSelThreads), 0, stream, p);
  if (e != cudaSuccess) return e;
  return launch_pdl(topk_write_kernel, g2, dim3(kSelThreads), 0, stream, p);
}

// Indexer top-k of the queries of one prefill (all scoring the same keys): the shared-key
// scoring kernel, then the two selection kernels.
cudaError_t launch_prefill_indexer_topk(const csa_topk_args& a, void* workspace, int num_sms,
                                        const CUtensorMap& kmap, cudaStream_t stream) {
  IxWs ws;
  ix_ws_layout(a.B, a.Nmax, a.k, (char*)workspace, &ws);
  IxParams p{a.B, a.H_I, a.k, 0, 0, kWaitLimitNs, a.Nmax, a.n_entries, a.q_fp4, a.q_sf, a.w,
             a.k_sf, ws, a.idx, a.scores, a.dev_status, PageMap{}, kDxQuad};  // keys contiguous
  const size_t smem = sizeof(PxSmem) + 1024;
  static std::atomic<uint64_t> configured{0};
  if (cudaError_t e = configure_smem_once(prefill_score_kernel, smem, configured);
      e != cudaSuccess)
    return e;
  cudaError_t e = launch_pdl(prefill_score_kernel, dim3(num_sms), dim3(kPxThreads), smem,
                             stream, kmap, p);
  if (e != cudaSuccess) return e;
  return launch_pdl(topk_query_kernel, dim3(a.B), dim3(kSelThreads), 0, stream, p);
}

}  // namespace csa
