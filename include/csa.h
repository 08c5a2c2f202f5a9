/* C ABI of the B200 (sm_100a) CSA/HCA compressed attention layer.
 *
 * The layer is the hybrid compressed attention of the DeepSeek-V4 pages:
 *   CSA (Compressed Sparse Attention): KV compressed by m = 4 with overlapping
 *       gated-softmax merges, lightning-indexer scoring of the compressed entries in FP4,
 *       top-k selection, shared-KV MQA over the selected entries;
 *   HCA (Heavily Compressed Attention): KV compressed by m' = 128 without overlap, dense
 *       MQA over every compressed entry;
 *   both with a 128-token uncompressed sliding window and a per-head sink logit in the
 *   same softmax, head_dim 512 with RoPE on the last 64 dims, and an entry stored as 448
 *   FP8-E4M3 dims (with one fp32 scale per entry) plus 64 BF16 dims.
 * Sources: cyqw.cn/news/842812 DeepSeek-V4 walkthrough §2.2 (CSA/HCA, overlap, indexer,
 * top-k, window, sink), §2.3 (RMSNorm on KV entries), §3.4 (FP4 indexer QK path), §3.5
 * (state cache); chooseai.net/news/3476 §一 (m = 4 / 128, softmax merge with positional
 * bias, FP8 + BF16 split, top-k 512/1024); "DeepSeek V4技术报告详解" §2 (head_dim 512,
 * partial RoPE on the last 64 dims, sink logit); "DeepSeek-V4：百万上下文的工程答案",
 * Hybrid Attention / Partial RoPE / Attention sink (shared-KV MQA, output de-rotation).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers, caller-owned, 16-byte aligned, dense
 *    row-major in the shapes given. The library never allocates, frees or synchronises.
 *    Scratch memory comes from a caller workspace of at least the size reported by the
 *    matching *_workspace_size function, 256-byte aligned.
 *  - Work is enqueued on `stream` (a cudaStream_t; 0 = legacy default stream).
 *  - Arguments are checked on the host before any launch. On a bad argument the call
 *    returns CSA_ERR_INVALID_ARG / CSA_ERR_UNSUPPORTED / CSA_ERR_WORKSPACE and launches
 *    nothing. A failed launch returns CSA_ERR_CUDA.
 *  - Data-dependent problems found by a kernel (an index outside the eligible range, a
 *    length beyond the capacity) are written to the optional device word *dev_status
 *    (first error wins, CSA_ERR_DEVICE); the affected rows are skipped. Read it after
 *    synchronising the stream.
 *  - Results are deterministic and batch-invariant: a sequence gives the same bits
 *    whatever the batch around it.
 */
#ifndef CSA_B200_H
#define CSA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* csa_stream_t; /* the same type as cudaStream_t */

enum {
  CSA_OK = 0,
  CSA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or flag */
  CSA_ERR_UNSUPPORTED = 2, /* valid but not built (e.g. a head count outside the list) */
  CSA_ERR_WORKSPACE = 3,   /* workspace missing, misaligned or too small */
  CSA_ERR_CUDA = 4,        /* a CUDA launch or driver call failed */
  CSA_ERR_DEVICE = 5,      /* written to dev_status by a kernel: bad data, rows skipped */
  CSA_ERR_TIMEOUT = 6      /* written to dev_status: a bounded device wait gave up */
};

#define CSA_HEAD_DIM 512   /* shared KV entry dims */
#define CSA_NOPE_DIM 448   /* dims stored as FP8 E4M3 */
#define CSA_ROPE_DIM 64    /* last dims, RoPE, stored as BF16 */
#define CSA_ROW_BYTES 576  /* 448 E4M3 bytes then 64 BF16 values */
#define CSA_INDEX_DIM 128  /* indexer head dim (E2M1, 64 bytes per head) */
#define CSA_WINDOW 128     /* sliding-window tokens */

/* Short description of a status code (static storage). */
const char* csa_status_string(int status);

/* ------------------------------------------------------------------------------------
 * Paged compressed cache (walkthrough §3.5: the classical cache holds the compressed
 * entries, in blocks aligned to 128 tokens, the least common multiple of the CSA and HCA
 * block sizes). With block_table == NULL the cache arrays of a call are contiguous per
 * sequence: kv [B][Nmax][576], kv_scale [B][Nmax], k_fp4 [B][Nmax][64],
 * k_sf [B][Nmax/128][512]. Otherwise they are pools of num_pages pages of page_entries
 * entries each: kv [num_pages][page_entries][576], kv_scale [num_pages][page_entries],
 * k_fp4 [num_pages][page_entries][64], k_sf [num_pages][page_entries/128][512], and entry
 * j of sequence b is slot j % page_entries of page block_table[b * pages_max +
 * j / page_entries] (the key scales follow their entries: group g of sequence b is group
 * (128 g % page_entries) / 128 of the page of entry 128 g).
 *   page_entries: a power of two, 128 .. 1048576 (512 or more CSA tokens per page);
 *   pages_max * page_entries >= Nmax; num_pages >= 1; block_table 16-byte aligned,
 *   [B][pages_max] int32, read only.
 * Only the pages that hold entries below n_entries[b] (or, for csa_decode_append, the
 * entry being written) are read from the table; such an entry outside 0 .. num_pages-1 is
 * reported as CSA_ERR_DEVICE (the call's results are then unspecified). Pages are never
 * allocated or freed by the library.
 */
typedef struct {
  const int32_t* block_table; /* [B][pages_max] physical page of each logical page, or NULL */
  int32_t pages_max;          /* table row length */
  int32_t page_entries;       /* entries per page */
  int32_t num_pages;          /* pages in each pool */
} csa_pages;

/* ------------------------------------------------------------------------------------
 * csa_compress: gated-softmax block compression of the KV stream into stored entries.
 * (walkthrough §2.2: two independent KV sequences merged with softmax-normalised gate
 * weights, adjacent blocks overlap; chooseai §一: positional bias; walkthrough §2.3:
 * RMSNorm on the entries; chooseai §一: RoPE dims BF16, others FP8.)
 *
 * The T tokens at absolute positions pos0 .. pos0+T-1 of each sequence (pos0 a multiple
 * of m) give N = floor(T/m) entries; entry i covers tokens pos0+m*i .. pos0+m*i+m-1 and is
 * stored at row pos0/m + i. For every dim d the merge is a softmax over the candidates
 *   own block:  a[m*i + r][d]       with logit za[m*i + r][d] + bias[r],        r < m
 *   previous:   b[m*(i-1) + r][d]   with logit zb[m*(i-1) + r][d] + bias[m + r]
 *               (overlap = 1 only; for i = 0 from prev_b / prev_zb when pos0 > 0, absent
 *               when pos0 == 0)
 * followed by y = e / sqrt(mean(e^2) + eps) * norm_w, RoPE on the interleaved pairs
 * (448+2j, 449+2j) by angle (pos0 + m*i) * rope_base^(-j/32), and the split store:
 * scale = max|y[0..447]| / 448 (1 if zero), bytes 0..447 = E4M3(y[d] / scale) rounded to
 * nearest even and saturated, bytes 448..575 = BF16(y[448..511]) rounded to nearest even.
 * Computed in fp32 on the device. Supports 1 <= m <= 128.
 */
typedef struct {
  int32_t B;             /* sequences */
  int32_t T;             /* tokens per sequence in this call (row pitch of a, b, za, zb) */
  int32_t m;             /* block size: 4 for CSA, 128 for HCA */
  int32_t overlap;       /* 1: CSA overlapping merge (needs b, zb); 0: HCA */
  int64_t pos0;          /* absolute position of token 0, a multiple of m */
  float rope_base;       /* 10000 */
  float eps;             /* RMSNorm epsilon, e.g. 1e-6 */
  const uint16_t* a;     /* bf16 [B][T][512] */
  const uint16_t* b;     /* bf16 [B][T][512]; NULL when overlap == 0 */
  const float* za;       /* [B][T][512] gate logits paired with a */
  const float* zb;       /* [B][T][512] gate logits paired with b; NULL when overlap == 0 */
  const float* bias;     /* [2m] (overlap) or [m] */
  const float* norm_w;   /* [512] RMSNorm weight, NULL = ones */
  const uint16_t* prev_b; /* bf16 [B][m][512]: tokens pos0-m .. pos0-1 of b (overlap, pos0>0) */
  const float* prev_zb;  /* [B][m][512] */
  uint8_t* kv;           /* out [B][Nmax][576] */
  float* kv_scale;       /* out [B][Nmax] */
  int64_t Nmax;          /* entry capacity per sequence; pos0/m + N <= Nmax */
  float* dbg;            /* optional out [B][N][512]: fp32 y before quantisation */
} csa_compress_args;

/* Unlike the other compute calls, csa_compress takes no workspace: each block's merge,
 * norm, rotation and quantisation stay on chip, so it needs no scratch memory. */
int csa_compress(const csa_compress_args* args, csa_stream_t stream);

/* ------------------------------------------------------------------------------------
 * csa_decode_append: one decode step's update of the per-sequence state (walkthrough
 * §3.5: the state cache holds the 128 window tokens and the tail of the unfinished
 * block, the classical cache the compressed entries).
 * For each sequence b with new token t = pos[b]:
 *   - a / za go to tail row t % m of tail_a / tail_za [B][m][512]; b / zb (overlap) to
 *     row t % m of slot (t / m) & 1 of the two-block ring tail_b / tail_zb [B][2][m][512]
 *     (the slot of block i - 1 is block i's previous block);
 *   - the window row of t (RMSNorm, RoPE at t, BF16, as csa_prefill's) is written to
 *     swa[b][t % 128];
 *   - when t % m == m - 1 the block t / m is compressed from the tails exactly as
 *     csa_compress (previous block from the ring when t / m > 0 and overlap = 1) into row
 *     t / m of kv / kv_scale, n_entries[b] = t / m + 1, and when the indexer-key stream
 *     is given (ia != NULL) its key is compressed as csa_compress_index_keys into
 *     k_fp4 / k_sf from the tails itail_* ([B][m][128], ring [B][2][m][128]).
 * The state buffers are the caller's; a sequence starting mid-stream must hold its
 * previous block in the ring slot of block t / m - 1. A position whose block would not
 * fit Nmax is reported through dev_status and skipped.
 */
typedef struct {
  int32_t B;               /* sequences, one new token each */
  int32_t m;               /* block size: 4 for CSA, 128 for HCA */
  int32_t overlap;         /* 1: CSA overlapping merge */
  float rope_base;         /* 10000 */
  float eps;               /* RMSNorm epsilon of entries and window rows */
  const int32_t* pos;      /* [B] position of the new token */
  const uint16_t* a;       /* bf16 [B][512] */
  const uint16_t* b;       /* bf16 [B][512] (overlap) */
  const float* za;         /* [B][512] */
  const float* zb;         /* [B][512] (overlap) */
  const float* bias;       /* [2m] or [m] */
  const float* norm_w;     /* [512] or NULL */
  uint16_t* tail_a;        /* state bf16 [B][m][512] */
  float* tail_za;          /* state [B][m][512] */
  uint16_t* tail_b;        /* state bf16 [B][2][m][512] (overlap) */
  float* tail_zb;          /* state [B][2][m][512] (overlap) */
  uint16_t* swa;           /* state bf16 [B][128][512] window ring */
  uint8_t* kv;             /* cache [B][Nmax][576] */
  float* kv_scale;         /* cache [B][Nmax] */
  int64_t Nmax;            /* entry capacity, multiple of 128 */
  int32_t* n_entries;      /* [B] updated when a block closes */
  const uint16_t* ia;      /* optional indexer-key stream: bf16 [B][128] (NULL: none) */
  const uint16_t* ib;      /* bf16 [B][128]: the key stream of the previous-block slots (as b) */
  const float* iza;        /* [B][128] gate logits paired with ia */
  const float* izb;        /* [B][128] gate logits paired with ib */
  const float* ibias;      /* [2m] */
  uint16_t* itail_a;       /* state bf16 [B][m][128] */
  float* itail_za;         /* state [B][m][128] */
  uint16_t* itail_b;       /* state bf16 [B][2][m][128] */
  float* itail_zb;         /* state [B][2][m][128] */
  uint8_t* k_fp4;          /* [B][Nmax][64] */
  uint8_t* k_sf;           /* [B][Nmax/128][512] */
  int32_t* dev_status;     /* optional device word */
  csa_pages pages;         /* kv, kv_scale, k_fp4, k_sf paged (block_table != NULL) */
} csa_append_args;

int csa_decode_append(const csa_append_args* args, csa_stream_t stream);

/* ------------------------------------------------------------------------------------
 * csa_compress_index_keys: the indexer keys of the compressed entries.
 * (walkthrough §2.2: the lightning indexer scores the compressed entries; §3.4: its QK
 * path is FP4.) The pages do not spell out how the indexer keys are built; this call
 * applies the gated merge of csa_compress (same candidate slots, bias layout and
 * previous-block handling) to a 128-dim indexer-key stream, with no norm and no RoPE,
 * and stores each entry as MXFP4 exactly as csa_indexer_topk reads it:
 *   per 32-element block s: e = floor(log2(max |y|)) - 2 (E8M0 code e + 127, clamped
 *   to 0..254; an all-zero block gets code 0), codes = E2M1(y / 2^e) rounded to nearest
 *   (ties to the even code) and saturated at +-6; element 2i in the low nibble of byte i
 *   of k_fp4 row pos0/m + i, the scale at the grouped k_sf position of that row.
 * Computed in fp32. Nmax must be a multiple of 128.
 */
typedef struct {
  int32_t B;              /* sequences */
  int32_t T;              /* tokens per sequence in this call (row pitch of a, b, za, zb) */
  int32_t m;              /* block size (4 for CSA) */
  int32_t overlap;        /* 1: overlapping merge (needs b, zb); 0: own block only */
  int64_t pos0;           /* absolute position of token 0, a multiple of m */
  const uint16_t* a;      /* bf16 [B][T][128] */
  const uint16_t* b;      /* bf16 [B][T][128]; NULL when overlap == 0 */
  const float* za;        /* [B][T][128] */
  const float* zb;        /* [B][T][128]; NULL when overlap == 0 */
  const float* bias;      /* [2m] (overlap) or [m] */
  const uint16_t* prev_b; /* bf16 [B][m][128] (overlap, pos0 > 0) */
  const float* prev_zb;   /* [B][m][128] */
  uint8_t* k_fp4;         /* out [B][Nmax][64] */
  uint8_t* k_sf;          /* out [B][Nmax/128][512] */
  int64_t Nmax;           /* multiple of 128; pos0/m + N <= Nmax */
  float* dbg;             /* optional out [B][N][128]: y before quantisation */
} csa_ikey_args;

int csa_compress_index_keys(const csa_ikey_args* args, csa_stream_t stream);

/* ------------------------------------------------------------------------------------
 * csa_indexer_query: the indexer queries of T tokens (walkthrough §2.2: low-rank indexer
 * queries, down-projected then up-projected into the indexer heads, the down projection
 * shared with the main attention; §3.4: FP4 QK path).
 *   y[t][o] = sum_j W[o][j] * c[t][j],  o < H_I * 128,  j < r
 * with c the query latent and W the up-projection (both BF16; BF16 tensor-core products,
 * fp32 accumulation), no norm and no RoPE, stored per head as MXFP4 with the rule of
 * csa_compress_index_keys: q_fp4 [T][H_I][64] (element 2i in the low nibble of byte i),
 * q_sf [T][H_I][4] -- the query layout of csa_indexer_topk. r is a multiple of 64
 * (at most 16384), H_I in {16, 32, 64}.
 */
typedef struct {
  int32_t T;              /* tokens */
  int32_t r;              /* latent dims, multiple of 64 */
  int32_t H_I;            /* indexer heads: 16, 32 or 64 */
  const uint16_t* c;      /* bf16 [T][r] */
  const uint16_t* W;      /* bf16 [H_I * 128][r] */
  uint8_t* q_fp4;         /* out [T][H_I][64] */
  uint8_t* q_sf;          /* out [T][H_I][4] */
  float* dbg;             /* optional out [T][H_I * 128]: y before quantisation */
  int32_t* dev_status;    /* optional device word */
} csa_iquery_args;

int csa_indexer_query(const csa_iquery_args* args, csa_stream_t stream);

/* ------------------------------------------------------------------------------------
 * csa_indexer_topk: lightning-indexer scores of every eligible entry and the top-k set.
 * (walkthrough §2.2: the indexer scores compressed entries, each query keeps the top-k,
 * one set shared by all heads; §3.4 and chooseai §二: the indexer QK path is MXFP4.)
 *
 *   s_j = sum_h w[h] * max(0, sum_d q[h][d] * k_j[d]),   j < n_entries[b]
 * where q and k are E2M1 codes times their E8M0 block scale (one per 32 dims). The set
 * is the first min(k, n) entries by (score descending, index ascending), written in
 * ascending index order and padded with -1. Scores are formed in fp32 from the FP4
 * tensor-core products (tcgen05 kind::mxf4).
 *
 * Layouts: q_fp4 [B][H_I][64] and k_fp4 [B][Nmax][64] hold two E2M1 codes per byte,
 * element 2i in the low nibble of byte i. q_sf [B][H_I][4] holds the 4 block scales of
 * each query head. k_sf is grouped by 128 entries: [B][Nmax/128][512] bytes, and the
 * scale of entry j (j = 128g + 32r1 + r0), block s, sits at byte 16*r0 + 4*r1 + s of
 * group g -- the tensor-core scale-factor atom, so a group is copied as is. This is not
 * the plain per-entry order [B][Nmax][4]: the keys' writers (csa_compress_index_keys,
 * csa_decode_append) store the atom order once, so no call has to repack the scales of
 * every entry it reads. Nmax must be a multiple of 128. 1 <= k <= 2048, H_I in {16, 32, 64}.
 * The workspace must be zero-filled once before its first use; every call that ends with
 * dev_status still zero leaves it zeroed again. After a call that reported
 * CSA_ERR_TIMEOUT or CSA_ERR_DEVICE (or any call whose dev_status was not read), zero-fill
 * the workspace again before reusing it: a call that gave up part-way leaves counts
 * behind. One workspace serves calls of any B and Nmax up to the sizes it was created
 * for (the parts kept at zero sit at offsets that do not depend on B). Calls that share a
 * workspace must not overlap on the device.
 *
 * Scoring and selection normally run in one cooperative launch with at most one CTA per
 * SM (and no more CTAs than the call has 512-entry key quads) and two grid-wide barriers;
 * if the runtime refuses that launch (for instance when other work holds SMs), scoring
 * runs as an ordinary launch followed by two selection kernels, with the same results.
 * The key stream is loaded with an L2 evict-first policy: it is read once per call. `flags` = CSA_TOPK_SEPARATE_SELECT takes that second path on
 * purpose (for testing it). `select_wait_ns` bounds each wait at the grid barriers of the
 * cooperative path (0 = 2 s); a wait that runs out writes CSA_ERR_TIMEOUT to dev_status
 * and the call returns with its outputs undefined.
 */
#define CSA_TOPK_SEPARATE_SELECT 1u
typedef struct {
  int32_t B;              /* queries (one per sequence) */
  int32_t H_I;                /* indexer heads: 16, 32 or 64 */
  int32_t k;                  /* top-k */
  int64_t Nmax;               /* entry capacity per sequence, multiple of 128 */
  const int32_t* n_entries;   /* [B] eligible entries per sequence, <= Nmax */
  const uint8_t* q_fp4;       /* [B][H_I][64] */
  const uint8_t* q_sf;        /* [B][H_I][4] E8M0 */
  const float* w;             /* [B][H_I] head weights */
  const uint8_t* k_fp4;       /* [B][Nmax][64] */
  const uint8_t* k_sf;        /* [B][Nmax/128][512] grouped E8M0 */
  int32_t* idx;               /* out [B][k] ascending, -1 padded */
  float* scores;              /* optional out [B][k]: score of idx[b][i] (NaN for -1) */
  int32_t* dev_status;        /* optional device word, see conventions */
  uint32_t flags;             /* 0 or CSA_TOPK_SEPARATE_SELECT */
  int64_t select_wait_ns;     /* limit of a grid-barrier wait in ns; 0 = the default */
  csa_pages pages;            /* k_fp4, k_sf paged (block_table != NULL) */
} csa_topk_args;

size_t csa_indexer_topk_workspace_size(int32_t B, int64_t Nmax, int32_t k);
int csa_indexer_topk(const csa_topk_args* args, void* workspace, size_t workspace_bytes,
                     csa_stream_t stream);

/* csa_indexer_topk_bf16: csa_indexer_topk with every score rounded to BF16 (nearest even)
 * before selection (walkthrough §3.4: the index scores are quantised from FP32 to BF16
 * for the top-k selector). Scores that round to the same BF16 value are ordered by
 * index. Same arguments, workspace and errors; `scores`, when given, returns the
 * rounded values. */
int csa_indexer_topk_bf16(const csa_topk_args* args, void* workspace, size_t workspace_bytes,
                          csa_stream_t stream);

/* ------------------------------------------------------------------------------------
 * csa_sparse_attn_decode / hca_attn_decode: one query token per sequence.
 * (tutorial "Hybrid Attention": shared key-value MQA; walkthrough §2.2: the 128 most
 * recent uncompressed tokens join the core attention, sink added to the denominator;
 * tutorial "Partial RoPE": the output is de-rotated.)
 *
 * For head h of sequence b at position t = pos[b], over the rows
 *   CSA: the entries idx[b][0..k) (-1 = padding, skipped), every index < n_entries[b];
 *   HCA: the entries 0 .. n_entries[b]-1;
 *   both: window tokens p = max(0, t-127) .. t from the ring swa[b][p % 128];
 *   l_j = tau * q[b][h] . v_j,  Z = exp(sink[h]) + sum_j exp(l_j),
 *   out[b][h] = sum_j exp(l_j) / Z * v_j,  lse[b][h] = log Z,
 * with v_j the dequantised entry (E4M3 code * entry scale, then the BF16 dims) or the
 * BF16 window row; when derotate = 1, output pairs (448+2j, 449+2j) are turned by
 * -t * rope_base^(-j/32). Products run on tcgen05 FP16 tensor cores: an entry row is
 * staged as its E4M3 codes (exact in FP16) and its BF16 dims divided by the entry scale,
 * the scale enters the logit and the probability instead; accumulation and softmax in
 * fp32. H in {64, 128}. k <= 2048 (CSA); n_entries <= Nmax (HCA, any size).
 *
 * Workspace: csa_attn_workspace_size(B, H, rows_max) bytes with rows_max = k + 128 (CSA)
 * or Nmax + 128 (HCA), 256-byte aligned, for the per-chunk partial outputs (rows are
 * taken 64 at a time; a second kernel merges the chunks in index order, so results do not
 * depend on the batch). It needs no initialisation.
 */
typedef struct {
  int32_t B;              /* queries (one per sequence) */
  int32_t H;                  /* query heads: 64 or 128 */
  int32_t k;                  /* CSA: selected entries per sequence; ignored by HCA */
  int64_t Nmax;               /* entry capacity per sequence */
  const uint16_t* q;          /* bf16 [B][H][512], already normalised and rotated */
  const int32_t* pos;         /* [B] query positions t >= 0 */
  const int32_t* idx;         /* [B][k] (CSA only) */
  const int32_t* n_entries;   /* [B] eligible entries */
  const uint8_t* kv;          /* [B][Nmax][576] stored entries */
  const float* kv_scale;      /* [B][Nmax] */
  const uint16_t* swa;        /* bf16 [B][128][512] window ring */
  const float* sink;          /* [H] sink logits (+-inf allowed) */
  float tau;                  /* softmax scale; 0 selects 1/sqrt(512) */
  float rope_base;            /* 10000 */
  int32_t derotate;           /* 1: de-rotate the last 64 output dims by the query position */
  uint16_t* out;              /* out bf16 [B][H][512] */
  float* lse;                 /* optional out [B][H] */
  int32_t* dev_status;        /* optional device word */
  csa_pages pages;            /* kv, kv_scale paged (block_table != NULL) */
} csa_attn_args;

size_t csa_attn_workspace_size(int32_t B, int32_t H, int32_t rows_max);
int csa_sparse_attn_decode(const csa_attn_args* args, void* workspace, size_t workspace_bytes,
                           csa_stream_t stream);
int hca_attn_decode(const csa_attn_args* args, void* workspace, size_t workspace_bytes,
                    csa_stream_t stream);

/* ------------------------------------------------------------------------------------
 * csa_prefill: causal CSA prefill of T new tokens of one sequence after a P-token prefix.
 * (walkthrough §2.2 for every step; §3.5: the state cache carries the 128 window tokens
 * and the previous block across chunks, the classical cache the compressed entries.)
 *
 * 1. Compression of the new blocks (as csa_compress with pos0 = P, overlap on): entries
 *    P/m .. (P+T)/m - 1 are written into kv / kv_scale; rows 0 .. P/m - 1 are the cached
 *    prefix and are only read. T may leave a tail of T % m tokens: their block is not
 *    emitted (it stays in the caller's state).
 * 2. For every new token t = P + r (r = 0 .. T-1), with n(t) eligible entries (below):
 *    the indexer top-k over entries j < n(t) (as csa_indexer_topk, all queries
 *    scoring the one key array k_fp4 / k_sf, which must hold the indexer keys of every
 *    entry up to (P+T)/m), then CSA attention over the selected entries, the window
 *    t-127 .. t and the sink (as csa_sparse_attn_decode with pos = t). Window rows of
 *    prefix positions come from the ring swa_prefix[p % 128]; window rows of new tokens
 *    are RMSNorm (eps, norm_w) then RoPE at position p of a[p - P], rounded to BF16.
 *
 * Eligibility: the pages say a query sees the compressed blocks that are complete. With
 * strict_eligibility = 0 (the default reading) the block whose last token is t itself
 * counts: n(t) = floor((t+1)/m), so a prefill row at t equals a decode step at t just after
 * that block closed. With strict_eligibility = 1 only blocks completed before t count:
 * n(t) = floor(t/m). The window t-127 .. t is the same under both.
 *
 * Layouts: a, b bf16 [T][512]; za, zb [T][512]; bias [2m]; prev_b bf16 [m][512] and
 * prev_zb [m][512] are the m tokens before P (needed when P > 0); kv [Nmax][576];
 * kv_scale [Nmax]; q_fp4 [T][H_I][64]; q_sf [T][H_I][4]; w [T][H_I]; k_fp4 [Nmax][64];
 * k_sf [Nmax/128][512] (grouped as in csa_indexer_topk); q bf16 [T][H][512];
 * swa_prefix bf16 [128][512] (needed when P > 0); out bf16 [T][H][512]; lse [T][H];
 * idx [T][k]. m in 1..128, P % m == 0, Nmax a positive multiple of 128 with
 * (P+T)/m <= Nmax (the key array is read in 128-entry tiles, so it holds at least one
 * tile even when no block is complete), H in {64, 128}, H_I in {16, 32, 64},
 * 1 <= k <= 2048.
 * The workspace (csa_prefill_workspace_size) must be zero-filled once before its first
 * use; every call leaves the parts that must start at zero zeroed again. It includes a
 * staging area of Nmax x 648 bytes that a call on a paged cache (csa_pages) fills with
 * the prefix's rows and all keys before it runs, and copies the new rows back from.
 */
typedef struct {
  int64_t P;                  /* prefix tokens, a multiple of m */
  int32_t T;                  /* new tokens */
  int32_t m;                  /* compression ratio (4 for CSA) */
  int32_t H;                  /* query heads: 64 or 128 */
  int32_t H_I;                /* indexer heads: 16, 32 or 64 */
  int32_t k;                  /* top-k */
  int64_t Nmax;               /* entry capacity, positive multiple of 128 */
  float tau;                  /* softmax scale; 0 selects 1/sqrt(512) */
  float rope_base;            /* 10000 */
  float eps;                  /* RMSNorm epsilon */
  int32_t derotate;           /* 1: de-rotate the last 64 output dims by t */
  int32_t strict_eligibility; /* 0: n(t) = floor((t+1)/m); 1: n(t) = floor(t/m) */
  const uint16_t* a;          /* new tokens (see Layouts) */
  const uint16_t* b;          /* bf16 [T][512], the previous-block stream */
  const float* za;            /* [T][512] gate logits paired with a */
  const float* zb;            /* [T][512] gate logits paired with b */
  const float* bias;          /* [2m] slot bias */
  const float* norm_w;        /* [512] or NULL = ones (entries and window rows) */
  const uint16_t* prev_b;     /* bf16 [m][512]: tokens P-m .. P-1 of b (P > 0) */
  const float* prev_zb;       /* [m][512] (P > 0) */
  uint8_t* kv;                /* in: prefix rows; out: the new rows */
  float* kv_scale;            /* [Nmax], as kv */
  const uint8_t* q_fp4;       /* [T][H_I][64] MXFP4 indexer queries */
  const uint8_t* q_sf;        /* [T][H_I][4] E8M0 scales */
  const float* w;             /* [T][H_I] indexer head weights */
  const uint8_t* k_fp4;       /* [Nmax][64] indexer keys of every entry up to (P+T)/m */
  const uint8_t* k_sf;        /* [Nmax/128][512] grouped key scales */
  const uint16_t* q;          /* bf16 [T][H][512] queries (RMS-normalised, rotated at t) */
  const float* sink;          /* [H] */
  const uint16_t* swa_prefix; /* bf16 [128][512] window ring of the prefix (P > 0) */
  uint16_t* out;              /* out bf16 [T][H][512] */
  float* lse;                 /* optional */
  int32_t* idx;               /* optional: the selected sets */
  int32_t* dev_status;        /* optional device word */
  csa_pages pages;            /* kv, kv_scale, k_fp4, k_sf paged (table [1][pages_max]) */
} csa_prefill_args;

size_t csa_prefill_workspace_size(int32_t T, int64_t Nmax, int32_t H, int32_t k);
int csa_prefill(const csa_prefill_args* args, void* workspace, size_t workspace_bytes,
                csa_stream_t stream);

/* ------------------------------------------------------------------------------------
 * csa_grouped_out_proj: the grouped output projection after the attention (walkthrough
 * §2.2: the heads are reduced group by group, then the concatenation is projected).
 * The H heads of a token form G groups of H/G consecutive heads:
 *   mid[t][g*d_g + o] = BF16( sum_j Wg[g][o][j] * attn[t][g*H/G*512 + j] )
 *   out[t][o]         = BF16( sum_j Wo[o][j] * mid[t][j] )
 * BF16 tensor-core products with fp32 accumulation. attn bf16 [T][H][512] (the
 * attention output), Wg bf16 [G][d_g][H/G * 512], Wo bf16 [d_model][G * d_g],
 * out bf16 [T][d_model]; the workspace holds mid [T][G * d_g]
 * (csa_grouped_out_proj_workspace_size). H in {64, 128}, G divides H, d_g and d_model
 * multiples of 128.
 */
typedef struct {
  int32_t T;             /* tokens */
  int32_t H;             /* heads: 64 or 128 */
  int32_t G;             /* groups of H/G consecutive heads */
  int32_t d_g;           /* reduced width per group, multiple of 128 */
  int32_t d_model;       /* output width, multiple of 128 */
  const uint16_t* attn;  /* bf16 [T][H][512] attention output */
  const uint16_t* Wg;    /* bf16 [G][d_g][H/G * 512] per-group reductions */
  const uint16_t* Wo;    /* bf16 [d_model][G * d_g] output projection */
  uint16_t* out;         /* out bf16 [T][d_model] */
  int32_t* dev_status;   /* optional device word */
} csa_oproj_args;

size_t csa_grouped_out_proj_workspace_size(int32_t T, int32_t G, int32_t d_g);
int csa_grouped_out_proj(const csa_oproj_args* args, void* workspace, size_t workspace_bytes,
                         csa_stream_t stream);

/* ------------------------------------------------------------------------------------
 * csa_sparse_attn_decode_noalloc: csa_sparse_attn_decode without a workspace argument.
 * The pages have no counterpart: this is an interface convenience, not part of the method.
 *
 * It is for callers that cannot hand over scratch memory: a host that exposes only a
 * C function taking the layer's inputs and outputs (a plugin slot with no allocator), or
 * code running while a stream is being captured into a graph, where cudaMalloc/cudaFree
 * are not allowed and would otherwise synchronise the device.
 *
 * Scratch comes from one file-scope device array of CSA_NOALLOC_SCRATCH_BYTES per device
 * (12 MiB; enough for B = 4, H = 128, k = 1024). Its address is looked up with
 * cudaGetSymbolAddress on the first call on each device and cached together with the
 * current context; a call under another context of that device (or after the device's
 * primary context was reset) looks it up again. Make the first call of each device and
 * context outside stream capture (for instance one ordinary call before capturing).
 * Nothing in the scratch has to start at zero: every partial result is written before it
 * is read.
 *
 * Results are the same as csa_sparse_attn_decode with a caller workspace (the same
 * kernels run). Arguments are checked as there; a problem whose scratch
 * (csa_attn_workspace_size(B, H, k + 128)) exceeds the array returns CSA_ERR_UNSUPPORTED
 * before anything touches the device. Calls that can overlap in time on one device (two
 * streams, two host threads, or concurrently replayed graphs) share the array and race;
 * calls on a single stream are ordered and safe.
 */
#define CSA_NOALLOC_SCRATCH_BYTES (12u << 20)
int csa_sparse_attn_decode_noalloc(const csa_attn_args* args, csa_stream_t stream);

/* ------------------------------------------------------------------------------------
 * csa_mma_peak: a measurement helper, not part of the layer. One CTA per SM issues `iters`
 * back-to-back tcgen05 MMAs (M = 128) on operands resident in shared memory, with no DRAM
 * traffic: kind = 0 is kind::mxf4 (E2M1 inputs, E8M0 block scales, K = 64 per MMA, N = 64),
 * kind = 1 is kind::f16 with BF16 inputs (K = 16 per MMA, N = 64 or 256). The caller times
 * the launch on `stream`; csa_mma_peak_flops gives the FLOPs of one launch on the current
 * device (0 for an unsupported kind or N). The ratio of the two kinds' rates at one shape
 * scales a measured BF16 GEMM peak into an FP4 one. iters in 1 .. 1e6; a wait that runs
 * out writes CSA_ERR_TIMEOUT to dev_status (optional).
 */
int csa_mma_peak(int32_t kind, int32_t N, int32_t iters, int32_t* dev_status,
                 csa_stream_t stream);
double csa_mma_peak_flops(int32_t kind, int32_t N, int32_t iters);

#ifdef __cplusplus
}
#endif

#endif /* CSA_B200_H */
