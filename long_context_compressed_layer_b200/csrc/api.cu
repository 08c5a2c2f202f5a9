// extern "C" entry points of the CSA/HCA layer library: argument checks on the host, TMA
// tensor maps, workspace carving and kernel launches. Nothing here allocates, frees or
// synchronises; every failure is a status code.
#include <atomic>
#include <cstring>

#include "common.cuh"

namespace csa {
cudaError_t launch_compress(const csa_compress_args& a, cudaStream_t stream);
cudaError_t launch_ikey_compress(const csa_ikey_args& a, cudaStream_t stream);
cudaError_t launch_append(const csa_append_args& a, cudaStream_t stream);
cudaError_t launch_gemm_bf16(const CUtensorMap& amap, const CUtensorMap& bmap, int M, int N,
                             int K, int G, int a_x_group, int b_y_group, int64_t c_x_group,
                             uint16_t* C, int64_t ldc, int32_t* dev_status, cudaStream_t stream);
cudaError_t launch_iquery(const csa_iquery_args& a, const CUtensorMap& cmap,
                          const CUtensorMap& wmap, cudaStream_t stream);
cudaError_t launch_indexer_topk(const csa_topk_args& a, void* workspace, int num_sms,
                                const CUtensorMap& kmap, cudaStream_t stream, int bf16);
size_t ix_workspace_size(int B, int64_t Nmax, int k);
cudaError_t launch_prefill_indexer_topk(const csa_topk_args& a, void* workspace, int num_sms,
                                        const CUtensorMap& kmap, cudaStream_t stream);
size_t at_workspace_size(int B, int H, int rows_max);
cudaError_t launch_prefill_attn(const csa_attn_args& a, const __half* rows16, int64_t swa_base,
                                const CUtensorMap& qmap, cudaStream_t stream);
cudaError_t launch_prefill_rows16(const uint8_t* kv, const float* kv_scale, int64_t n,
                                  __half* rows16, cudaStream_t stream);
cudaError_t launch_prefill_prep(const csa_prefill_args& a, __half* lin, int32_t* n_all,
                                int32_t* pos_all, cudaStream_t stream);
cudaError_t launch_attn(const csa_attn_args& a, int sparse, int rows_max, void* workspace,
                        const CUtensorMap& qmap, cudaStream_t stream);
cudaError_t launch_page_gather(const PageMap& pm, const uint8_t* kv, const float* kv_scale,
                               const uint8_t* k_fp4, const uint8_t* k_sf, uint8_t* kv_c,
                               float* sc_c, uint8_t* kf_c, uint8_t* ksf_c, int64_t n_kv,
                               int64_t n_keys, int32_t* dev_status, cudaStream_t stream);
cudaError_t launch_page_scatter(const PageMap& pm, const uint8_t* kv_c, const float* sc_c,
                                uint8_t* kv, float* kv_scale, int64_t j0, int64_t j1,
                                int32_t* dev_status, cudaStream_t stream);
double mma_peak_flops_per_cta(int kind, int N, int iters);
cudaError_t launch_mma_peak(int kind, int N, int iters, int num_sms, int32_t* dev_status,
                            cudaStream_t stream);

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once (a function-local static: thread-safe
// initialisation); nullptr when the driver does not provide it.
EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    return nullptr;
  }();
  return fn;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }
bool ok_opt(const void* p) { return p == nullptr || aligned16(p); }

// a paged-cache descriptor: unused (no table), or a consistent one covering Nmax entries
bool ok_pages(const csa_pages& pg, int64_t Nmax) {
  if (!pg.block_table) return true;
  const int64_t pe = pg.page_entries;
  return aligned16(pg.block_table) && pe >= 128 && pe <= (1 << 20) && (pe & (pe - 1)) == 0 &&
         pg.pages_max >= 1 && pg.num_pages >= 1 && (int64_t)pg.pages_max * pe >= Nmax;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? CSA_OK : CSA_ERR_CUDA; }

// Scratch of csa_sparse_attn_decode_noalloc: one array per device, zero-initialised when
// the module loads. Its device address is looked up with cudaGetSymbolAddress and cached
// per device together with the context it belongs to: a call under another context of
// that device (or after the primary context was reset) looks it up again.
__device__ __align__(256) unsigned char g_noalloc_scratch[CSA_NOALLOC_SCRATCH_BYTES];
constexpr int kMaxDevices = 64;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CtxGetCurrentFn ctx_get_current_fn() {
  static const CtxGetCurrentFn fn = []() -> CtxGetCurrentFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<CtxGetCurrentFn>(p);
    return nullptr;
  }();
  return fn;
}

void* noalloc_scratch() {
  struct Slot {
    std::atomic<void*> ctx{nullptr};
    std::atomic<void*> ptr{nullptr};
  };
  static Slot cache[kMaxDevices];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  CtxGetCurrentFn get_ctx = ctx_get_current_fn();
  if (!get_ctx) return nullptr;
  CUcontext ctx = nullptr;  // null before the runtime has made its context current
  if (get_ctx(&ctx) != CUDA_SUCCESS) return nullptr;
  Slot& s = cache[dev];
  void* p = s.ptr.load(std::memory_order_acquire);
  if (ctx && p && s.ctx.load(std::memory_order_acquire) == (void*)ctx) return p;
  p = nullptr;  // the lookup also sets up the runtime's context when it is not yet current
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return nullptr;
  // both words are rewritten on a change of context; a thread that reads a mixed pair
  // looks the address up again, which returns the same value
  s.ptr.store(nullptr, std::memory_order_release);
  s.ctx.store((void*)ctx, std::memory_order_release);
  s.ptr.store(p, std::memory_order_release);
  return p;
}

// Queries of a prefill handled per indexer / attention launch (the indexer keeps one
// prefix-sum slot per query in shared memory).
constexpr int kPrefillChunk = 1024;

struct PrefillWs {
  char* ix;           // indexer workspace for kPrefillChunk queries (kept zeroed)
  int32_t* n_all;     // [T]
  int32_t* pos_all;   // [T]
  __half* rows16;     // FP16 rows: [Nmax] entries, then [T + 127] window rows in position order
  int32_t* idx;       // [chunk][k] selected sets when the caller passes none
  // contiguous staging of a paged cache: rows [Nmax][576], scales [Nmax], keys [Nmax][64],
  // key scales [Nmax/128][512]
  uint8_t* kv_c;
  float* sc_c;
  uint8_t* kf_c;
  uint8_t* ksf_c;
};

size_t prefill_ws_layout(int T, int64_t Nmax, int H, int k, char* base, PrefillWs* w) {
  const int qc = T < kPrefillChunk ? (T > 0 ? T : 1) : kPrefillChunk;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off += (bytes + 255) & ~(size_t)255;
    return p;
  };
  char* ix = take(ix_workspace_size(qc, Nmax, k));
  char* n_all = take((size_t)T * 4);
  char* pos_all = take((size_t)T * 4);
  char* rows16 = take(((size_t)Nmax + T + CSA_WINDOW - 1) * CSA_HEAD_DIM * 2);
  char* idx = take((size_t)qc * k * 4);
  char* kv_c = take((size_t)Nmax * CSA_ROW_BYTES);
  char* sc_c = take((size_t)Nmax * 4);
  char* kf_c = take((size_t)Nmax * 64);
  char* ksf_c = take((size_t)Nmax / 128 * 512);
  (void)H;
  if (w) {
    w->kv_c = reinterpret_cast<uint8_t*>(kv_c);
    w->sc_c = reinterpret_cast<float*>(sc_c);
    w->kf_c = reinterpret_cast<uint8_t*>(kf_c);
    w->ksf_c = reinterpret_cast<uint8_t*>(ksf_c);
    w->ix = ix;
    w->n_all = reinterpret_cast<int32_t*>(n_all);
    w->pos_all = reinterpret_cast<int32_t*>(pos_all);
    w->rows16 = reinterpret_cast<__half*>(rows16);
    w->idx = reinterpret_cast<int32_t*>(idx);
  }
  return off;
}

bool encode_q_map(EncodeTiledFn enc, CUtensorMap* qmap, const uint16_t* q, int64_t rows, int H) {
  const cuuint64_t dims[2] = {CSA_HEAD_DIM, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {CSA_HEAD_DIM * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)H};
  const cuuint32_t estr[2] = {1, 1};
  return enc(qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(q), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// A BF16 matrix [rows][cols] (row-major) read in 64 x 128 boxes with the 128-byte swizzle.
bool encode_bf16_map(EncodeTiledFn enc, CUtensorMap* map, const uint16_t* base, int64_t cols,
                     int64_t rows) {
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(base), dims,
             strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

bool encode_key_map(EncodeTiledFn enc, CUtensorMap* kmap, const uint8_t* k_fp4, int64_t Nmax,
                    int64_t B) {
  const cuuint64_t dims[3] = {64, (cuuint64_t)Nmax, (cuuint64_t)B};
  const cuuint64_t strides[2] = {64, (cuuint64_t)Nmax * 64};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(k_fp4), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

}  // namespace
}  // namespace csa

using namespace csa;

extern "C" {

const char* csa_status_string(int status) {
  switch (status) {
    case CSA_OK: return "ok";
    case CSA_ERR_INVALID_ARG: return "invalid argument";
    case CSA_ERR_UNSUPPORTED: return "unsupported configuration";
    case CSA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case CSA_ERR_CUDA: return "CUDA launch or driver error";
    case CSA_ERR_DEVICE: return "a kernel found invalid data (rows skipped)";
    case CSA_ERR_TIMEOUT: return "a bounded device wait gave up";
    default: return "unknown status";
  }
}

int csa_compress(const csa_compress_args* a, csa_stream_t stream) {
  if (!a) return CSA_ERR_INVALID_ARG;
  if (a->B < 0 || a->T < 0 || a->m < 1 || a->m > 128 || a->pos0 < 0 || a->pos0 % a->m ||
      a->Nmax < 0 || (a->overlap != 0 && a->overlap != 1) || !(a->eps >= 0.f) ||
      !(a->rope_base > 0.f))
    return CSA_ERR_INVALID_ARG;
  if (a->B > 65535) return CSA_ERR_UNSUPPORTED;
  const int N = a->T / a->m;
  if (a->pos0 / a->m + N > a->Nmax) return CSA_ERR_INVALID_ARG;
  if (a->B == 0 || N == 0) return CSA_OK;
  if (!ok_ptr(a->a) || !ok_ptr(a->za) || !ok_ptr(a->bias) || !ok_ptr(a->kv) ||
      !ok_ptr(a->kv_scale) || !ok_opt(a->norm_w) || !ok_opt(a->dbg))
    return CSA_ERR_INVALID_ARG;
  if (a->overlap) {
    if (!ok_ptr(a->b) || !ok_ptr(a->zb)) return CSA_ERR_INVALID_ARG;
    if (a->pos0 > 0 && (!ok_ptr(a->prev_b) || !ok_ptr(a->prev_zb))) return CSA_ERR_INVALID_ARG;
  }
  return cuda_status(launch_compress(*a, reinterpret_cast<cudaStream_t>(stream)));
}

int csa_decode_append(const csa_append_args* a, csa_stream_t stream) {
  if (!a) return CSA_ERR_INVALID_ARG;
  if (a->B < 0 || a->m < 1 || a->m > 128 || a->Nmax < 0 || a->Nmax % 128 ||
      (a->overlap != 0 && a->overlap != 1) || !(a->eps >= 0.f) || !(a->rope_base > 0.f))
    return CSA_ERR_INVALID_ARG;
  if (a->B > 65535) return CSA_ERR_UNSUPPORTED;
  if (a->B == 0) return CSA_OK;
  if (!ok_ptr(a->pos) || !ok_ptr(a->a) || !ok_ptr(a->za) || !ok_ptr(a->bias) ||
      !ok_opt(a->norm_w) || !ok_ptr(a->tail_a) || !ok_ptr(a->tail_za) || !ok_ptr(a->swa) ||
      !ok_ptr(a->kv) || !ok_ptr(a->kv_scale) || !ok_ptr(a->n_entries) ||
      (a->dev_status && (reinterpret_cast<uintptr_t>(a->dev_status) & 3)) ||
      !ok_pages(a->pages, a->Nmax))
    return CSA_ERR_INVALID_ARG;
  if (a->overlap && (!ok_ptr(a->b) || !ok_ptr(a->zb) || !ok_ptr(a->tail_b) || !ok_ptr(a->tail_zb)))
    return CSA_ERR_INVALID_ARG;
  if (a->ia && (!ok_ptr(a->ib) || !ok_ptr(a->iza) || !ok_ptr(a->izb) || !ok_ptr(a->ibias) ||
                !ok_ptr(a->itail_a) || !ok_ptr(a->itail_za) || !ok_ptr(a->itail_b) ||
                !ok_ptr(a->itail_zb) || !ok_ptr(a->k_fp4) || !ok_ptr(a->k_sf) || !a->overlap))
    return CSA_ERR_INVALID_ARG;
  return cuda_status(launch_append(*a, reinterpret_cast<cudaStream_t>(stream)));
}

int csa_compress_index_keys(const csa_ikey_args* a, csa_stream_t stream) {
  if (!a) return CSA_ERR_INVALID_ARG;
  if (a->B < 0 || a->T < 0 || a->m < 1 || a->m > 128 || a->pos0 < 0 || a->pos0 % a->m ||
      a->Nmax < 0 || a->Nmax % 128 || (a->overlap != 0 && a->overlap != 1))
    return CSA_ERR_INVALID_ARG;
  if (a->B > 65535) return CSA_ERR_UNSUPPORTED;
  const int N = a->T / a->m;
  if (a->pos0 / a->m + N > a->Nmax) return CSA_ERR_INVALID_ARG;
  if (a->B == 0 || N == 0) return CSA_OK;
  if (!ok_ptr(a->a) || !ok_ptr(a->za) || !ok_ptr(a->bias) || !ok_ptr(a->k_fp4) ||
      !ok_ptr(a->k_sf) || !ok_opt(a->dbg))
    return CSA_ERR_INVALID_ARG;
  if (a->overlap) {
    if (!ok_ptr(a->b) || !ok_ptr(a->zb)) return CSA_ERR_INVALID_ARG;
    if (a->pos0 > 0 && (!ok_ptr(a->prev_b) || !ok_ptr(a->prev_zb))) return CSA_ERR_INVALID_ARG;
  }
  return cuda_status(launch_ikey_compress(*a, reinterpret_cast<cudaStream_t>(stream)));
}

int csa_indexer_query(const csa_iquery_args* a, csa_stream_t stream) {
  if (!a) return CSA_ERR_INVALID_ARG;
  if (a->T < 0 || a->r < 64 || a->r % 64) return CSA_ERR_INVALID_ARG;
  if (a->r > 16384 || (a->H_I != 16 && a->H_I != 32 && a->H_I != 64)) return CSA_ERR_UNSUPPORTED;
  if (a->T == 0) return CSA_OK;
  if (!ok_ptr(a->c) || !ok_ptr(a->W) || !ok_ptr(a->q_fp4) || !ok_ptr(a->q_sf) ||
      !ok_opt(a->dbg) || (a->dev_status && (reinterpret_cast<uintptr_t>(a->dev_status) & 3)))
    return CSA_ERR_INVALID_ARG;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return CSA_ERR_CUDA;
  CUtensorMap cmap, wmap;
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  const cuuint64_t cdims[2] = {(cuuint64_t)a->r, (cuuint64_t)a->T};
  const cuuint64_t wdims[2] = {(cuuint64_t)a->r, (cuuint64_t)a->H_I * 128};
  const cuuint64_t strides[1] = {(cuuint64_t)a->r * 2};
  if (enc(&cmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a->c), cdims,
          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
      enc(&wmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a->W), wdims,
          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return CSA_ERR_CUDA;
  return cuda_status(launch_iquery(*a, cmap, wmap, reinterpret_cast<cudaStream_t>(stream)));
}

size_t csa_grouped_out_proj_workspace_size(int32_t T, int32_t G, int32_t d_g) {
  if (T < 0 || G < 1 || d_g < 1) return 0;
  return (((size_t)T * G * d_g * 2) + 255) & ~(size_t)255;
}

int csa_grouped_out_proj(const csa_oproj_args* a, void* ws, size_t ws_bytes,
                         csa_stream_t stream) {
  if (!a) return CSA_ERR_INVALID_ARG;
  if (a->T < 0 || a->G < 1 || a->d_g < 1 || a->d_model < 1) return CSA_ERR_INVALID_ARG;
  if ((a->H != 64 && a->H != 128) || a->H % a->G || a->d_g % 128 || a->d_model % 128 ||
      (int64_t)a->G * a->d_g > 65536)
    return CSA_ERR_UNSUPPORTED;
  if (a->T == 0) return CSA_OK;
  if (!ok_ptr(a->attn) || !ok_ptr(a->Wg) || !ok_ptr(a->Wo) || !ok_ptr(a->out) ||
      (a->dev_status && (reinterpret_cast<uintptr_t>(a->dev_status) & 3)))
    return CSA_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255) ||
      ws_bytes < csa_grouped_out_proj_workspace_size(a->T, a->G, a->d_g))
    return CSA_ERR_WORKSPACE;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return CSA_ERR_CUDA;
  const int K1 = a->H / a->G * CSA_HEAD_DIM, M = a->G * a->d_g;
  uint16_t* mid = reinterpret_cast<uint16_t*>(ws);
  CUtensorMap m_attn, m_wg, m_mid, m_wo;
  if (!encode_bf16_map(enc, &m_attn, a->attn, (int64_t)a->H * CSA_HEAD_DIM, a->T) ||
      !encode_bf16_map(enc, &m_wg, a->Wg, K1, (int64_t)a->G * a->d_g) ||
      !encode_bf16_map(enc, &m_mid, mid, M, a->T) ||
      !encode_bf16_map(enc, &m_wo, a->Wo, M, a->d_model))
    return CSA_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_gemm_bf16(m_attn, m_wg, a->T, a->d_g, K1, a->G, K1, a->d_g, a->d_g,
                                   mid, M, a->dev_status, st);
  if (e != cudaSuccess) return CSA_ERR_CUDA;
  return cuda_status(launch_gemm_bf16(m_mid, m_wo, a->T, a->d_model, M, 1, 0, 0, 0, a->out,
                                      a->d_model, a->dev_status, st));
}

size_t csa_indexer_topk_workspace_size(int32_t B, int64_t Nmax, int32_t k) {
  if (B < 0 || Nmax < 0 || k < 1) return 0;
  return ix_workspace_size(B, Nmax, k);
}

static int indexer_common(const csa_topk_args* a, void* ws, size_t ws_bytes,
                          csa_stream_t stream, int bf16) {
  if (!a) return CSA_ERR_INVALID_ARG;
  if (a->B < 0 || a->k < 1 || a->Nmax < 0 || a->Nmax % 128 != 0 ||
      (a->flags & ~CSA_TOPK_SEPARATE_SELECT) || a->select_wait_ns < 0)
    return CSA_ERR_INVALID_ARG;
  if (a->H_I != 16 && a->H_I != 32 && a->H_I != 64) return CSA_ERR_UNSUPPORTED;
  if (a->k > 2048 || a->B > 1024 || a->Nmax > ((int64_t)1 << 30)) return CSA_ERR_UNSUPPORTED;
  if (a->B == 0) return CSA_OK;
  if (!ok_ptr(a->n_entries) || !ok_ptr(a->q_fp4) || !ok_ptr(a->q_sf) || !ok_ptr(a->w) ||
      !ok_ptr(a->k_fp4) || !ok_ptr(a->k_sf) || !ok_ptr(a->idx) || !ok_opt(a->scores) ||
      (a->dev_status && (reinterpret_cast<uintptr_t>(a->dev_status) & 3)) ||
      !ok_pages(a->pages, a->Nmax))
    return CSA_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255) ||
      ws_bytes < ix_workspace_size(a->B, a->Nmax, a->k))
    return CSA_ERR_WORKSPACE;
  const int sms = num_sms();
  EncodeTiledFn enc = encode_fn();
  if (sms <= 0 || !enc) return CSA_ERR_CUDA;
  if (a->Nmax == 0) {
    // no entry can be eligible: the select pass alone writes the -1 padding
  }
  // the keys as [B][Nmax/128 tiles][128 entries][64 bytes], read four tiles per copy; a
  // paged pool as [num_pages][page_entries/128 tiles][128][64], read min(4, tiles per
  // page) tiles per copy
  CUtensorMap kmap;
  std::memset(&kmap, 0, sizeof(kmap));
  if (a->Nmax > 0) {
    const bool paged = a->pages.block_table != nullptr;
    const int64_t tiles = paged ? a->pages.page_entries / 128 : a->Nmax / 128;
    const cuuint64_t dims[4] = {64, 128, (cuuint64_t)tiles,
                                (cuuint64_t)(paged ? a->pages.num_pages : a->B)};
    const cuuint64_t strides[3] = {64, 128 * 64, (cuuint64_t)tiles * 128 * 64};
    // contiguous: always four tiles (those past Nmax read as zeros, and the barrier expects
    // the whole box); paged: the tiles of one copy never leave their page
    const cuuint32_t box[4] = {64, 128, (cuuint32_t)(paged && tiles < 4 ? tiles : 4), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    if (enc(&kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<uint8_t*>(a->k_fp4), dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return CSA_ERR_CUDA;
  }
  return cuda_status(
      launch_indexer_topk(*a, ws, sms, kmap, reinterpret_cast<cudaStream_t>(stream), bf16));
}

int csa_indexer_topk(const csa_topk_args* a, void* ws, size_t ws_bytes, csa_stream_t stream) {
  return indexer_common(a, ws, ws_bytes, stream, 0);
}

int csa_indexer_topk_bf16(const csa_topk_args* a, void* ws, size_t ws_bytes,
                          csa_stream_t stream) {
  return indexer_common(a, ws, ws_bytes, stream, 1);
}

size_t csa_attn_workspace_size(int32_t B, int32_t H, int32_t rows_max) {
  if (B < 0 || H < 1 || rows_max < 0) return 0;
  return at_workspace_size(B, H, rows_max);
}

static int attn_common(const csa_attn_args* a, int sparse, void* ws, size_t ws_bytes,
                       csa_stream_t stream) {
  if (!a) return CSA_ERR_INVALID_ARG;
  if (a->B < 0 || a->Nmax < 0 || (sparse && a->k < 1) || !(a->tau >= 0.f) ||
      !(a->rope_base > 0.f) || (a->derotate != 0 && a->derotate != 1))
    return CSA_ERR_INVALID_ARG;
  if (a->H != 64 && a->H != 128) return CSA_ERR_UNSUPPORTED;
  if ((sparse && a->k > 2048) || a->B > 65535 || a->Nmax > ((int64_t)1 << 30))
    return CSA_ERR_UNSUPPORTED;
  if (a->B == 0) return CSA_OK;
  if (!ok_ptr(a->q) || !ok_ptr(a->pos) || !ok_ptr(a->n_entries) || !ok_ptr(a->kv) ||
      !ok_ptr(a->kv_scale) || !ok_ptr(a->swa) || !ok_ptr(a->sink) || !ok_ptr(a->out) ||
      !ok_opt(a->lse) || (sparse && !ok_ptr(a->idx)) ||
      (a->dev_status && (reinterpret_cast<uintptr_t>(a->dev_status) & 3)) ||
      !ok_pages(a->pages, a->Nmax))
    return CSA_ERR_INVALID_ARG;
  const int64_t rows_max64 = (sparse ? (int64_t)a->k : a->Nmax) + CSA_WINDOW;
  const int rows_max = (int)rows_max64;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255) ||
      ws_bytes < at_workspace_size(a->B, a->H, rows_max))
    return CSA_ERR_WORKSPACE;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return CSA_ERR_CUDA;
  CUtensorMap qmap;
  const cuuint64_t dims[2] = {CSA_HEAD_DIM, (cuuint64_t)a->B * a->H};
  const cuuint64_t strides[1] = {CSA_HEAD_DIM * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)a->H};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a->q), dims, strides,
          box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return CSA_ERR_CUDA;
  return cuda_status(
      launch_attn(*a, sparse, rows_max, ws, qmap, reinterpret_cast<cudaStream_t>(stream)));
}

int csa_sparse_attn_decode(const csa_attn_args* a, void* ws, size_t ws_bytes,
                           csa_stream_t stream) {
  return attn_common(a, 1, ws, ws_bytes, stream);
}

int hca_attn_decode(const csa_attn_args* a, void* ws, size_t ws_bytes, csa_stream_t stream) {
  return attn_common(a, 0, ws, ws_bytes, stream);
}

size_t csa_prefill_workspace_size(int32_t T, int64_t Nmax, int32_t H, int32_t k) {
  if (T < 0 || Nmax < 0 || H < 1 || k < 1) return 0;
  return prefill_ws_layout(T, Nmax, H, k, nullptr, nullptr);
}

int csa_prefill(const csa_prefill_args* a, void* ws, size_t ws_bytes, csa_stream_t stream_) {
  if (!a) return CSA_ERR_INVALID_ARG;
  if (a->P < 0 || a->T < 0 || a->m < 1 || a->m > 128 || a->P % a->m || a->Nmax < 128 ||
      a->Nmax % 128 || (a->P + a->T) / a->m > a->Nmax || !(a->eps >= 0.f) ||
      !(a->rope_base > 0.f) || !(a->tau >= 0.f) || (a->derotate != 0 && a->derotate != 1) ||
      (a->strict_eligibility != 0 && a->strict_eligibility != 1) || a->k < 1)
    return CSA_ERR_INVALID_ARG;
  if ((a->H != 64 && a->H != 128) || (a->H_I != 16 && a->H_I != 32 && a->H_I != 64) ||
      a->k > 2048 || a->P + a->T >= ((int64_t)1 << 31) || a->Nmax > ((int64_t)1 << 30))
    return CSA_ERR_UNSUPPORTED;
  if (a->T == 0) return CSA_OK;
  if (!ok_ptr(a->a) || !ok_ptr(a->b) || !ok_ptr(a->za) || !ok_ptr(a->zb) || !ok_ptr(a->bias) ||
      !ok_ptr(a->kv) || !ok_ptr(a->kv_scale) || !ok_ptr(a->q_fp4) || !ok_ptr(a->q_sf) ||
      !ok_ptr(a->w) || !ok_ptr(a->k_fp4) || !ok_ptr(a->k_sf) || !ok_ptr(a->q) ||
      !ok_ptr(a->sink) || !ok_ptr(a->out) || !ok_opt(a->norm_w) || !ok_opt(a->lse) ||
      !ok_opt(a->idx) || (a->dev_status && (reinterpret_cast<uintptr_t>(a->dev_status) & 3)) ||
      !ok_pages(a->pages, a->Nmax))
    return CSA_ERR_INVALID_ARG;
  if (a->P > 0 && (!ok_ptr(a->prev_b) || !ok_ptr(a->prev_zb) || !ok_ptr(a->swa_prefix)))
    return CSA_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255) ||
      ws_bytes < prefill_ws_layout(a->T, a->Nmax, a->H, a->k, nullptr, nullptr))
    return CSA_ERR_WORKSPACE;
  const int sms = num_sms();
  EncodeTiledFn enc = encode_fn();
  if (sms <= 0 || !enc) return CSA_ERR_CUDA;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  PrefillWs w;
  prefill_ws_layout(a->T, a->Nmax, a->H, a->k, reinterpret_cast<char*>(ws), &w);
  // a paged cache: the call runs on a contiguous staging copy (the prefix's rows, every
  // key), and the new entries go back to their pages at the end
  const bool paged = a->pages.block_table != nullptr;
  const PageMap pm = page_map(a->pages, a->Nmax);
  uint8_t* kv = paged ? w.kv_c : a->kv;
  float* kv_scale = paged ? w.sc_c : a->kv_scale;
  const uint8_t* k_fp4 = paged ? w.kf_c : a->k_fp4;
  const uint8_t* k_sf = paged ? w.ksf_c : a->k_sf;
  CUtensorMap kmap;  // encoded before the first launch, so a refusal leaves no partial work
  if (!encode_key_map(enc, &kmap, k_fp4, a->Nmax, 1)) return CSA_ERR_CUDA;
  if (paged &&
      launch_page_gather(pm, a->kv, a->kv_scale, a->k_fp4, a->k_sf, w.kv_c, w.sc_c, w.kf_c,
                         w.ksf_c, a->P / a->m, (a->P + a->T) / a->m, a->dev_status,
                         stream) != cudaSuccess)
    return CSA_ERR_CUDA;

  // 1. the new blocks' entries
  csa_compress_args c;
  std::memset(&c, 0, sizeof(c));
  c.B = 1;
  c.T = a->T;
  c.m = a->m;
  c.overlap = 1;
  c.pos0 = a->P;
  c.rope_base = a->rope_base;
  c.eps = a->eps;
  c.a = a->a;
  c.b = a->b;
  c.za = a->za;
  c.zb = a->zb;
  c.bias = a->bias;
  c.norm_w = a->norm_w;
  c.prev_b = a->prev_b;
  c.prev_zb = a->prev_zb;
  c.kv = kv;
  c.kv_scale = kv_scale;
  c.Nmax = a->Nmax;
  cudaError_t e = launch_compress(c, stream);
  if (e != cudaSuccess) return CSA_ERR_CUDA;
  // 2. per-query lengths, positions; FP16 rows of the entries and of the window in
  //    position order
  e = launch_prefill_prep(*a, w.rows16 + (size_t)a->Nmax * CSA_HEAD_DIM, w.n_all, w.pos_all,
                          stream);
  if (e != cudaSuccess) return CSA_ERR_CUDA;
  e = launch_prefill_rows16(kv, kv_scale, (a->P + a->T) / a->m, w.rows16, stream);
  if (e != cudaSuccess) return CSA_ERR_CUDA;
  // 3. per chunk of queries: indexer top-k over the shared keys, then attention
  for (int c0 = 0; c0 < a->T; c0 += kPrefillChunk) {
    const int nq = a->T - c0 < kPrefillChunk ? a->T - c0 : kPrefillChunk;
    int32_t* idx = a->idx ? a->idx + (size_t)c0 * a->k : w.idx;
    csa_topk_args t;
    std::memset(&t, 0, sizeof(t));
    t.B = nq;
    t.H_I = a->H_I;
    t.k = a->k;
    t.Nmax = a->Nmax;
    t.n_entries = w.n_all + c0;
    t.q_fp4 = a->q_fp4 + (size_t)c0 * a->H_I * 64;
    t.q_sf = a->q_sf + (size_t)c0 * a->H_I * 4;
    t.w = a->w + (size_t)c0 * a->H_I;
    t.k_fp4 = k_fp4;
    t.k_sf = k_sf;
    t.idx = idx;
    t.dev_status = a->dev_status;
    e = launch_prefill_indexer_topk(t, w.ix, sms, kmap, stream);
    if (e != cudaSuccess) return CSA_ERR_CUDA;
    csa_attn_args at;
    std::memset(&at, 0, sizeof(at));
    at.B = nq;
    at.H = a->H;
    at.k = a->k;
    at.Nmax = a->Nmax;
    at.q = a->q + (size_t)c0 * a->H * CSA_HEAD_DIM;
    at.pos = w.pos_all + c0;
    at.idx = idx;
    at.n_entries = w.n_all + c0;
    at.kv = kv;
    at.kv_scale = kv_scale;
    at.swa = nullptr;
    at.sink = a->sink;
    at.tau = a->tau;
    at.rope_base = a->rope_base;
    at.derotate = a->derotate;
    at.out = a->out + (size_t)c0 * a->H * CSA_HEAD_DIM;
    at.lse = a->lse ? a->lse + (size_t)c0 * a->H : nullptr;
    at.dev_status = a->dev_status;
    CUtensorMap qmap;
    if (!encode_q_map(enc, &qmap, at.q, (int64_t)nq * a->H, a->H)) return CSA_ERR_CUDA;
    e = launch_prefill_attn(at, w.rows16, a->P - (CSA_WINDOW - 1), qmap, stream);
    if (e != cudaSuccess) return CSA_ERR_CUDA;
  }
  if (paged &&
      launch_page_scatter(pm, w.kv_c, w.sc_c, a->kv, a->kv_scale, a->P / a->m,
                          (a->P + a->T) / a->m, a->dev_status, stream) != cudaSuccess)
    return CSA_ERR_CUDA;
  return CSA_OK;
}

static bool mma_peak_shape(int32_t kind, int32_t N, int32_t iters) {
  return ((kind == 0 && N == 64) || (kind == 1 && (N == 64 || N == 256))) && iters >= 1 &&
         iters <= 1000000;
}

int csa_mma_peak(int32_t kind, int32_t N, int32_t iters, int32_t* dev_status,
                 csa_stream_t stream) {
  if (!mma_peak_shape(kind, N, iters) ||
      (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3)))
    return CSA_ERR_INVALID_ARG;
  const int sms = num_sms();
  if (sms <= 0) return CSA_ERR_CUDA;
  return cuda_status(
      launch_mma_peak(kind, N, iters, sms, dev_status, reinterpret_cast<cudaStream_t>(stream)));
}

double csa_mma_peak_flops(int32_t kind, int32_t N, int32_t iters) {
  if (!mma_peak_shape(kind, N, iters)) return 0.0;
  const int sms = num_sms();
  return sms > 0 ? sms * mma_peak_flops_per_cta(kind, N, iters) : 0.0;
}

int csa_sparse_attn_decode_noalloc(const csa_attn_args* a, csa_stream_t stream) {
  // The ordinary checks first, with no workspace: they return before touching the device,
  // and anything other than the missing workspace is the answer.
  const int st = attn_common(a, 1, nullptr, 0, stream);
  if (st != CSA_ERR_WORKSPACE) return st;
  if (at_workspace_size(a->B, a->H, a->k + CSA_WINDOW) > CSA_NOALLOC_SCRATCH_BYTES)
    return CSA_ERR_UNSUPPORTED;
  void* ws = noalloc_scratch();
  if (!ws) return CSA_ERR_CUDA;
  return attn_common(a, 1, ws, CSA_NOALLOC_SCRATCH_BYTES, stream);
}

}  // extern "C"
