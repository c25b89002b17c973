// ksa_api.cu -- the C ABI of libksa (declared in include/ksa.h).
//
// Host-side argument validation, status codes and messages, TMA descriptor
// encoding, and the launches.  Nothing here allocates device memory or
// synchronises the host.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <map>
#include <mutex>
#include <string>
#include <tuple>

#include "../../include/ksa.h"
#include "ksa_internal.h"

namespace {

thread_local std::string g_last_error;

ksa_status fail(ksa_status st, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
ksa_status fail(ksa_status st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

ksa_status cuda_status(cudaError_t err, const char *what) {
  if (err == cudaSuccess) {
    g_last_error.clear();
    return KSA_OK;
  }
  return fail(KSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(err));
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

using ksa::device_sm_count;

ksa_status check_shape(const ksa_shape *s, bool need_block) {
  if (s == nullptr) return fail(KSA_ERR_INVALID_ARG, "shape is NULL");
  if (s->batch < 1 || s->num_q_heads < 1 || s->num_kv_heads < 1 || s->capacity < 1)
    return fail(KSA_ERR_INVALID_ARG, "batch, heads and capacity must be >= 1");
  if (s->num_q_heads % s->num_kv_heads != 0)
    return fail(KSA_ERR_INVALID_ARG, "num_q_heads (%d) is not a multiple of num_kv_heads (%d)",
                s->num_q_heads, s->num_kv_heads);
  if (s->head_dim != 64 && s->head_dim != 128)
    return fail(KSA_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", s->head_dim);
  if (need_block && s->block_size != 16 && s->block_size != 32 && s->block_size != 64)
    return fail(KSA_ERR_UNSUPPORTED, "block_size %d not supported (16, 32 or 64)",
                s->block_size);
  const long long rows = static_cast<long long>(s->batch) * s->num_kv_heads * s->capacity;
  if (rows >= (1LL << 31))
    return fail(KSA_ERR_UNSUPPORTED, "batch * num_kv_heads * capacity must be < 2^31");
  if (static_cast<long long>(s->batch) * s->num_q_heads * 8 >= (1LL << 31))
    return fail(KSA_ERR_UNSUPPORTED, "batch * num_q_heads too large");
  return KSA_OK;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

namespace ksa {

namespace {
constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];  // 0: not yet queried
std::mutex g_occ_mu;
// (device, kernel) -> largest dynamic shared-memory size enabled so far
std::map<std::tuple<int, const void *>, size_t> g_smem_enabled;
// (device, kernel, threads, smem) -> resident CTAs per SM
std::map<std::tuple<int, const void *, int, size_t>, int> g_occ;
}  // namespace

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < kMaxDevices) {
    const int n = g_sm_count[dev].load(std::memory_order_relaxed);
    if (n > 0) return n;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  if (dev >= 0 && dev < kMaxDevices) g_sm_count[dev].store(n, std::memory_order_relaxed);
  return n;
}

cudaError_t kernel_occupancy(const void *func, int threads, size_t smem, int *occ) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  std::lock_guard<std::mutex> lock(g_occ_mu);
  const auto key = std::make_tuple(dev, func, threads, smem);
  const auto hit = g_occ.find(key);
  if (hit != g_occ.end()) {
    *occ = hit->second;
    return cudaSuccess;
  }
  // the limit only ever grows, so every size seen before stays launchable
  size_t &enabled = g_smem_enabled[std::make_tuple(dev, func)];
  if (smem > enabled) {
    err = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    enabled = smem;
  }
  int n = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, func, threads, smem);
  if (err != cudaSuccess) return err;
  g_occ[key] = n;
  *occ = n;
  return cudaSuccess;
}

ksa_status set_last_error(ksa_status status, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return status;
}

bool encode_kv_tensor_map(CUtensorMap *map, const void *base, uint64_t rows, int D,
                          int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2u};
  const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estride[2] = {1u, 1u};
  const CUresult r =
      fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
         estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace ksa

extern "C" {

namespace {

// Validates the page pool of a paged cache and fills the kernels' layout.
ksa_status check_pages(const ksa_shape *shape, const ksa_pages *pages, ksa::KvLayout *kv) {
  if (pages == nullptr || pages->block_table == nullptr)
    return fail(KSA_ERR_INVALID_ARG, "pages and pages->block_table must be non-NULL");
  if (pages->max_blocks < 1 || pages->num_pages < 1)
    return fail(KSA_ERR_INVALID_ARG, "max_blocks and num_pages must be >= 1");
  if (static_cast<long long>(pages->max_blocks) * shape->block_size != shape->capacity)
    return fail(KSA_ERR_INVALID_ARG, "capacity %d must equal max_blocks * block_size (%d * %d)",
                shape->capacity, pages->max_blocks, shape->block_size);
  if (static_cast<long long>(pages->num_pages) * shape->num_kv_heads * shape->block_size >=
      (1LL << 31))
    return fail(KSA_ERR_UNSUPPORTED, "num_pages * num_kv_heads * block_size must be < 2^31");
  if (!aligned(pages->block_table, 4))
    return fail(KSA_ERR_INVALID_ARG, "block_table must be 4-byte aligned");
  kv->table = pages->block_table;
  kv->max_blocks = pages->max_blocks;
  kv->num_pages = pages->num_pages;
  kv->bs = shape->block_size;
  return KSA_OK;
}

ksa_status summaries_common(const ksa_shape *shape, const uint16_t *K, const ksa_pages *pages,
                            const int32_t *seq_lens, int32_t mode, int32_t summary_dtype,
                            void *summaries, uint32_t *dev_status, void *stream) {
  ksa_status st = check_shape(shape, true);
  if (st != KSA_OK) return st;
  if (K == nullptr || seq_lens == nullptr || summaries == nullptr)
    return fail(KSA_ERR_INVALID_ARG, "K, seq_lens and summaries must be non-NULL");
  if (mode != KSA_SUMMARY_ALL && mode != KSA_SUMMARY_LAST_BLOCK)
    return fail(KSA_ERR_INVALID_ARG, "mode %d is neither ALL nor LAST_BLOCK", mode);
  if (summary_dtype != KSA_SUMMARIES_F32 && summary_dtype != KSA_SUMMARIES_BF16 &&
      summary_dtype != KSA_SUMMARIES_FP8)
    return fail(KSA_ERR_INVALID_ARG, "summary_dtype %d is not F32, BF16 or FP8", summary_dtype);
  if (summary_dtype == KSA_SUMMARIES_FP8 && shape->head_dim != 128)
    return fail(KSA_ERR_UNSUPPORTED, "fp8 summaries need head_dim 128 (got %d)",
                shape->head_dim);
  if (!aligned(K, 16) || !aligned(summaries, 16) || !aligned(seq_lens, 4))
    return fail(KSA_ERR_INVALID_ARG, "K and summaries must be 16-byte aligned");
  ksa::SummaryArgs a;
  if (pages != nullptr && (st = check_pages(shape, pages, &a.kv)) != KSA_OK) return st;
  a.K = K;
  a.seq_lens = seq_lens;
  a.S = summaries;
  a.sfmt = summary_dtype;
  a.status = dev_status;
  a.B = shape->batch;
  a.Hkv = shape->num_kv_heads;
  a.T = shape->capacity;
  a.D = shape->head_dim;
  a.bs = shape->block_size;
  a.mode = mode;
  return cuda_status(ksa::launch_block_summaries(a, static_cast<cudaStream_t>(stream)),
                     "ksa_build_block_summaries launch");
}

}  // namespace

ksa_status ksa_build_block_summaries_ex(const ksa_shape *shape, const uint16_t *K,
                                        const int32_t *seq_lens, int32_t mode,
                                        int32_t summary_dtype, void *summaries,
                                        uint32_t *dev_status, void *stream) {
  return summaries_common(shape, K, nullptr, seq_lens, mode, summary_dtype, summaries,
                          dev_status, stream);
}

ksa_status ksa_build_block_summaries_paged(const ksa_shape *shape, const uint16_t *K_pages,
                                           const ksa_pages *pages, const int32_t *seq_lens,
                                           int32_t mode, int32_t summary_dtype, void *summaries,
                                           uint32_t *dev_status, void *stream) {
  if (pages == nullptr) return fail(KSA_ERR_INVALID_ARG, "pages must be non-NULL");
  return summaries_common(shape, K_pages, pages, seq_lens, mode, summary_dtype, summaries,
                          dev_status, stream);
}

namespace {

ksa_status append_common(const ksa_shape *shape, const uint16_t *k_new, const uint16_t *v_new,
                         uint16_t *K, uint16_t *V, const ksa_pages *pages,
                         const int32_t *seq_lens, uint32_t *dev_status, void *stream) {
  ksa_status st = check_shape(shape, pages != nullptr);
  if (st != KSA_OK) return st;
  if (k_new == nullptr || v_new == nullptr || K == nullptr || V == nullptr || seq_lens == nullptr)
    return fail(KSA_ERR_INVALID_ARG, "k_new, v_new, K, V and seq_lens must be non-NULL");
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(K, 16) || !aligned(V, 16) ||
      !aligned(seq_lens, 4))
    return fail(KSA_ERR_INVALID_ARG, "k_new, v_new, K and V must be 16-byte aligned");
  ksa::AppendArgs a;
  if (pages != nullptr && (st = check_pages(shape, pages, &a.kv)) != KSA_OK) return st;
  a.k_new = k_new;
  a.v_new = v_new;
  a.K = K;
  a.V = V;
  a.seq_lens = seq_lens;
  a.status = dev_status;
  a.B = shape->batch;
  a.Hkv = shape->num_kv_heads;
  a.T = shape->capacity;
  a.D = shape->head_dim;
  return cuda_status(ksa::launch_append_kv(a, static_cast<cudaStream_t>(stream)),
                     "ksa_append_kv launch");
}

}  // namespace

ksa_status ksa_append_kv(const ksa_shape *shape, const uint16_t *k_new, const uint16_t *v_new,
                         uint16_t *K, uint16_t *V, const int32_t *seq_lens, uint32_t *dev_status,
                         void *stream) {
  return append_common(shape, k_new, v_new, K, V, nullptr, seq_lens, dev_status, stream);
}

ksa_status ksa_append_kv_paged(const ksa_shape *shape, const uint16_t *k_new,
                               const uint16_t *v_new, uint16_t *K_pages, uint16_t *V_pages,
                               const ksa_pages *pages, const int32_t *seq_lens,
                               uint32_t *dev_status, void *stream) {
  if (pages == nullptr) return fail(KSA_ERR_INVALID_ARG, "pages must be non-NULL");
  return append_common(shape, k_new, v_new, K_pages, V_pages, pages, seq_lens, dev_status,
                       stream);
}

ksa_status ksa_build_block_summaries(const ksa_shape *shape, const uint16_t *K,
                                     const int32_t *seq_lens, int32_t mode, float *summaries,
                                     uint32_t *dev_status, void *stream) {
  return ksa_build_block_summaries_ex(shape, K, seq_lens, mode, KSA_SUMMARIES_F32, summaries,
                                      dev_status, stream);
}

size_t ksa_select_blocks_workspace(const ksa_shape *shape, int32_t k_blocks) {
  (void)k_blocks;
  if (check_shape(shape, true) != KSA_OK) return 0;
  return ksa::select_workspace_bytes(shape->batch, shape->num_kv_heads, shape->capacity,
                                     shape->block_size);
}

namespace {

// Validates a selection call's arguments (not its workspace) and fills *a.
ksa_status select_args(const ksa_shape *shape, const uint16_t *q, const ksa_pages *pages,
                       void *summaries, int32_t summary_dtype, const int32_t *seq_lens,
                       int32_t k_blocks, int32_t *block_idx, int32_t *num_sel,
                       uint32_t *dev_status, ksa::SelectArgs *a) {
  ksa_status st = check_shape(shape, true);
  if (st != KSA_OK) return st;
  if (q == nullptr || summaries == nullptr || seq_lens == nullptr || block_idx == nullptr ||
      num_sel == nullptr)
    return fail(KSA_ERR_INVALID_ARG, "q, summaries, seq_lens, block_idx, num_sel must be non-NULL");
  if (summary_dtype != KSA_SUMMARIES_F32 && summary_dtype != KSA_SUMMARIES_BF16 &&
      summary_dtype != KSA_SUMMARIES_FP8)
    return fail(KSA_ERR_INVALID_ARG, "summary_dtype %d is not F32, BF16 or FP8", summary_dtype);
  if (summary_dtype == KSA_SUMMARIES_FP8 && shape->head_dim != 128)
    return fail(KSA_ERR_UNSUPPORTED, "fp8 summaries need head_dim 128 (got %d)",
                shape->head_dim);
  if (k_blocks < 1) return fail(KSA_ERR_INVALID_ARG, "k_blocks must be >= 1 (got %d)", k_blocks);
  const int nb_max = (shape->capacity + shape->block_size - 1) / shape->block_size;
  if (nb_max > 16384)
    return fail(KSA_ERR_UNSUPPORTED, "ceil(capacity/block_size) = %d exceeds 16384", nb_max);
  if (!aligned(summaries, 16) || !aligned(q, 4))
    return fail(KSA_ERR_INVALID_ARG, "summaries must be 16-byte aligned");
  if (pages != nullptr && (st = check_pages(shape, pages, &a->kv)) != KSA_OK) return st;
  a->q = q;
  a->S = summaries;  // written only when K is given (the fused refresh)
  a->sfmt = summary_dtype;
  a->seq_lens = seq_lens;
  a->block_idx = block_idx;
  a->num_sel = num_sel;
  a->status = dev_status;
  a->B = shape->batch;
  a->Hq = shape->num_q_heads;
  a->Hkv = shape->num_kv_heads;
  a->D = shape->head_dim;
  a->T = shape->capacity;
  a->bs = shape->block_size;
  a->k = k_blocks;
  return KSA_OK;
}

// Shared by the selection entry points; K non-NULL fuses the last-block refresh.
ksa_status select_common(const ksa_shape *shape, const uint16_t *q, const uint16_t *K,
                         const ksa_pages *pages, void *summaries, int32_t summary_dtype,
                         const int32_t *seq_lens,
                         int32_t k_blocks, int32_t *block_idx, int32_t *num_sel, void *ws,
                         size_t ws_bytes, uint32_t *dev_status, void *stream, const char *what) {
  ksa::SelectArgs a;
  ksa_status st = select_args(shape, q, pages, summaries, summary_dtype, seq_lens, k_blocks,
                              block_idx, num_sel, dev_status, &a);
  if (st != KSA_OK) return st;
  const size_t need = ksa::select_workspace_bytes(shape->batch, shape->num_kv_heads,
                                                  shape->capacity, shape->block_size);
  if (ws == nullptr || ws_bytes < need)
    return fail(KSA_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", need, ws_bytes);
  if (!aligned(ws, 256)) return fail(KSA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  return cuda_status(
      ksa::launch_select_blocks(a, K, ws, device_sm_count(), static_cast<cudaStream_t>(stream)),
      what);
}

}  // namespace

ksa_status ksa_select_blocks_ex(const ksa_shape *shape, const uint16_t *q, const void *summaries,
                                int32_t summary_dtype, const int32_t *seq_lens, int32_t k_blocks,
                                int32_t *block_idx, int32_t *num_sel, void *ws, size_t ws_bytes,
                                uint32_t *dev_status, void *stream) {
  // read only: no K is given, so nothing is refreshed
  return select_common(shape, q, nullptr, nullptr, const_cast<void *>(summaries), summary_dtype,
                       seq_lens,
                       k_blocks, block_idx, num_sel, ws, ws_bytes, dev_status, stream,
                       "ksa_select_blocks launch");
}

ksa_status ksa_select_blocks(const ksa_shape *shape, const uint16_t *q, const float *summaries,
                             const int32_t *seq_lens, int32_t k_blocks, int32_t *block_idx,
                             int32_t *num_sel, void *ws, size_t ws_bytes, uint32_t *dev_status,
                             void *stream) {
  return ksa_select_blocks_ex(shape, q, summaries, KSA_SUMMARIES_F32, seq_lens, k_blocks,
                              block_idx, num_sel, ws, ws_bytes, dev_status, stream);
}

ksa_status ksa_decode_select_blocks_ex(const ksa_shape *shape, const uint16_t *q,
                                       const uint16_t *K, void *summaries, int32_t summary_dtype,
                                       const int32_t *seq_lens, int32_t k_blocks,
                                       int32_t *block_idx, int32_t *num_sel, void *ws,
                                       size_t ws_bytes, uint32_t *dev_status, void *stream) {
  if (K == nullptr) return fail(KSA_ERR_INVALID_ARG, "K must be non-NULL");
  if (!aligned(K, 16)) return fail(KSA_ERR_INVALID_ARG, "K must be 16-byte aligned");
  return select_common(shape, q, K, nullptr, summaries, summary_dtype, seq_lens, k_blocks,
                       block_idx, num_sel, ws, ws_bytes, dev_status, stream,
                       "ksa_decode_select_blocks launch");
}

ksa_status ksa_select_window(const ksa_shape *shape, const int32_t *seq_lens, int32_t k_blocks,
                             int32_t *block_idx, int32_t *num_sel, uint32_t *dev_status,
                             void *stream) {
  ksa_status st = check_shape(shape, true);
  if (st != KSA_OK) return st;
  if (seq_lens == nullptr || block_idx == nullptr || num_sel == nullptr)
    return fail(KSA_ERR_INVALID_ARG, "seq_lens, block_idx and num_sel must be non-NULL");
  if (k_blocks < 1) return fail(KSA_ERR_INVALID_ARG, "k_blocks must be >= 1 (got %d)", k_blocks);
  if (static_cast<long long>(shape->batch) * shape->num_kv_heads * k_blocks >= (1LL << 31))
    return fail(KSA_ERR_UNSUPPORTED, "batch * num_kv_heads * k_blocks must be < 2^31");
  ksa::SelectArgs a;
  a.q = nullptr;
  a.S = nullptr;
  a.sfmt = KSA_SUMMARIES_F32;
  a.seq_lens = seq_lens;
  a.block_idx = block_idx;
  a.num_sel = num_sel;
  a.status = dev_status;
  a.B = shape->batch;
  a.Hq = shape->num_q_heads;
  a.Hkv = shape->num_kv_heads;
  a.D = shape->head_dim;
  a.T = shape->capacity;
  a.bs = shape->block_size;
  a.k = k_blocks;
  return cuda_status(ksa::launch_select_window(a, static_cast<cudaStream_t>(stream)),
                     "ksa_select_window launch");
}

ksa_status ksa_decode_select_blocks_paged(const ksa_shape *shape, const uint16_t *q,
                                          const uint16_t *K_pages, const ksa_pages *pages,
                                          void *summaries, int32_t summary_dtype,
                                          const int32_t *seq_lens, int32_t k_blocks,
                                          int32_t *block_idx, int32_t *num_sel, void *ws,
                                          size_t ws_bytes, uint32_t *dev_status, void *stream) {
  if (K_pages == nullptr || pages == nullptr)
    return fail(KSA_ERR_INVALID_ARG, "K_pages and pages must be non-NULL");
  if (!aligned(K_pages, 16)) return fail(KSA_ERR_INVALID_ARG, "K_pages must be 16-byte aligned");
  return select_common(shape, q, K_pages, pages, summaries, summary_dtype, seq_lens, k_blocks,
                       block_idx, num_sel, ws, ws_bytes, dev_status, stream,
                       "ksa_decode_select_blocks_paged launch");
}

ksa_status ksa_decode_select_blocks(const ksa_shape *shape, const uint16_t *q, const uint16_t *K,
                                    float *summaries, const int32_t *seq_lens, int32_t k_blocks,
                                    int32_t *block_idx, int32_t *num_sel, void *ws,
                                    size_t ws_bytes, uint32_t *dev_status, void *stream) {
  return ksa_decode_select_blocks_ex(shape, q, K, summaries, KSA_SUMMARIES_F32, seq_lens,
                                     k_blocks, block_idx, num_sel, ws, ws_bytes, dev_status,
                                     stream);
}

size_t ksa_sparse_decode_attn_workspace(const ksa_shape *shape, int32_t idx_capacity,
                                        int32_t tokens_per_idx) {
  (void)idx_capacity;
  (void)tokens_per_idx;
  if (check_shape(shape, false) != KSA_OK) return 0;
  return ksa::attn_workspace_bytes(shape->batch, shape->num_q_heads, shape->num_kv_heads,
                                   shape->head_dim, device_sm_count());
}

namespace {

// Validates an attention call's arguments (not its workspace) and fills *a.
ksa_status attn_args(const ksa_shape *shape, const uint16_t *q, const uint16_t *K,
                     const uint16_t *V, const ksa_pages *pages, const int32_t *seq_lens,
                     const int32_t *idx, const int32_t *num_idx, int32_t idx_capacity,
                     int32_t tokens_per_idx, int32_t idx_shared, float scale, int32_t out_dtype,
                     void *out, float *lse, uint32_t *dev_status, ksa::AttnArgs *a) {
  ksa_status st = check_shape(shape, pages != nullptr);
  if (st != KSA_OK) return st;
  if (q == nullptr || K == nullptr || V == nullptr || seq_lens == nullptr || out == nullptr)
    return fail(KSA_ERR_INVALID_ARG, "q, K, V, seq_lens and out must be non-NULL");
  const int G = shape->num_q_heads / shape->num_kv_heads;
  if (G > 8)
    return fail(KSA_ERR_UNSUPPORTED, "query heads per kv-head = %d exceeds 8", G);
  if (out_dtype != KSA_OUT_F32 && out_dtype != KSA_OUT_BF16)
    return fail(KSA_ERR_INVALID_ARG, "out_dtype %d is neither F32 nor BF16", out_dtype);
  if (!(scale >= 0.f) || isinf(scale))
    return fail(KSA_ERR_INVALID_ARG, "scale must be finite and >= 0");
  if (idx != nullptr) {
    if (num_idx == nullptr) return fail(KSA_ERR_INVALID_ARG, "num_idx is NULL with idx given");
    if (idx_capacity < 1) return fail(KSA_ERR_INVALID_ARG, "idx_capacity must be >= 1");
    if (tokens_per_idx < 1 || tokens_per_idx > 256 ||
        (tokens_per_idx & (tokens_per_idx - 1)) != 0)
      return fail(KSA_ERR_UNSUPPORTED, "tokens_per_idx %d is not a power of two in [1, 256]",
                  tokens_per_idx);
    if (idx_shared != KSA_IDX_PER_KV_HEAD && idx_shared != KSA_IDX_SHARED &&
        idx_shared != KSA_IDX_PER_Q_HEAD)
      return fail(KSA_ERR_INVALID_ARG, "idx_shared must be 0, 1 or 2");
    if (!aligned(idx, 4) || !aligned(num_idx, 4))
      return fail(KSA_ERR_INVALID_ARG, "idx and num_idx must be 4-byte aligned");
  }
  if (!aligned(K, 16) || !aligned(V, 16) || !aligned(q, 4) ||
      !aligned(out, out_dtype == KSA_OUT_F32 ? 4 : 2) || (lse && !aligned(lse, 4)))
    return fail(KSA_ERR_INVALID_ARG, "K and V must be 16-byte aligned, q and out element-aligned");
  if (pages != nullptr && (st = check_pages(shape, pages, &a->kv)) != KSA_OK) return st;
  a->q = q;
  a->K = K;
  a->V = V;
  a->seq_lens = seq_lens;
  a->idx = idx;
  a->num_idx = num_idx;
  a->out_f32 = out_dtype == KSA_OUT_F32 ? static_cast<float *>(out) : nullptr;
  a->out_bf16 = out_dtype == KSA_OUT_BF16 ? static_cast<uint16_t *>(out) : nullptr;
  a->lse = lse;
  a->status = dev_status;
  a->B = shape->batch;
  a->Hq = shape->num_q_heads;
  a->Hkv = shape->num_kv_heads;
  a->D = shape->head_dim;
  a->T = shape->capacity;
  a->cap = idx ? idx_capacity : 0;
  a->tpi = idx ? tokens_per_idx : 1;
  a->shared = idx ? idx_shared : 0;
  a->scale = scale == 0.f ? static_cast<float>(1.0 / sqrt(static_cast<double>(shape->head_dim)))
                          : scale;
  return KSA_OK;
}

ksa_status attn_common(const ksa_shape *shape, const uint16_t *q, const uint16_t *K,
                       const uint16_t *V, const ksa_pages *pages, const int32_t *seq_lens,
                       const int32_t *idx, const int32_t *num_idx, int32_t idx_capacity,
                       int32_t tokens_per_idx, int32_t idx_shared, float scale, int32_t out_dtype,
                       void *out, float *lse, void *ws, size_t ws_bytes, uint32_t *dev_status,
                       void *stream) {
  ksa::AttnArgs a;
  const ksa_status st = attn_args(shape, q, K, V, pages, seq_lens, idx, num_idx, idx_capacity,
                                  tokens_per_idx, idx_shared, scale, out_dtype, out, lse,
                                  dev_status, &a);
  if (st != KSA_OK) return st;
  const int sms = device_sm_count();
  const size_t need = ksa::attn_workspace_bytes(shape->batch, shape->num_q_heads,
                                                shape->num_kv_heads, shape->head_dim, sms);
  if (ws == nullptr || ws_bytes < need)
    return fail(KSA_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", need, ws_bytes);
  if (!aligned(ws, 256)) return fail(KSA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  return cuda_status(
      ksa::launch_sparse_decode_attn(a, ws, sms, static_cast<cudaStream_t>(stream)),
      "ksa_sparse_decode_attn launch");
}

}  // namespace

ksa_status ksa_sparse_decode_attn(const ksa_shape *shape, const uint16_t *q, const uint16_t *K,
                                  const uint16_t *V, const int32_t *seq_lens, const int32_t *idx,
                                  const int32_t *num_idx, int32_t idx_capacity,
                                  int32_t tokens_per_idx, int32_t idx_shared, float scale,
                                  int32_t out_dtype, void *out, float *lse, void *ws,
                                  size_t ws_bytes, uint32_t *dev_status, void *stream) {
  return attn_common(shape, q, K, V, nullptr, seq_lens, idx, num_idx, idx_capacity,
                     tokens_per_idx, idx_shared, scale, out_dtype, out, lse, ws, ws_bytes,
                     dev_status, stream);
}

ksa_status ksa_sparse_decode_attn_paged(const ksa_shape *shape, const uint16_t *q,
                                        const uint16_t *K_pages, const uint16_t *V_pages,
                                        const ksa_pages *pages, const int32_t *seq_lens,
                                        const int32_t *idx, const int32_t *num_idx,
                                        int32_t idx_capacity, int32_t tokens_per_idx,
                                        int32_t idx_shared, float scale, int32_t out_dtype,
                                        void *out, float *lse, void *ws, size_t ws_bytes,
                                        uint32_t *dev_status, void *stream) {
  if (pages == nullptr) return fail(KSA_ERR_INVALID_ARG, "pages must be non-NULL");
  return attn_common(shape, q, K_pages, V_pages, pages, seq_lens, idx, num_idx, idx_capacity,
                     tokens_per_idx, idx_shared, scale, out_dtype, out, lse, ws, ws_bytes,
                     dev_status, stream);
}

size_t ksa_decode_step_workspace(const ksa_shape *shape, int32_t k_blocks) {
  (void)k_blocks;
  if (check_shape(shape, true) != KSA_OK) return 0;
  return ksa::decode_step_workspace_bytes(shape->batch, shape->num_q_heads, shape->num_kv_heads,
                                          shape->head_dim, shape->capacity, shape->block_size,
                                          device_sm_count());
}

ksa_status ksa_decode_step(const ksa_shape *shape, const uint16_t *q, const uint16_t *K,
                           const uint16_t *V, void *summaries, int32_t summary_dtype,
                           const int32_t *seq_lens, int32_t k_blocks, int32_t *block_idx,
                           int32_t *num_sel, float scale, int32_t out_dtype, void *out,
                           float *lse, void *ws, size_t ws_bytes, uint32_t *dev_status,
                           void *stream) {
  if (K == nullptr) return fail(KSA_ERR_INVALID_ARG, "K must be non-NULL");
  ksa::SelectArgs sa;
  ksa_status st = select_args(shape, q, nullptr, summaries, summary_dtype, seq_lens, k_blocks,
                              block_idx, num_sel, dev_status, &sa);
  if (st != KSA_OK) return st;
  ksa::AttnArgs aa;
  st = attn_args(shape, q, K, V, nullptr, seq_lens, block_idx, num_sel, k_blocks,
                 shape->block_size, KSA_IDX_PER_KV_HEAD, scale, out_dtype, out, lse, dev_status,
                 &aa);
  if (st != KSA_OK) return st;
  const int sms = device_sm_count();
  const size_t need = ksa::decode_step_workspace_bytes(
      shape->batch, shape->num_q_heads, shape->num_kv_heads, shape->head_dim, shape->capacity,
      shape->block_size, sms);
  if (ws == nullptr || ws_bytes < need)
    return fail(KSA_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", need, ws_bytes);
  if (!aligned(ws, 256)) return fail(KSA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  return cuda_status(
      ksa::launch_decode_step(sa, K, aa, ws, sms, static_cast<cudaStream_t>(stream)),
      "ksa_decode_step launch");
}

size_t ksa_unified_select_workspace(const ksa_shape *shape, int32_t per_head_topk,
                                    int32_t token_budget) {
  (void)per_head_topk;
  (void)token_budget;
  if (shape == nullptr || shape->batch < 1 || shape->num_q_heads < 1 || shape->capacity < 1)
    return 0;
  return ksa::unified_workspace_bytes(shape->batch, shape->num_q_heads, shape->capacity);
}

ksa_status ksa_unified_select(const ksa_shape *shape, const uint16_t *q, const uint16_t *K,
                              const int32_t *seq_lens, int32_t per_head_topk,
                              int32_t token_budget, int32_t recent_tokens, int32_t *token_idx,
                              int32_t *num_sel, void *ws, size_t ws_bytes, uint32_t *dev_status,
                              void *stream) {
  ksa_status st = check_shape(shape, false);
  if (st != KSA_OK) return st;
  if (q == nullptr || K == nullptr || seq_lens == nullptr || token_idx == nullptr ||
      num_sel == nullptr)
    return fail(KSA_ERR_INVALID_ARG, "q, K, seq_lens, token_idx and num_sel must be non-NULL");
  const int G = shape->num_q_heads / shape->num_kv_heads;
  if (G > 8) return fail(KSA_ERR_UNSUPPORTED, "query heads per kv-head = %d exceeds 8", G);
  if (shape->num_q_heads > 65535)
    return fail(KSA_ERR_UNSUPPORTED, "num_q_heads above 65535 (vote counts are 16-bit)");
  if (shape->capacity > 65536)
    return fail(KSA_ERR_UNSUPPORTED, "capacity %d exceeds 65536", shape->capacity);
  if (per_head_topk < 1) return fail(KSA_ERR_INVALID_ARG, "per_head_topk must be >= 1");
  if (token_budget < 1 || token_budget > shape->capacity)
    return fail(KSA_ERR_INVALID_ARG, "token_budget must be in [1, capacity]");
  if (recent_tokens < 0) recent_tokens = token_budget / 4;
  if (recent_tokens > token_budget)
    return fail(KSA_ERR_INVALID_ARG, "recent_tokens (%d) exceeds token_budget (%d)",
                recent_tokens, token_budget);
  const size_t need =
      ksa::unified_workspace_bytes(shape->batch, shape->num_q_heads, shape->capacity);
  if (ws == nullptr || ws_bytes < need)
    return fail(KSA_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", need, ws_bytes);
  if (!aligned(ws, 256)) return fail(KSA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (!aligned(K, 16) || !aligned(q, 4))
    return fail(KSA_ERR_INVALID_ARG, "K must be 16-byte aligned");
  ksa::UnifiedArgs a;
  a.q = q;
  a.K = K;
  a.seq_lens = seq_lens;
  a.token_idx = token_idx;
  a.num_sel = num_sel;
  const size_t keys_bytes =
      (static_cast<size_t>(shape->batch) * shape->num_q_heads * shape->capacity * 4 + 255) &
      ~static_cast<size_t>(255);
  a.keys = static_cast<uint32_t *>(ws);
  a.votes = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + keys_bytes);
  const size_t votes_bytes =
      (static_cast<size_t>(shape->batch) * shape->capacity * 4 + 255) & ~static_cast<size_t>(255);
  a.bits = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) + keys_bytes + votes_bytes);
  a.status = dev_status;
  a.B = shape->batch;
  a.Hq = shape->num_q_heads;
  a.Hkv = shape->num_kv_heads;
  a.D = shape->head_dim;
  a.T = shape->capacity;
  a.P = per_head_topk;
  a.budget = token_budget;
  a.R = recent_tokens;
  return cuda_status(
      ksa::launch_unified_select(a, device_sm_count(), static_cast<cudaStream_t>(stream)),
      "ksa_unified_select launch");
}

size_t ksa_select_tokens_per_head_workspace(const ksa_shape *shape, int32_t k_tokens) {
  (void)k_tokens;
  if (shape == nullptr || shape->batch < 1 || shape->num_q_heads < 1 || shape->capacity < 1)
    return 0;
  return ksa::unified_workspace_bytes(shape->batch, shape->num_q_heads, shape->capacity);
}

ksa_status ksa_select_tokens_per_head(const ksa_shape *shape, const uint16_t *q,
                                      const uint16_t *K, const int32_t *seq_lens,
                                      int32_t k_tokens, int32_t *token_idx, int32_t *num_sel,
                                      void *ws, size_t ws_bytes, uint32_t *dev_status,
                                      void *stream) {
  ksa_status st = check_shape(shape, false);
  if (st != KSA_OK) return st;
  if (q == nullptr || K == nullptr || seq_lens == nullptr || token_idx == nullptr ||
      num_sel == nullptr)
    return fail(KSA_ERR_INVALID_ARG, "q, K, seq_lens, token_idx and num_sel must be non-NULL");
  const int G = shape->num_q_heads / shape->num_kv_heads;
  if (G > 8) return fail(KSA_ERR_UNSUPPORTED, "query heads per kv-head = %d exceeds 8", G);
  if (shape->capacity > 65536)
    return fail(KSA_ERR_UNSUPPORTED, "capacity %d exceeds 65536", shape->capacity);
  if (k_tokens < 1) return fail(KSA_ERR_INVALID_ARG, "k_tokens must be >= 1");
  const size_t need =
      ksa::unified_workspace_bytes(shape->batch, shape->num_q_heads, shape->capacity);
  if (ws == nullptr || ws_bytes < need)
    return fail(KSA_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", need, ws_bytes);
  if (!aligned(ws, 256)) return fail(KSA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (!aligned(K, 16) || !aligned(q, 4))
    return fail(KSA_ERR_INVALID_ARG, "K must be 16-byte aligned");
  ksa::UnifiedArgs a;
  a.q = q;
  a.K = K;
  a.seq_lens = seq_lens;
  a.token_idx = token_idx;
  a.num_sel = num_sel;
  const size_t keys_bytes =
      (static_cast<size_t>(shape->batch) * shape->num_q_heads * shape->capacity * 4 + 255) &
      ~static_cast<size_t>(255);
  a.keys = static_cast<uint32_t *>(ws);
  a.votes = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + keys_bytes);
  a.bits = nullptr;
  a.status = dev_status;
  a.B = shape->batch;
  a.Hq = shape->num_q_heads;
  a.Hkv = shape->num_kv_heads;
  a.D = shape->head_dim;
  a.T = shape->capacity;
  a.P = k_tokens;
  a.budget = k_tokens;  // rows with L <= k keep every token and need no scores
  a.R = 0;
  return cuda_status(ksa::launch_tokens_per_head(a, static_cast<cudaStream_t>(stream)),
                     "ksa_select_tokens_per_head launch");
}

// Random-head aggregation's workspace: the per-head workspace, then every head's lists
// [B, Hq, k] and counts [B, Hq].
size_t ksa_select_tokens_one_head_workspace(const ksa_shape *shape, int32_t k_tokens) {
  if (shape == nullptr || shape->batch < 1 || shape->num_q_heads < 1 || shape->capacity < 1 ||
      k_tokens < 1)
    return 0;
  const size_t heads = static_cast<size_t>(shape->batch) * shape->num_q_heads;
  return ksa::unified_workspace_bytes(shape->batch, shape->num_q_heads, shape->capacity) +
         ((heads * k_tokens * sizeof(int32_t) + 255) & ~static_cast<size_t>(255)) +
         ((heads * sizeof(int32_t) + 255) & ~static_cast<size_t>(255)) +
         ((static_cast<size_t>(shape->batch) * sizeof(int32_t) + 255) & ~static_cast<size_t>(255));
}

ksa_status ksa_select_tokens_one_head(const ksa_shape *shape, const uint16_t *q,
                                      const uint16_t *K, const int32_t *seq_lens,
                                      const int32_t *head_of_row, int32_t k_tokens,
                                      int32_t *token_idx, int32_t *num_sel, void *ws,
                                      size_t ws_bytes, uint32_t *dev_status, void *stream) {
  ksa_status st = check_shape(shape, false);
  if (st != KSA_OK) return st;
  if (head_of_row == nullptr || token_idx == nullptr || num_sel == nullptr)
    return fail(KSA_ERR_INVALID_ARG, "head_of_row, token_idx and num_sel must be non-NULL");
  if (k_tokens < 1) return fail(KSA_ERR_INVALID_ARG, "k_tokens must be >= 1");
  const int B = shape->batch, Hq = shape->num_q_heads;
  for (int b = 0; b < B; ++b) {  // the host array holds one head per row
    if (head_of_row[b] < 0 || head_of_row[b] >= Hq)
      return fail(KSA_ERR_INVALID_ARG, "head_of_row[%d] = %d is outside [0, %d)", b,
                  head_of_row[b], Hq);
  }
  const size_t base = ksa::unified_workspace_bytes(B, Hq, shape->capacity);
  const size_t heads = static_cast<size_t>(B) * Hq;
  const size_t lists_bytes =
      (heads * k_tokens * sizeof(int32_t) + 255) & ~static_cast<size_t>(255);
  const size_t need = ksa_select_tokens_one_head_workspace(shape, k_tokens);
  if (ws == nullptr || ws_bytes < need)
    return fail(KSA_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", need, ws_bytes);
  if (!aligned(ws, 256)) return fail(KSA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  int32_t *lists = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + base);
  int32_t *counts = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + base + lists_bytes);
  const size_t counts_bytes = (heads * sizeof(int32_t) + 255) & ~static_cast<size_t>(255);
  int32_t *dev_heads = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + base +
                                                   lists_bytes + counts_bytes);
  // every head's own set into the workspace (the per-head kernels) ...
  st = ksa_select_tokens_per_head(shape, q, K, seq_lens, k_tokens, lists, counts, ws, base,
                                  dev_status, stream);
  if (st != KSA_OK) return st;
  // ... then the heads drawn for the rows (one copy; the host array is read before the
  // copy call returns) and each row's chosen list and count (one gather launch)
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t err = cudaMemcpyAsync(dev_heads, head_of_row, static_cast<size_t>(B) * sizeof(int32_t),
                                    cudaMemcpyHostToDevice, s);
  if (err != cudaSuccess) return cuda_status(err, "ksa_select_tokens_one_head heads copy");
  err = ksa::launch_gather_head_lists(lists, counts, dev_heads, B, Hq, k_tokens, token_idx,
                                      num_sel, s);
  if (err != cudaSuccess) return cuda_status(err, "ksa_select_tokens_one_head gather");
  return KSA_OK;
}

ksa_status ksa_get_device_status(const uint32_t *dev_status, void *stream, int32_t clear,
                                 uint32_t *flags) {
  if (dev_status == nullptr || flags == nullptr)
    return fail(KSA_ERR_INVALID_ARG, "dev_status and flags must be non-NULL");
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t word = 0u;
  cudaError_t err = cudaMemcpyAsync(&word, dev_status, sizeof word, cudaMemcpyDeviceToHost, s);
  if (err == cudaSuccess) err = cudaStreamSynchronize(s);
  if (err != cudaSuccess) return cuda_status(err, "reading the device status word");
  *flags = word;
  if (clear != 0) {
    err = cudaMemsetAsync(const_cast<uint32_t *>(dev_status), 0, sizeof(uint32_t), s);
    if (err != cudaSuccess) return cuda_status(err, "clearing the device status word");
  }
  return KSA_OK;
}

const char *ksa_status_string(ksa_status status) {
  switch (status) {
    case KSA_OK: return "KSA_OK";
    case KSA_ERR_INVALID_ARG: return "KSA_ERR_INVALID_ARG";
    case KSA_ERR_UNSUPPORTED: return "KSA_ERR_UNSUPPORTED";
    case KSA_ERR_WORKSPACE: return "KSA_ERR_WORKSPACE";
    case KSA_ERR_CUDA: return "KSA_ERR_CUDA";
  }
  return "KSA_UNKNOWN_STATUS";
}

const char *ksa_last_error(void) { return g_last_error.c_str(); }

int32_t ksa_version(void) { return 100; }

}  // extern "C"
