// ksa_internal.h -- launch entry points of the libksa kernels (host side).
//
// Every launcher assumes its arguments were validated by the C ABI layer
// (ksa_api.cu) and returns the cudaError_t of its launch.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ksa.h"

namespace ksa {

// Where the K/V rows of (row b, kv-head g, token t) live: a contiguous cache
// [B, Hkv, T, D] (table == nullptr), or a paged one [num_pages, Hkv, bs, D]
// whose block_table [B, max_blocks] names the page of logical block t / bs.
struct KvLayout {
  const int32_t *table = nullptr;
  int max_blocks = 0;
  int num_pages = 0;
  int bs = 0;
};

#ifdef __CUDACC__
// Row (in units of D elements) holding token t of (b, g); -1 when the block's
// page id is outside [0, num_pages) (nothing may be read for it).
__device__ __forceinline__ long long kv_row(const KvLayout &kv, int b, int g, int Hkv, int T,
                                            long long t) {
  if (kv.table == nullptr) return (static_cast<long long>(b) * Hkv + g) * T + t;
  const int page = __ldg(kv.table + static_cast<size_t>(b) * kv.max_blocks + t / kv.bs);
  if (page < 0 || page >= kv.num_pages) return -1;
  return (static_cast<long long>(page) * Hkv + g) * kv.bs + t % kv.bs;
}
#endif

struct SummaryArgs {
  const uint16_t *K;
  const int32_t *seq_lens;
  void *S;   // [B, Hkv, ceil(T/bs), D] fp32 / bf16 / fp8 values (+ fp8 scales)
  int sfmt;  // storage: KSA_SUMMARIES_F32, _BF16 or _FP8
  uint32_t *status;
  int B, Hkv, T, D, bs, mode;
  KvLayout kv;
};
cudaError_t launch_block_summaries(const SummaryArgs &a, cudaStream_t stream);

// The decode step's cache write: the new token's key and value rows of every
// (b, g) go to token slot L_b - 1 (seq_lens counts the new token).
struct AppendArgs {
  const uint16_t *k_new, *v_new;  // [B, Hkv, D]
  uint16_t *K, *V;                // caches (contiguous or paged, per kv)
  const int32_t *seq_lens;
  uint32_t *status;
  int B, Hkv, T, D;
  KvLayout kv;
};
cudaError_t launch_append_kv(const AppendArgs &a, cudaStream_t stream);

struct SelectArgs {
  const uint16_t *q;
  void *S;   // fp32 / bf16 / fp8; read; written only by the fused last-block refresh
  int sfmt;  // storage: KSA_SUMMARIES_F32, _BF16 or _FP8
  const int32_t *seq_lens;
  int32_t *block_idx;
  int32_t *num_sel;
  uint32_t *status;
  int B, Hq, Hkv, D, T, bs, k;
  KvLayout kv;  // of the key cache given for the fused refresh
};
// Local-window block selection (reads only seq_lens; writes block_idx, num_sel).
cudaError_t launch_select_window(const SelectArgs &a, cudaStream_t stream);
// workspace: semaphores [B*Hkv] (zero between calls) + score keys [B*Hkv, ceil(T/bs)]
size_t select_workspace_bytes(int B, int Hkv, int T, int bs);
// K non-null: first refresh each row's last-block summary from K (fused maintenance).
cudaError_t launch_select_blocks(const SelectArgs &a, const uint16_t *K, void *ws, int num_sms,
                                 cudaStream_t stream);

struct AttnArgs {
  const uint16_t *q, *K, *V;
  const int32_t *seq_lens;
  const int32_t *idx;
  const int32_t *num_idx;
  float *out_f32;
  uint16_t *out_bf16;
  float *lse;
  uint32_t *status;
  int B, Hq, Hkv, D, T;
  int cap, tpi, shared;
  float scale;
  KvLayout kv;
};
// Resident CTAs per SM the attention workspace is sized for (the launch never exceeds it).
constexpr int kAttnMaxCtasPerSm = 4;
// workspace: semaphores [B*Hkv] (zero between calls) + split-row partials
size_t attn_workspace_bytes(int B, int Hq, int Hkv, int D, int num_sms);
cudaError_t launch_sparse_decode_attn(const AttnArgs &a, void *ws, int num_sms,
                                      cudaStream_t stream);

// The decode step in one launch: last-block refresh, scoring, top-k (into
// a.block_idx / a.num_sel) and attention over the kept blocks (aa's lists are
// those outputs).  Workspace: the selection workspace followed by the attention
// workspace; falls back to the two-launch form where the one-launch kernel does
// not apply.
size_t decode_step_workspace_bytes(int B, int Hq, int Hkv, int D, int T, int bs, int num_sms);
cudaError_t launch_decode_step(const SelectArgs &sa, const uint16_t *K, const AttnArgs &aa,
                               void *ws, int num_sms, cudaStream_t stream);

struct UnifiedArgs {
  const uint16_t *q, *K;
  const int32_t *seq_lens;
  int32_t *token_idx;
  int32_t *num_sel;
  uint32_t *keys;   // workspace [B, Hq, T] score keys
  int32_t *votes;   // workspace [B, T]
  uint32_t *bits;   // workspace [B, Hq, ceil(T/32)]: each head's picks as a bit set
  uint32_t *status;
  int B, Hq, Hkv, D, T, P, budget, R;
};
size_t unified_workspace_bytes(int B, int Hq, int T);
cudaError_t launch_unified_select(const UnifiedArgs &a, int num_sms, cudaStream_t stream);
// Per-head token top-k lists (P = k = budget; token_idx [B, Hq, k], num_sel [B, Hq]).
cudaError_t launch_tokens_per_head(const UnifiedArgs &a, cudaStream_t stream);
// Row b's list and count <- those of query head head[b] (device array [B]), from
// lists [B, Hq, k] and counts [B, Hq].
cudaError_t launch_gather_head_lists(const int32_t *lists, const int32_t *counts,
                                     const int32_t *head, int B, int Hq, int k,
                                     int32_t *token_idx, int32_t *num_sel, cudaStream_t stream);

// Resident CTAs per SM of `func` launched with `threads` threads and `smem`
// bytes of dynamic shared memory, on the current device.  The first query per
// (device, kernel, threads, smem) raises the kernel's dynamic shared-memory
// limit as needed and asks the occupancy calculator; later ones read a memo,
// so a launch pays no driver query.  Thread-safe.
cudaError_t kernel_occupancy(const void *func, int threads, size_t smem, int *occ);

// Streaming multiprocessors of the current device (memo per device; 148 if
// the query fails).
int device_sm_count();

// Records a message for ksa_last_error() and returns `status`.
ksa_status set_last_error(ksa_status status, const char *fmt, ...)
    __attribute__((format(printf, 2, 3)));

// TMA descriptor for a [rows, D] bf16 matrix, 128B swizzle, box = 64 x box_rows.
bool encode_kv_tensor_map(CUtensorMap *map, const void *base, uint64_t rows, int D,
                          int box_rows);

}  // namespace ksa
