/*
 * ksa.h -- C ABI of libksa: decode-phase block top-k sparse attention over a
 * GQA KV cache, and LessIsMore unified token selection, for NVIDIA B200
 * (sm_100a).
 *
 * Sources of the method:
 *   [KIN] Kinetics: Rethinking Test-Time Scaling Laws (press summary,
 *         news.43u.com.cn), section 5 "from theory to practice: block top-k".
 *   [LIM] LessIsMore (press summary, techwalker.com), section 2 "unified head
 *         selection" / "stable recency window", section 4 "mechanism
 *         analysis", section 5 "implementation".
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers, dense row-major, owned by the
 *     caller; the one exception, head_of_row of ksa_select_tokens_one_head, is
 *     a host array.  The library allocates nothing, keeps no state between calls,
 *     and never synchronises the host: work is enqueued on `stream`
 *     (a cudaStream_t passed as void*; NULL = the legacy default stream).
 *   - bf16 tensors are passed as uint16_t* (the raw bf16 bit patterns).
 *   - Shapes: B = batch, Hq / Hkv = query / kv heads (G = Hq/Hkv query heads
 *     share one kv-head), D = head_dim, T = capacity (tokens per cache row),
 *     bs = block_size, L_b = seq_lens[b] (tokens held by row b, the current
 *     token included), NB_b = ceil(L_b / bs).
 *   - Caches K, V: [B, Hkv, T, D] bf16.  Queries q: [B, Hq, D] bf16.
 *   - Host-side validation failures return KSA_ERR_INVALID_ARG (bad argument)
 *     or KSA_ERR_UNSUPPORTED (valid but not covered by the kernels) and
 *     enqueue nothing.  A failed launch returns KSA_ERR_CUDA.
 *     ksa_last_error() gives a message for the calling thread's last failure.
 *   - dev_status (nullable): a device uint32 that kernels OR KSA_FLAG_* bits
 *     into when device data is out of range.  It is never cleared by the
 *     library; the caller zeroes it and reads it back when it wants to know.
 *   - Bad device data never faults: a seq_len outside [1, T] is clamped to
 *     [0, T] and flagged; an index entry outside the row is skipped and
 *     flagged.
 *   - Workspaces (ws): caller-allocated device scratch of the size the
 *     matching *_workspace() query returns for the same shape on the current
 *     device, 256-byte aligned.  The select and attention workspaces begin with
 *     per-row semaphores that must be zero when a call starts: zero-fill the
 *     buffer once after allocating it; every call that completes leaves them
 *     zero again, so one buffer serves any number of calls issued one after
 *     another.  Calls that may run concurrently need separate workspaces.
 *     After a KSA_FLAG_WAIT_TIMEOUT the workspace must be zero-filled again.
 */
#ifndef KSA_H
#define KSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KSA_OK = 0,
  KSA_ERR_INVALID_ARG = 1,
  KSA_ERR_UNSUPPORTED = 2,
  KSA_ERR_WORKSPACE = 3,
  KSA_ERR_CUDA = 4
} ksa_status;

typedef struct {
  int32_t batch;        /* B */
  int32_t num_q_heads;  /* Hq */
  int32_t num_kv_heads; /* Hkv; Hq % Hkv == 0 */
  int32_t head_dim;     /* D: 64 or 128 */
  int32_t capacity;     /* T: token slots per cache row */
  int32_t block_size;   /* bs: 16, 32 or 64 for the block entry points */
} ksa_shape;

enum { KSA_SUMMARY_ALL = 0, KSA_SUMMARY_LAST_BLOCK = 1 };
/* Storage type of the block summaries (the *_ex entry points). */
enum { KSA_SUMMARIES_F32 = 0, KSA_SUMMARIES_BF16 = 1, KSA_SUMMARIES_FP8 = 2 };
enum { KSA_OUT_F32 = 0, KSA_OUT_BF16 = 1 };
/* Index-list layouts of ksa_sparse_decode_attn (idx_shared). */
enum { KSA_IDX_PER_KV_HEAD = 0, KSA_IDX_SHARED = 1, KSA_IDX_PER_Q_HEAD = 2 };

enum {
  KSA_FLAG_SEQ_LEN_CLAMPED = 1u << 0, /* some seq_len was outside [1, T] */
  KSA_FLAG_INDEX_SKIPPED = 1u << 1,   /* some index entry named no valid token */
  KSA_FLAG_NONFINITE_SCORE = 1u << 2, /* a NaN score was ranked lowest */
  KSA_FLAG_WAIT_TIMEOUT = 1u << 3     /* a pipeline wait gave up: results invalid */
};

/*
 * Block summaries (maintenance of the block mean representation) [KIN s.5].
 *   S[b,g,j,:] = (1/n_j) * sum_{t=j*bs}^{j*bs+n_j-1} K[b,g,t,:],
 *   n_j = min(bs, L_b - j*bs), computed in fp32 from bf16 keys.
 * mode KSA_SUMMARY_ALL rebuilds every block j < NB_b (prefill);
 * mode KSA_SUMMARY_LAST_BLOCK rebuilds only j = NB_b - 1 (one decode step
 * after appending a token).  Entries j >= NB_b are not written.
 *   K:         [B, Hkv, T, D] bf16 (read)
 *   seq_lens:  [B] int32 (read)
 *   summaries: [B, Hkv, ceil(T/bs), D] fp32 (written)
 */
ksa_status ksa_build_block_summaries(const ksa_shape *shape, const uint16_t *K,
                                     const int32_t *seq_lens, int32_t mode,
                                     float *summaries, uint32_t *dev_status,
                                     void *stream);

/*
 * Block scoring and top-k selection [KIN s.5]: for every (b, kv-head g)
 *   s_j = sum_{h in group g} <q[b,h,:], S[b,g,j,:]>   (j < NB_b, fp32)
 * and the k_blocks largest s_j are kept, ties to the lower j, listed in
 * ascending j.  If NB_b <= k_blocks every block is kept and no summary is
 * read.  A NaN score ranks lowest and sets KSA_FLAG_NONFINITE_SCORE.
 *   q:         [B, Hq, D] bf16
 *   summaries: [B, Hkv, ceil(T/bs), D] fp32 (from ksa_build_block_summaries)
 *   block_idx: [B, Hkv, k_blocks] int32, ascending, -1 padded (written)
 *   num_sel:   [B, Hkv] int32 = min(k_blocks, NB_b) (written)
 *   ws:        device scratch of ksa_select_blocks_workspace() bytes, 256-byte
 *              aligned (see "Workspaces" above).
 * Limits: k_blocks >= 1; ceil(T/bs) <= 16384 (the scores of one row are
 * ranked in on-chip memory), else KSA_ERR_UNSUPPORTED.
 */
size_t ksa_select_blocks_workspace(const ksa_shape *shape, int32_t k_blocks);
ksa_status ksa_select_blocks(const ksa_shape *shape, const uint16_t *q,
                             const float *summaries, const int32_t *seq_lens,
                             int32_t k_blocks, int32_t *block_idx,
                             int32_t *num_sel, void *ws, size_t ws_bytes,
                             uint32_t *dev_status, void *stream);

/*
 * One decode step's selection in one call [KIN s.5]: for every row b and
 * kv-head g, first recompute the mean of the last block j = NB_b - 1 from K
 * and store it in `summaries` (what ksa_build_block_summaries does with
 * KSA_SUMMARY_LAST_BLOCK, bit for bit), then score and select exactly as
 * ksa_select_blocks.  The refresh runs inside the scoring launch, so the call
 * is two launches (scoring, ranking), or one when no row can hold more than
 * k_blocks blocks.  Use after appending the step's token to K.
 * Arguments as ksa_select_blocks, plus K [B, Hkv, T, D] bf16 (read);
 * `summaries` is read and its last-block entries are written.
 */
ksa_status ksa_decode_select_blocks(const ksa_shape *shape, const uint16_t *q,
                                    const uint16_t *K, float *summaries,
                                    const int32_t *seq_lens, int32_t k_blocks,
                                    int32_t *block_idx, int32_t *num_sel, void *ws,
                                    size_t ws_bytes, uint32_t *dev_status, void *stream);

/*
 * Token-level sparse attention's selection [KIN s.5: the ideal, per-token
 * top-K; costly, the reason for blocks]: every query head h of row b keeps its
 * own k_tokens highest-scoring tokens, s_t = <q[b,h,:], K[b,g,t,:]> over
 * t < L_b (exact fp32 products of bf16, ties to the lower t), listed
 * ascending and -1 padded.  If L_b <= k_tokens every token is kept.  Use the
 * lists with ksa_sparse_decode_attn, idx_shared = KSA_IDX_PER_Q_HEAD,
 * tokens_per_idx = 1.
 *   q: [B, Hq, D] bf16;  K: [B, Hkv, T, D] bf16
 *   token_idx: [B, Hq, k_tokens] int32;  num_sel: [B, Hq] int32 (written)
 *   ws: device scratch of ksa_select_tokens_per_head_workspace() bytes,
 *       256-byte aligned, no initialisation needed.
 * Limits: G <= 8; capacity <= 65536; k_tokens >= 1.
 */
size_t ksa_select_tokens_per_head_workspace(const ksa_shape *shape, int32_t k_tokens);
ksa_status ksa_select_tokens_per_head(const ksa_shape *shape, const uint16_t *q,
                                      const uint16_t *K, const int32_t *seq_lens,
                                      int32_t k_tokens, int32_t *token_idx,
                                      int32_t *num_sel, void *ws, size_t ws_bytes,
                                      uint32_t *dev_status, void *stream);

/*
 * Random-head aggregation [LIM s.4, mechanism analysis: of three ways to turn
 * the heads' choices into one set -- a randomly chosen head's selection used
 * for all heads, a set per head, the unified vote -- the random head does
 * worst]: row b takes query head head_of_row[b]'s own top-k_tokens set (the
 * ranking of ksa_select_tokens_per_head) as the one set every head reads.
 * The random draw is the caller's: head_of_row is a HOST array [B] of heads in
 * [0, Hq), read before this call returns.  Use the lists with
 * ksa_sparse_decode_attn, idx_shared = KSA_IDX_SHARED, tokens_per_idx = 1.
 *   token_idx: [B, k_tokens] int32;  num_sel: [B] int32 (written)
 *   ws: device scratch of ksa_select_tokens_one_head_workspace() bytes,
 *       256-byte aligned, no initialisation needed.
 * It runs the per-head kernels into the workspace, copies head_of_row into
 * the workspace (one host-to-device cudaMemcpyAsync on `stream`), and gathers
 * each row's chosen list and count with one launch.  A head outside [0, Hq)
 * is KSA_ERR_INVALID_ARG before any launch.
 * Limits: as ksa_select_tokens_per_head.
 */
size_t ksa_select_tokens_one_head_workspace(const ksa_shape *shape, int32_t k_tokens);
ksa_status ksa_select_tokens_one_head(const ksa_shape *shape, const uint16_t *q,
                                      const uint16_t *K, const int32_t *seq_lens,
                                      const int32_t *head_of_row, int32_t k_tokens,
                                      int32_t *token_idx, int32_t *num_sel, void *ws,
                                      size_t ws_bytes, uint32_t *dev_status, void *stream);

/*
 * Local attention as a block selection [KIN s.5 compares block top-k with
 * local attention, a fixed pattern over the nearest tokens]: every (b, g)
 * keeps its last min(k_blocks, NB_b) blocks, NB_b - n .. NB_b - 1, ascending
 * and -1 padded, in the layout of ksa_select_blocks, for the same attention
 * call.  Reads only seq_lens; no workspace.
 */
ksa_status ksa_select_window(const ksa_shape *shape, const int32_t *seq_lens,
                             int32_t k_blocks, int32_t *block_idx, int32_t *num_sel,
                             uint32_t *dev_status, void *stream);

/*
 * The same three calls with the summaries stored as fp32, bf16 or fp8
 * (summary_dtype: KSA_SUMMARIES_F32, _BF16 or _FP8).  Each block mean is
 * computed in fp32 as above and stored in the chosen format: fewer bytes for
 * the maintenance writes and, above all, for the scoring reads, which
 * dominate at long context and small budget [KIN s.5 names the block mean;
 * the storage precision is this library's option, not the source's].
 *   BF16: each value rounded to the nearest bf16 (ties to even).
 *   FP8:  each block's D values scaled by 2^-e, e the smallest exponent with
 *         max |mean| <= 448 2^e, and rounded to the nearest fp8 e4m3 value
 *         (ties to even); the block keeps the scale 2^e as an fp32.  Layout:
 *         the values [B, Hkv, ceil(T/bs), D] bytes, then the scales
 *         [B, Hkv, ceil(T/bs)] fp32 -- B Hkv ceil(T/bs) (D + 4) bytes in all.
 *         head_dim 128 only (else KSA_ERR_UNSUPPORTED).
 * Scores are accumulated in fp32 from the stored values, so blocks whose
 * scores differ by less than the rounding of their means may rank
 * differently than with fp32 summaries.
 *   summaries: [B, Hkv, ceil(T/bs), D] of the given type (FP8: as above),
 *              16-byte aligned.
 * Every other argument, limit and error as the fp32 calls, which are these
 * with KSA_SUMMARIES_F32.  An unknown summary_dtype is KSA_ERR_INVALID_ARG.
 */
ksa_status ksa_build_block_summaries_ex(const ksa_shape *shape, const uint16_t *K,
                                        const int32_t *seq_lens, int32_t mode,
                                        int32_t summary_dtype, void *summaries,
                                        uint32_t *dev_status, void *stream);
ksa_status ksa_select_blocks_ex(const ksa_shape *shape, const uint16_t *q,
                                const void *summaries, int32_t summary_dtype,
                                const int32_t *seq_lens, int32_t k_blocks,
                                int32_t *block_idx, int32_t *num_sel, void *ws,
                                size_t ws_bytes, uint32_t *dev_status, void *stream);
ksa_status ksa_decode_select_blocks_ex(const ksa_shape *shape, const uint16_t *q,
                                       const uint16_t *K, void *summaries,
                                       int32_t summary_dtype, const int32_t *seq_lens,
                                       int32_t k_blocks, int32_t *block_idx,
                                       int32_t *num_sel, void *ws, size_t ws_bytes,
                                       uint32_t *dev_status, void *stream);

/*
 * Paged KV cache [KIN s.5 pairs block top-k with paged attention; here a page
 * holds one block].  K and V are a pool of pages [num_pages, Hkv, block_size, D]
 * bf16; block_table[b * max_blocks + j] is the page of logical block j of row
 * b, so token t of row b, kv-head g is pages[block_table[b, t / bs], g, t % bs].
 * The logical capacity T (shape->capacity) must equal max_blocks * block_size.
 * The block table is device data: a page id outside [0, num_pages) is never
 * read; it sets KSA_FLAG_INDEX_SKIPPED, its block summarises to zeros, and its
 * tokens are left out of attention.
 */
typedef struct {
  const int32_t *block_table; /* [B, max_blocks] int32, device */
  int32_t max_blocks;         /* entries per row of the table */
  int32_t num_pages;          /* pages in the K and V pools */
} ksa_pages;

/* ksa_build_block_summaries_ex on a paged key cache (K_pages, pages). */
ksa_status ksa_build_block_summaries_paged(const ksa_shape *shape, const uint16_t *K_pages,
                                           const ksa_pages *pages, const int32_t *seq_lens,
                                           int32_t mode, int32_t summary_dtype, void *summaries,
                                           uint32_t *dev_status, void *stream);
/* ksa_decode_select_blocks_ex on a paged key cache (the last-block refresh reads pages). */
ksa_status ksa_decode_select_blocks_paged(const ksa_shape *shape, const uint16_t *q,
                                          const uint16_t *K_pages, const ksa_pages *pages,
                                          void *summaries, int32_t summary_dtype,
                                          const int32_t *seq_lens, int32_t k_blocks,
                                          int32_t *block_idx, int32_t *num_sel, void *ws,
                                          size_t ws_bytes, uint32_t *dev_status, void *stream);

/*
 * The decode step in one call [KIN s.5: keep the block representation
 * current, score every block against the query, keep the K' best, attend
 * over their tokens]: ksa_decode_select_blocks_ex followed by
 * ksa_sparse_decode_attn over its block lists (tokens_per_idx = block_size,
 * KSA_IDX_PER_KV_HEAD), issued from one call on one workspace -- the same
 * launches, so the same results bit for bit.
 *   q, K, V, summaries, summary_dtype, seq_lens, k_blocks: as
 *              ksa_decode_select_blocks_ex (the summary of each row's last
 *              block is refreshed from K and written back)
 *   block_idx: [B, Hkv, k_blocks] int32 and num_sel [B, Hkv] (written)
 *   scale, out_dtype, out, lse: as ksa_sparse_decode_attn
 *   ws:        ksa_decode_step_workspace() bytes, 256-byte aligned: the
 *              selection workspace followed by the attention workspace, with
 *              their rules (zero-fill once; calls that may run concurrently
 *              need separate workspaces).
 * Limits and errors: those of both calls.
 */
size_t ksa_decode_step_workspace(const ksa_shape *shape, int32_t k_blocks);
ksa_status ksa_decode_step(const ksa_shape *shape, const uint16_t *q, const uint16_t *K,
                           const uint16_t *V, void *summaries, int32_t summary_dtype,
                           const int32_t *seq_lens, int32_t k_blocks, int32_t *block_idx,
                           int32_t *num_sel, float scale, int32_t out_dtype, void *out,
                           float *lse, void *ws, size_t ws_bytes, uint32_t *dev_status,
                           void *stream);

/*
 * Cache append: the decode step's write of the new token [KIN s.5: the
 * history the blocks are cut from is the cached keys and values of every
 * token so far; each step adds one].  For every (b, kv-head g):
 *   K[b,g,L_b-1,:] = k_new[b,g,:],   V[b,g,L_b-1,:] = v_new[b,g,:]
 * where L_b = seq_lens[b] already counts the new token.  Run it before the
 * step's selection and attention (ksa_decode_select_blocks then refreshes the
 * summary of the block the token landed in).
 *   k_new, v_new: [B, Hkv, D] bf16 (read)
 *   K, V:         [B, Hkv, T, D] bf16 (one row of each (b, g) written)
 * A row whose seq_len is outside [1, T] is not written and sets
 * KSA_FLAG_SEQ_LEN_CLAMPED (a clamped slot would overwrite a valid token).
 * shape->num_q_heads and block_size are not used (any valid values).
 * Pointers 16-byte aligned, else KSA_ERR_INVALID_ARG.
 */
ksa_status ksa_append_kv(const ksa_shape *shape, const uint16_t *k_new,
                         const uint16_t *v_new, uint16_t *K, uint16_t *V,
                         const int32_t *seq_lens, uint32_t *dev_status, void *stream);
/* ksa_append_kv on a paged cache: the token goes to slot (L_b-1) % bs of page
 * block_table[b, (L_b-1) / bs]; a page id outside the pool is not written and
 * sets KSA_FLAG_INDEX_SKIPPED. */
ksa_status ksa_append_kv_paged(const ksa_shape *shape, const uint16_t *k_new,
                               const uint16_t *v_new, uint16_t *K_pages, uint16_t *V_pages,
                               const ksa_pages *pages, const int32_t *seq_lens,
                               uint32_t *dev_status, void *stream);

/*
 * Sparse decode attention over a selected token set [KIN s.5; LIM s.5
 * "sparse attention layer", GQA kernel sharing one KV set per group].
 * For query head h of row b (kv-head g = h / G) and selected tokens T_sel:
 *   z_t = scale * <q[b,h,:], K[b,g,t,:]>,  w = softmax(z over T_sel),
 *   out[b,h,:] = sum_t w_t V[b,g,t,:],   lse[b,h] = log sum_t exp(z_t).
 * T_sel: idx == NULL -> dense, every t < L_b.  Otherwise entry e < num_idx
 * of the list names tokens [idx*tpi, idx*tpi + tpi) with tpi =
 * tokens_per_idx (block_size for block lists, 1 for token lists); tokens
 * t >= L_b are dropped (partial tail block).  The list is [B, Hkv, cap]
 * with num_idx [B, Hkv] (idx_shared == KSA_IDX_PER_KV_HEAD: one set per GQA
 * group), [B, cap] with num_idx [B] shared by every kv-head (KSA_IDX_SHARED,
 * the LessIsMore layout), or [B, Hq, cap] with num_idx [B, Hq], one set per
 * query head (KSA_IDX_PER_Q_HEAD, e.g. the per-head token top-k of
 * ksa_select_tokens_per_head; each head then reads its own K/V rows, so the
 * group no longer shares one gather).
 * Entries are expected distinct; a negative entry or one naming no token
 * below L_b is skipped and flagged.  An empty set gives out = 0,
 * lse = -inf.  Accumulation is fp32; scale == 0 selects 1/sqrt(D).
 *   out: [B, Hq, D] fp32 (out_dtype KSA_OUT_F32) or bf16 (KSA_OUT_BF16)
 *   lse: [B, Hq] fp32, nullable
 *   ws:  device scratch of ksa_sparse_decode_attn_workspace() bytes, 256-byte
 *        aligned (see "Workspaces" above); rows whose tokens are split between
 *        CTAs leave partial results there.
 * Limits: D in {64, 128}; G <= 8; tokens_per_idx a power of two <= 256.
 */
size_t ksa_sparse_decode_attn_workspace(const ksa_shape *shape,
                                        int32_t idx_capacity,
                                        int32_t tokens_per_idx);
ksa_status ksa_sparse_decode_attn(const ksa_shape *shape, const uint16_t *q,
                                  const uint16_t *K, const uint16_t *V,
                                  const int32_t *seq_lens, const int32_t *idx,
                                  const int32_t *num_idx, int32_t idx_capacity,
                                  int32_t tokens_per_idx, int32_t idx_shared,
                                  float scale, int32_t out_dtype, void *out,
                                  float *lse, void *ws, size_t ws_bytes,
                                  uint32_t *dev_status, void *stream);

/*
 * ksa_sparse_decode_attn on a paged K/V cache (K_pages, V_pages share the
 * block table in `pages`; see "Paged KV cache" above).  shape->block_size is
 * the page size and must be 16, 32 or 64; the workspace is the same as for
 * ksa_sparse_decode_attn.
 */
ksa_status ksa_sparse_decode_attn_paged(const ksa_shape *shape, const uint16_t *q,
                                        const uint16_t *K_pages, const uint16_t *V_pages,
                                        const ksa_pages *pages, const int32_t *seq_lens,
                                        const int32_t *idx, const int32_t *num_idx,
                                        int32_t idx_capacity, int32_t tokens_per_idx,
                                        int32_t idx_shared, float scale, int32_t out_dtype,
                                        void *out, float *lse, void *ws, size_t ws_bytes,
                                        uint32_t *dev_status, void *stream);

/*
 * ksa_sparse_decode_attn without a workspace argument: the same computation,
 * arguments and results, for callers that cannot allocate device memory (a
 * serving loop that allows no new device memory after start-up, or a layer
 * handed only its input and output buffers, with no allocator of its own).  The sources describe no such entry point;
 * it is an integration convenience with no counterpart in the method.
 * The library keeps one fixed 8 MiB scratch area per GPU (held from the first
 * call on that GPU, or from library load when CUDA loads modules eagerly,
 * until the process exits) and uses it in place of the workspace.  Shapes whose
 * ksa_sparse_decode_attn_workspace() exceeds 8 MiB return KSA_ERR_UNSUPPORTED
 * with a message.  It allocates nothing: it clears the scratch's semaphores
 * with cudaMemsetAsync on `stream` and launches the attention kernel.
 * The first call on a device looks up the scratch's device address
 * (cudaGetSymbolAddress), and so does the first call after the device's
 * context has changed (cudaDeviceReset).
 * Every call shares the one scratch area, so calls that may overlap on the
 * GPU (different streams, or different host threads) race: issue them one
 * after another on one stream.
 */
ksa_status ksa_sparse_decode_attn_noalloc(const ksa_shape *shape, const uint16_t *q,
                                          const uint16_t *K, const uint16_t *V,
                                          const int32_t *seq_lens, const int32_t *idx,
                                          const int32_t *num_idx, int32_t idx_capacity,
                                          int32_t tokens_per_idx, int32_t idx_shared,
                                          float scale, int32_t out_dtype, void *out,
                                          float *lse, uint32_t *dev_status, void *stream);

/*
 * LessIsMore unified selection [LIM s.2, s.5 "token selection layer"].
 * For each row b with L = L_b:
 *   1. every query head h scores every token t < L: s_h[t] = <q[b,h], K[b,g(h),t]>
 *      (fp32) and picks its per_head_topk best tokens, ties to the lower t;
 *   2. votes[t] = number of heads that picked t;
 *   3. the result is the (token_budget - recent_tokens) tokens of
 *      [0, L - recent_tokens) with the most votes (ties to the lower t),
 *      plus the window [L - recent_tokens, L), listed ascending.
 *   If L <= token_budget every token [0, L) is selected.
 *   token_idx: [B, token_budget] int32 ascending, -1 padded (written)
 *   num_sel:   [B] int32 (written)
 *   ws:        device scratch of at least ksa_unified_select_workspace() bytes,
 *              256-byte aligned; contents need no initialisation.
 * recent_tokens < 0 selects token_budget / 4 (the 25% window).
 * Limits: 1 <= per_head_topk; 0 <= recent_tokens <= token_budget <= T;
 * T <= 65536.
 */
size_t ksa_unified_select_workspace(const ksa_shape *shape,
                                    int32_t per_head_topk, int32_t token_budget);
ksa_status ksa_unified_select(const ksa_shape *shape, const uint16_t *q,
                              const uint16_t *K, const int32_t *seq_lens,
                              int32_t per_head_topk, int32_t token_budget,
                              int32_t recent_tokens, int32_t *token_idx,
                              int32_t *num_sel, void *ws, size_t ws_bytes,
                              uint32_t *dev_status, void *stream);

/*
 * Reads back a device status word (the dev_status of earlier calls): copies it
 * to *flags on `stream` and waits for the stream, so every call enqueued on
 * it before has finished.  This is the one call that synchronises the host.
 * clear != 0 then zeroes the word on `stream` for the next calls.  One word
 * may collect the KSA_FLAG_* bits of a whole decode step.
 *   dev_status: device uint32;  flags: host uint32 (written).
 */
ksa_status ksa_get_device_status(const uint32_t *dev_status, void *stream, int32_t clear,
                                 uint32_t *flags);

/* Human-readable name of a status code (static string). */
const char *ksa_status_string(ksa_status status);
/* Message describing the calling thread's last failed call ("" if none). */
const char *ksa_last_error(void);
/* Library version: major * 10000 + minor * 100 + patch. */
int32_t ksa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KSA_H */
