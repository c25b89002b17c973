// select_blocks.cu -- block scoring and top-k block selection.
//
// Kinetics (block top-k section): every block's mean key is scored against the
// query and the K' most relevant blocks are kept.  Reading of the relevance
// (the source gives no formula): the dot product of the block mean with the
// sum of the kv-group's query heads, one selection per kv-head.
//
// One CTA per (row b, kv-head g, chunk of up to 64 blocks).  The CTA pulls its
// chunk of fp32 summaries (<= 32 KB, contiguous) into shared memory with one
// TMA bulk copy, so the whole chunk is in flight at once, forms the group
// query sum meanwhile, scores the blocks (8 lanes per summary row, warp
// shuffles) and stores order-preserving uint32 score keys in the workspace.
// The row's chunks count themselves on a semaphore; the CTA finishing last
// stages the row's keys in shared memory and runs an exact radix select
// (k-th largest key; ties at the threshold go to the lower block index),
// writes the winners in ascending block order, and resets the semaphore.
//
// With a key cache given (the fused decode-step entry point), the CTA whose
// chunk holds a row's last block first recomputes that block's mean from the
// keys -- the per-step maintenance of the block representation -- while its
// chunk is in flight, stores it in the summaries and scores the fresh value.
#include "ksa_device.cuh"
#include "ksa_internal.h"

namespace ksa {

namespace {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelRows = 64;  // summary rows per CTA (32 KB at D = 128: many CTAs resident)

struct SelDev {
  SelectArgs a;
  const uint16_t *K;  // non-null: refresh each row's last-block summary from K first
  int chunks;      // CTAs per (row, kv-head)
  uint32_t *keys;  // workspace [B*Hkv, nb_max]
  int32_t *sem;    // workspace [B*Hkv], zero between calls
};

__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

template <int D>
__global__ void __launch_bounds__(kSelThreads) select_blocks_kernel(const SelDev p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float *sbuf = reinterpret_cast<float *>(smem_raw);  // chunk summaries, later the row's keys
  __shared__ uint64_t bar;
  __shared__ __align__(16) float qsum[D];
  __shared__ __align__(16) float fresh[D];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t info[4];
  __shared__ uint32_t scratch[33];
  __shared__ int is_last;
  __shared__ int timed_out;

  const SelectArgs &a = p.a;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.x / p.chunks, chunk = blockIdx.x % p.chunks;
  pdl_wait();
  pdl_launch_dependents();
  const int b = row / a.Hkv, g = row % a.Hkv;
  const int G = a.Hq / a.Hkv;
  const int nb_max = (a.T + a.bs - 1) / a.bs;
  const int L = clamp_len(a.seq_lens[b], a.T, (chunk == 0 && tid == 0) ? a.status : nullptr);
  const int nb = (L + a.bs - 1) / a.bs;
  const int k = a.k;
  int32_t *out = a.block_idx + static_cast<size_t>(row) * k;

  if (nb <= k) {  // every block is kept; no summary is read
    if (chunk == 0) {
      for (int i = tid; i < k; i += kSelThreads) out[i] = i < nb ? i : -1;
      if (tid == 0) a.num_sel[row] = nb;
      if (p.K != nullptr && nb > 0 && warp == 0) {
        // fused maintenance still keeps the last block's mean current
        float mean[8];
        const int jl = nb - 1;
        const uint16_t *rows =
            p.K + (static_cast<size_t>(row) * a.T + static_cast<size_t>(jl) * a.bs) * D;
        if (warp_block_mean<D>(rows, L - jl * a.bs, mean)) {
          float *dst = a.S + (static_cast<size_t>(row) * nb_max + jl) * D + (lane % (D / 8)) * 8;
          reinterpret_cast<float4 *>(dst)[0] = make_float4(mean[0], mean[1], mean[2], mean[3]);
          reinterpret_cast<float4 *>(dst)[1] = make_float4(mean[4], mean[5], mean[6], mean[7]);
        }
      }
    }
    return;
  }
  const int j0 = static_cast<int>(static_cast<long long>(chunk) * nb / p.chunks);
  const int j1 = static_cast<int>(static_cast<long long>(chunk + 1) * nb / p.chunks);
  const int n = j1 - j0;
  if (tid == 0) {
    mbar_init(&bar, 1u);
    timed_out = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0 && n > 0) {
    const uint32_t bytes = static_cast<uint32_t>(n) * D * 4u;
    mbar_arrive_expect_tx(&bar, bytes);
    bulk_g2s(sbuf, a.S + (static_cast<size_t>(row) * nb_max + j0) * D, bytes, &bar);
  }
  // group query sum while the chunk is in flight
  for (int d = tid; d < D; d += kSelThreads) {
    const uint16_t *qp = a.q + (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(g) * G) * D + d;
    float s = 0.f;
    for (int h = 0; h < G; ++h) s += bf16_bits_to_f32(qp[static_cast<size_t>(h) * D]);
    qsum[d] = s;
  }
  // fused maintenance: the chunk holding the row's last block refreshes its mean
  const bool refresh = p.K != nullptr && n > 0 && j1 == nb;
  if (refresh && warp == 0) {
    float mean[8];
    const int jl = nb - 1;
    const uint16_t *rows =
        p.K + (static_cast<size_t>(row) * a.T + static_cast<size_t>(jl) * a.bs) * D;
    if (warp_block_mean<D>(rows, L - jl * a.bs, mean)) {
      const int c8 = (lane % (D / 8)) * 8;
      float *dst = a.S + (static_cast<size_t>(row) * nb_max + jl) * D + c8;
      reinterpret_cast<float4 *>(dst)[0] = make_float4(mean[0], mean[1], mean[2], mean[3]);
      reinterpret_cast<float4 *>(dst)[1] = make_float4(mean[4], mean[5], mean[6], mean[7]);
#pragma unroll
      for (int i = 0; i < 8; ++i) fresh[c8 + i] = mean[i];
    }
  }
  __syncthreads();

  uint32_t bad = 0u;
  if (n > 0 && !__all_sync(0xffffffffu, mbar_wait(&bar, 0u))) {
    bad |= KSA_FLAG_WAIT_TIMEOUT;
    timed_out = 1;
  }
  if (refresh && bad == 0u) {  // after the copy landed: overwrite the stale summary
    for (int d = tid; d < D; d += kSelThreads) sbuf[static_cast<size_t>(n - 1) * D + d] = fresh[d];
  }
  __syncthreads();
  if (n > 0 && bad == 0u) {
    constexpr int PER = D / 32;  // float4 chunks per lane: chunk (sub + 8*i) of the row
    const int sub = lane & 7;
    float4 qv[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) qv[i] = reinterpret_cast<const float4 *>(qsum)[sub + 8 * i];
    uint32_t *krow = p.keys + static_cast<size_t>(row) * nb_max;
    // warp-uniform trip count: every lane reaches the full-mask shuffles
    for (int jw = warp * 4; jw < n; jw += kSelWarps * 4) {
      const int jr = jw + (lane >> 3);
      const bool live = jr < n;
      const float4 *srow = reinterpret_cast<const float4 *>(sbuf + static_cast<size_t>(jr) * D);
      float s = 0.f;
      if (live) {
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          const float4 v = srow[sub + 8 * i];
          s = fmaf(qv[i].x, v.x, s);
          s = fmaf(qv[i].y, v.y, s);
          s = fmaf(qv[i].z, v.z, s);
          s = fmaf(qv[i].w, v.w, s);
        }
      }
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      s += __shfl_xor_sync(0xffffffffu, s, 4);
      if (live && sub == 0) {
        bool nan;
        krow[j0 + jr] = score_key(s, nan);
        bad |= nan ? KSA_FLAG_NONFINITE_SCORE : 0u;
      }
    }
  }
  flag_status(a.status, bad);
  __threadfence();
  __syncthreads();
  if (tid == 0) is_last = (atomicAdd(&p.sem[row], 1) == p.chunks - 1) ? 1 : 0;
  __syncthreads();
  if (timed_out) {  // block-uniform: read after the barrier above
    if (tid == 0) mbar_wait(&bar, 0u);  // let the copy land before the smem is reused
    __syncthreads();
  }
  if (!is_last) return;

  // ---- last chunk of the row: exact top-k over the row's keys
  __threadfence();
  uint32_t *kb = reinterpret_cast<uint32_t *>(sbuf);
  const uint32_t *krow = p.keys + static_cast<size_t>(row) * nb_max;
  for (int j = tid; j < nb; j += kSelThreads) kb[j] = __ldcg(krow + j);
  __syncthreads();
  uint32_t tau, n_gt, n_eq;
  radix_select_desc<kSelThreads>(kb, nb, k, 32, hist, info, tau, n_gt, n_eq);
  select_ascending<kSelThreads>(kb, nb, tau, n_gt, n_eq, k, out, scratch, [](int) {});
  if (tid == 0) {
    a.num_sel[row] = k;
    p.sem[row] = 0;  // ready for the next call
  }
}

}  // namespace

size_t select_workspace_bytes(int B, int Hkv, int T, int bs) {
  const size_t rows = static_cast<size_t>(B) * Hkv;
  const size_t nb_max = static_cast<size_t>((T + bs - 1) / bs);
  const size_t sems = (rows * sizeof(int32_t) + 255) & ~static_cast<size_t>(255);
  const size_t keys = (rows * nb_max * sizeof(uint32_t) + 255) & ~static_cast<size_t>(255);
  return sems + keys;
}

cudaError_t launch_select_blocks(const SelectArgs &a, const uint16_t *K, void *ws, int num_sms,
                                 cudaStream_t stream) {
  (void)num_sms;
  const int nb_max = (a.T + a.bs - 1) / a.bs;
  SelDev p;
  p.a = a;
  p.K = K;
  p.chunks = (nb_max + kSelRows - 1) / kSelRows;
  const size_t rows = static_cast<size_t>(a.B) * a.Hkv;
  const size_t sems = (rows * sizeof(int32_t) + 255) & ~static_cast<size_t>(255);
  p.sem = static_cast<int32_t *>(ws);
  p.keys = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) + sems);
  size_t smem = static_cast<size_t>(kSelRows) * a.D * sizeof(float);
  if (static_cast<size_t>(nb_max) * sizeof(uint32_t) > smem)
    smem = static_cast<size_t>(nb_max) * sizeof(uint32_t);
  const unsigned grid = static_cast<unsigned>(rows * p.chunks);
  cudaError_t err;
  if (a.D == 128) {
    err = cudaFuncSetAttribute(select_blocks_kernel<128>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    return launch_pdl(select_blocks_kernel<128>, dim3(grid), dim3(kSelThreads), smem, stream, p);
  } else {
    err = cudaFuncSetAttribute(select_blocks_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    return launch_pdl(select_blocks_kernel<64>, dim3(grid), dim3(kSelThreads), smem, stream, p);
  }
}

}  // namespace ksa
