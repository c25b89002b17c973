// summaries.cu -- maintenance of the block mean representation.
//
// Kinetics (block top-k section): the history is cut into blocks of bs tokens
// and every block is represented by its mean key,
//   S[b,g,j,:] = (1/n_j) sum_{t in block j, t < L_b} K[b,g,t,:],  n_j = min(bs, L_b - j*bs).
//
// One warp per block.  Lane l reads 16-byte chunk (l % (D/8)) of the block's
// rows l / (D/8), l / (D/8) + 32/(D/8), ... so every warp-wide load covers
// 2 (D = 128) or 4 (D = 64) whole key rows and all of a block's loads are
// independent (in flight together).  Partial sums meet through warp shuffles;
// then one IEEE division by n_j, in fp32, and the mean is stored as fp32, as
// bf16 rounded to nearest even, or as fp8 e4m3 with a per-block scale.
//
// Also here: the decode step's cache append (the new token's key and value
// rows written into their slot), the write that the last-block refresh of the
// summaries follows.
#include "ksa_device.cuh"
#include "ksa_internal.h"

namespace ksa {

namespace {

template <int D>
__global__ void __launch_bounds__(256) block_summaries_kernel(SummaryArgs a) {
  const int lane = threadIdx.x & 31;
  const int wpc = blockDim.x >> 5;
  const int nb_max = (a.T + a.bs - 1) / a.bs;
  const bool all = (a.mode == KSA_SUMMARY_ALL);
  pdl_wait();
  pdl_launch_dependents();
  const long long total =
      all ? static_cast<long long>(a.B) * a.Hkv * nb_max : static_cast<long long>(a.B) * a.Hkv;
  for (long long w = static_cast<long long>(blockIdx.x) * wpc + (threadIdx.x >> 5); w < total;
       w += static_cast<long long>(gridDim.x) * wpc) {
    const long long bg = all ? w / nb_max : w;
    const int b = static_cast<int>(bg / a.Hkv);
    const int L = clamp_len(a.seq_lens[b], a.T, lane == 0 ? a.status : nullptr);
    const int nb = (L + a.bs - 1) / a.bs;
    int j;
    if (all) {
      j = static_cast<int>(w % nb_max);
      if (j >= nb) continue;
    } else {
      if (nb == 0) continue;
      j = nb - 1;
    }
    const int n = min(a.bs, L - j * a.bs);
    float mean[8];
    const long long row0 = kv_row(a.kv, b, static_cast<int>(bg - static_cast<long long>(b) * a.Hkv),
                                  a.Hkv, a.T, static_cast<long long>(j) * a.bs);
    bool mine;
    if (row0 < 0) {  // a page id that names no page: flagged, the block reads as zeros
      if (lane == 0) flag_status(a.status, KSA_FLAG_INDEX_SKIPPED);
#pragma unroll
      for (int i = 0; i < 8; ++i) mean[i] = 0.f;
      mine = lane < D / 8;
    } else {
      mine = warp_block_mean<D>(a.K + static_cast<size_t>(row0) * D, n, mean);
    }
    store_block_mean_any<D>(a.S, a.sfmt, static_cast<size_t>(a.B) * a.Hkv * nb_max,
                            static_cast<size_t>(bg) * nb_max + j, mine, mean);
  }
}

// One thread per 16-byte chunk of the new K rows, then of the new V rows.  A
// row whose seq_len is outside [1, T], or whose slot's page id names no page,
// is not written (a clamped slot would overwrite a valid token) and is flagged.
__global__ void __launch_bounds__(256) append_kv_kernel(const AppendArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const int ch = a.D / 8;  // 16-byte chunks per row
  const long long n = static_cast<long long>(a.B) * a.Hkv * ch;
  long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= 2 * n) return;
  const bool is_v = e >= n;
  if (is_v) e -= n;
  const int c = static_cast<int>(e % ch);
  const long long bg = e / ch;
  const int b = static_cast<int>(bg / a.Hkv), g = static_cast<int>(bg - static_cast<long long>(b) * a.Hkv);
  const bool reporter = c == 0 && !is_v;
  const int len = a.seq_lens[b];
  if (len < 1 || len > a.T) {
    if (reporter && g == 0) flag_status(a.status, KSA_FLAG_SEQ_LEN_CLAMPED);
    return;
  }
  const long long row = kv_row(a.kv, b, g, a.Hkv, a.T, len - 1);
  if (row < 0) {
    if (reporter) flag_status(a.status, KSA_FLAG_INDEX_SKIPPED);
    return;
  }
  const uint16_t *src = (is_v ? a.v_new : a.k_new) + bg * a.D + c * 8;
  uint16_t *dst = (is_v ? a.V : a.K) + row * a.D + c * 8;
  *reinterpret_cast<uint4 *>(dst) = __ldg(reinterpret_cast<const uint4 *>(src));
}

}  // namespace

cudaError_t launch_append_kv(const AppendArgs &a, cudaStream_t stream) {
  const long long n = 2LL * a.B * a.Hkv * (a.D / 8);
  return launch_pdl(append_kv_kernel, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0,
                    stream, a);
}

cudaError_t launch_block_summaries(const SummaryArgs &a, cudaStream_t stream) {
  const int nb_max = (a.T + a.bs - 1) / a.bs;
  const long long warps = (a.mode == KSA_SUMMARY_ALL)
                              ? static_cast<long long>(a.B) * a.Hkv * nb_max
                              : static_cast<long long>(a.B) * a.Hkv;
  // last-block updates are few and latency-bound: one warp per CTA spreads them
  // over every SM; full rebuilds stream with 8 warps per CTA
  const int threads = (a.mode == KSA_SUMMARY_ALL) ? 256 : 32;
  const int wpc = threads / 32;
  long long blocks = (warps + wpc - 1) / wpc;
  if (blocks > 148LL * 64) blocks = 148LL * 64;
  if (blocks < 1) blocks = 1;
  const dim3 grid(static_cast<unsigned>(blocks)), block(threads);
  if (a.D == 128) return launch_pdl(block_summaries_kernel<128>, grid, block, 0, stream, a);
  return launch_pdl(block_summaries_kernel<64>, grid, block, 0, stream, a);
}

}  // namespace ksa
