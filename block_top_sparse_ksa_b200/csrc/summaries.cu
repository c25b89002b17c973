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
// then one IEEE division by n_j, in fp32, and the mean is stored as fp32 or
// as bf16 rounded to nearest even.
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
    if (mine)
      store_mean8(a.S, a.sbf16, (static_cast<size_t>(bg) * nb_max + j) * D, (lane % (D / 8)) * 8,
                  mean);
  }
}

}  // namespace

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
