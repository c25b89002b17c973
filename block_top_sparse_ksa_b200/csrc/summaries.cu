// summaries.cu -- maintenance of the block mean representation.
//
// Kinetics (block top-k section): the history is cut into blocks of bs tokens
// and every block is represented by its mean key,
//   S[b,g,j,:] = (1/n_j) sum_{t in block j, t < L_b} K[b,g,t,:],  n_j = min(bs, L_b - j*bs).
//
// One warp per block: lane l owns D/32 consecutive dims, so every warp-wide
// load reads one whole 2*D-byte key row (fully coalesced); the bs rows of a
// block are independent loads kept in flight by unrolling.  Sums are fp32 in
// token order, then one IEEE division by n_j.
#include "ksa_device.cuh"
#include "ksa_internal.h"

namespace ksa {

namespace {

template <int D>
__device__ __forceinline__ void load_dims(const uint16_t *p, float (&v)[D / 32]) {
  if constexpr (D == 128) {
    const uint2 x = __ldg(reinterpret_cast<const uint2 *>(p));
    v[0] = bf16_lo(x.x);
    v[1] = bf16_hi(x.x);
    v[2] = bf16_lo(x.y);
    v[3] = bf16_hi(x.y);
  } else {
    const uint32_t x = __ldg(reinterpret_cast<const uint32_t *>(p));
    v[0] = bf16_lo(x);
    v[1] = bf16_hi(x);
  }
}

template <int D>
__global__ void __launch_bounds__(256) block_summaries_kernel(SummaryArgs a) {
  constexpr int DPL = D / 32;
  const int lane = threadIdx.x & 31;
  const int wpc = blockDim.x >> 5;
  const int nb_max = (a.T + a.bs - 1) / a.bs;
  const bool all = (a.mode == KSA_SUMMARY_ALL);
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
    const uint16_t *src = a.K + (static_cast<size_t>(bg) * a.T + static_cast<size_t>(j) * a.bs) * D +
                          lane * DPL;
    float acc[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[i] = 0.f;
#pragma unroll 8
    for (int t = 0; t < n; ++t) {
      float v[DPL];
      load_dims<D>(src + static_cast<size_t>(t) * D, v);
#pragma unroll
      for (int i = 0; i < DPL; ++i) acc[i] += v[i];
    }
    float *dst = a.S + (static_cast<size_t>(bg) * nb_max + j) * D + lane * DPL;
    const float fn = static_cast<float>(n);
    if constexpr (DPL == 4) {
      *reinterpret_cast<float4 *>(dst) =
          make_float4(acc[0] / fn, acc[1] / fn, acc[2] / fn, acc[3] / fn);
    } else {
      *reinterpret_cast<float2 *>(dst) = make_float2(acc[0] / fn, acc[1] / fn);
    }
  }
}

}  // namespace

cudaError_t launch_block_summaries(const SummaryArgs &a, cudaStream_t stream) {
  const int nb_max = (a.T + a.bs - 1) / a.bs;
  const long long warps = (a.mode == KSA_SUMMARY_ALL)
                              ? static_cast<long long>(a.B) * a.Hkv * nb_max
                              : static_cast<long long>(a.B) * a.Hkv;
  const int threads = 256;
  long long blocks = (warps + 7) / 8;
  if (blocks > 148LL * 32) blocks = 148LL * 32;
  if (blocks < 1) blocks = 1;
  if (a.D == 128)
    block_summaries_kernel<128><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(a);
  else
    block_summaries_kernel<64><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace ksa
