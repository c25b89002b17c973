// select_blocks.cu -- block scoring and top-k block selection.
//
// Kinetics (block top-k section): every block's mean key is scored against the
// query and the K' most relevant blocks are kept.  Reading of the relevance
// (the source gives no formula): the dot product of the block mean with the
// sum of the kv-group's query heads, one selection per kv-head.
//
// One thread-block cluster per (row b, kv-head g).  Each CTA of the cluster
// streams a contiguous slice of the row's fp32 summaries (8 lanes per 512-byte
// summary row, 128-bit loads, two row groups in flight per warp), reduces the
// dot products with warp shuffles, and stores order-preserving uint32 score
// keys straight into the shared memory of CTA rank 0 (distributed shared
// memory).  After a cluster barrier, rank 0 runs an exact radix select (k-th
// largest key; ties at the threshold resolved toward the lower block index)
// and writes the winners in ascending block order.  Scores never touch HBM.
#include "ksa_device.cuh"
#include "ksa_internal.h"

namespace ksa {

namespace {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;

template <int D>
__global__ void __launch_bounds__(kSelThreads) select_blocks_kernel(SelectArgs a, int csize) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint32_t *keys = reinterpret_cast<uint32_t *>(smem_raw);  // [nb_max], used on rank 0
  __shared__ uint32_t hist[256];
  __shared__ uint32_t info[4];
  __shared__ uint32_t scratch[33];
  __shared__ __align__(16) float qsum[D];

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.x / csize;
  const int b = row / a.Hkv, g = row % a.Hkv;
  const int G = a.Hq / a.Hkv;
  const int nb_max = (a.T + a.bs - 1) / a.bs;
  const int L = clamp_len(a.seq_lens[b], a.T, (rank == 0 && tid == 0) ? a.status : nullptr);
  const int nb = (L + a.bs - 1) / a.bs;
  const int k = a.k;
  int32_t *out = a.block_idx + static_cast<size_t>(row) * k;

  if (nb <= k) {  // every block is kept; no summary is read (same branch for the whole cluster)
    if (rank == 0) {
      for (int i = tid; i < k; i += kSelThreads) out[i] = i < nb ? i : -1;
      if (tid == 0) a.num_sel[row] = nb;
    }
    return;
  }

  for (int d = tid; d < D; d += kSelThreads) {
    const uint16_t *qp = a.q + (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(g) * G) * D + d;
    float s = 0.f;
    for (int h = 0; h < G; ++h) s += bf16_bits_to_f32(qp[static_cast<size_t>(h) * D]);
    qsum[d] = s;
  }
  cluster.sync();  // all CTAs of the cluster are running before any remote store

  constexpr int PER = D / 32;  // float4 chunks per lane: chunk (sub + 8*i) of the row
  const int sub = lane & 7;
  float4 qv[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) qv[i] = reinterpret_cast<const float4 *>(qsum)[sub + 8 * i];

  const int j0 = static_cast<int>(static_cast<long long>(rank) * nb / csize);
  const int j1 = static_cast<int>(static_cast<long long>(rank + 1) * nb / csize);
  uint32_t *keys0 = cluster.map_shared_rank(keys, 0);
  const float4 *srow =
      reinterpret_cast<const float4 *>(a.S + static_cast<size_t>(row) * nb_max * D);
  uint32_t bad = 0u;
  constexpr int kStride = kSelWarps * 4;  // summary rows covered by the CTA per step
  for (int jb = j0 + warp * 4; jb < j1; jb += 2 * kStride) {
    const int ja = jb + (lane >> 3);
    const int jc = ja + kStride;
    float4 va[PER], vc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      va[i] = ja < j1 ? __ldg(srow + static_cast<size_t>(ja) * (D / 4) + sub + 8 * i)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
      vc[i] = jc < j1 ? __ldg(srow + static_cast<size_t>(jc) * (D / 4) + sub + 8 * i)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float sa = 0.f, sc = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      sa = fmaf(qv[i].x, va[i].x, sa);
      sa = fmaf(qv[i].y, va[i].y, sa);
      sa = fmaf(qv[i].z, va[i].z, sa);
      sa = fmaf(qv[i].w, va[i].w, sa);
      sc = fmaf(qv[i].x, vc[i].x, sc);
      sc = fmaf(qv[i].y, vc[i].y, sc);
      sc = fmaf(qv[i].z, vc[i].z, sc);
      sc = fmaf(qv[i].w, vc[i].w, sc);
    }
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) {
      sa += __shfl_xor_sync(0xffffffffu, sa, off);
      sc += __shfl_xor_sync(0xffffffffu, sc, off);
    }
    if (sub == 0) {
      bool nan;
      if (ja < j1) {
        keys0[ja] = score_key(sa, nan);
        bad |= nan ? KSA_FLAG_NONFINITE_SCORE : 0u;
      }
      if (jc < j1) {
        keys0[jc] = score_key(sc, nan);
        bad |= nan ? KSA_FLAG_NONFINITE_SCORE : 0u;
      }
    }
  }
  flag_status(a.status, bad);
  cluster.sync();  // every key of the row is in rank 0's shared memory
  if (rank != 0) return;

  uint32_t tau, n_gt, n_eq;
  radix_select_desc<kSelThreads>(keys, nb, k, 32, hist, info, tau, n_gt, n_eq);
  select_ascending<kSelThreads>(keys, nb, tau, n_gt, n_eq, k, out, scratch, [](int) {});
  if (tid == 0) a.num_sel[row] = k;
}

}  // namespace

cudaError_t launch_select_blocks(const SelectArgs &a, int num_sms, cudaStream_t stream) {
  (void)num_sms;
  const int nb_max = (a.T + a.bs - 1) / a.bs;
  int csize = (nb_max + 255) / 256;
  csize = csize < 1 ? 1 : (csize > 8 ? 8 : csize);
  const size_t smem = static_cast<size_t>(nb_max) * sizeof(uint32_t);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.B) * a.Hkv * csize, 1, 1);
  cfg.blockDim = dim3(kSelThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err;
  if (a.D == 128) {
    err = cudaFuncSetAttribute(select_blocks_kernel<128>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    err = cudaLaunchKernelEx(&cfg, select_blocks_kernel<128>, a, csize);
  } else {
    err = cudaFuncSetAttribute(select_blocks_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    err = cudaLaunchKernelEx(&cfg, select_blocks_kernel<64>, a, csize);
  }
  return err;
}

}  // namespace ksa
