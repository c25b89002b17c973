// decode_step.cu -- one decode step of block top-k sparse attention in one launch.
//
// Kinetics (block top-k section): at every step the block representation is
// kept current, every block is scored against the query, the K' best blocks
// are kept, and attention runs over their tokens only.  The two-call form
// (ksa_decode_select_blocks, then ksa_sparse_decode_attn) takes three launches
// per step -- scoring, ranking, attention -- and at decode batch sizes each
// launch's ramp and tail, the gaps between them and the latency-bound ranking
// launch are a large share of the step.  Here the three run as phases of one
// cooperative, persistent launch (every CTA resident at once, so CTAs may wait
// for one another; every wait is bounded):
//  1. scoring: the CTA's five warps each take an equal contiguous slice of the
//     flat sequence of 8 KB summary pieces -- the same pieces, the same fused
//     last-block refresh and the same arithmetic as the scoring kernel;
//  2. a grid-wide barrier: every score key is written;
//  3. ranking: row r goes to CTA r % N (N CTAs), whose threads hold its keys
//     in registers and run the ranking kernel's fast_topk; the CTA writes the
//     ascending list and the count and publishes the row (release) tagged
//     with this launch's epoch;
//  4. attention: the attention kernel's own stream-K partition and pipeline;
//     each CTA first waits (acquire) until every row it reads is published.
// The attention grid is the attention kernel's (same CTA shape, shared memory
// and occupancy), so the results equal the two calls' bit for bit.  Rows of
// more than 2048 blocks (more keys than the CTA ranks from registers) take the
// two-launch path.
#include <string.h>

#include "attn_device.cuh"
#include "ksa_device.cuh"
#include "ksa_internal.h"
#include "select_device.cuh"

namespace ksa {

namespace {

using att::AttnDev;
using sel::ScoreDev;

constexpr int kStepThreads = att::kAttnThreads;  // 4 consumer warps + 1 producer warp
constexpr int kStepWarps = kStepThreads / 32;
constexpr int kMaxFusedBlocks = 2048;  // longest row the one-launch ranking holds in registers

// Flags and barrier words of the step, in the leading (reserved) region of the
// selection part of the workspace.
struct StepDev {
  uint32_t *ready;  // [B*Hkv]: the epoch of the launch that published the row
  uint32_t *bar;    // [2]: grid barrier (arrivals, generation)
};

template <int D, bool SBF, int RK>
__global__ void __launch_bounds__(kStepThreads, 3)
    decode_step_kernel(const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap vmap, const ScoreDev sp,
                       const AttnDev ap, const StepDev st) {
  extern __shared__ uint8_t smem_raw[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, sub = lane & 7;
  const SelectArgs &a = sp.a;

  // ---- 1. scoring (warp-uniform control flow)
  {
    uint32_t bad = 0u;
    int qrow = -1;
    float4 qv[D / 32];
    const long long NW = static_cast<long long>(gridDim.x) * kStepWarps;
    const long long gw = static_cast<long long>(blockIdx.x) * kStepWarps + warp;
    int pcs[sel::kWalkPerLane];
    sel::PieceWalk walk = sel::walk_begin(sp, pcs);
    const long long u0 = gw * walk.total / NW, u1 = (gw + 1) * walk.total / NW;
    if (walk.compact && u0 < u1) sel::walk_seek(sp, walk, pcs, u0);
    for (long long u = u0; u < u1; ++u) {
      const sel::Piece x = sel::walk_next(sp, walk, u);
      if (x.n == 0) continue;
      if (x.row != qrow) {
        qrow = x.row;
        sel::load_qsum<D, SBF>(a, x.b, x.g, sub, qv);
      }
      sel::score_piece<D, SBF>(sp, x, qv, bad);
    }
    bad = __reduce_or_sync(0xffffffffu, bad);
    if (bad != 0u && lane == 0) flag_status(a.status, bad);
  }

  // ---- 2. every key written
  uint32_t epoch = 0u;
  if (!grid_barrier(st.bar, a.status, &epoch)) return;  // flagged; rows stay unpublished

  // ---- 3. ranking: one CTA per row; its shared memory lies in the stage buffers, which
  // are unused until phase 4
  {
    static_assert(sel::fast_topk_words<kStepThreads, RK>() * 4 <= 8 * 4096,
                  "the ranking's shared arrays fit in the stage buffers");
    uint32_t *sm = reinterpret_cast<uint32_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int rows = a.B * a.Hkv;
    const int nb_max = (a.T + a.bs - 1) / a.bs;
    for (int row = blockIdx.x; row < rows; row += static_cast<int>(gridDim.x)) {
      const int L =
          clamp_len(a.seq_lens[row / a.Hkv], a.T, threadIdx.x == 0 ? a.status : nullptr);
      const int nb = (L + a.bs - 1) / a.bs;
      if (nb <= a.k) {
        if (warp == 0) sel::keep_all_blocks<D>(sp, row, L, nb);
      } else {
        sel::fast_topk<kStepThreads, RK>(sp.keys + static_cast<size_t>(row) * nb_max, nb, a.k,
                                         a.block_idx + static_cast<size_t>(row) * a.k, sm);
        if (threadIdx.x == 0) a.num_sel[row] = a.k;
      }
      __threadfence();  // this thread's list entries before the publication
      __syncthreads();  // (also: the shared arrays are free for the next row)
      if (threadIdx.x == 0) st_release_gpu(st.ready + row, epoch);
    }
    fence_proxy_async_smem();  // the ranking's shared stores before the TMA writes that follow
  }
  __syncthreads();

  // ---- 4. attention over the kept blocks
  att::attn_cta<D, att::kModeTma, true>(kmap, vmap, ap, smem_raw, st.ready, epoch);
}

template <int D, bool SBF>
cudaError_t launch_fused(const CUtensorMap &km, const CUtensorMap &vm, const ScoreDev &sp,
                         AttnDev ap, const StepDev &st, int nb_max, int num_sms,
                         cudaStream_t stream, bool *launched) {
  const void *fn;
  void (*k4)(CUtensorMap, CUtensorMap, ScoreDev, AttnDev, StepDev) = nullptr;
  if (nb_max <= 4 * kStepThreads) k4 = decode_step_kernel<D, SBF, 4>;
  else if (nb_max <= 8 * kStepThreads) k4 = decode_step_kernel<D, SBF, 8>;
  else k4 = decode_step_kernel<D, SBF, (kMaxFusedBlocks + kStepThreads - 1) / kStepThreads>;
  fn = reinterpret_cast<const void *>(k4);
  const size_t smem = att::attn_smem_bytes(D, ap.gw);
  int occ = 0;
  cudaError_t err = kernel_occupancy(fn, kStepThreads, smem, &occ);
  if (err != cudaSuccess) return err;
  if (occ < 1) return cudaSuccess;  // cannot be resident: the caller takes two launches
  if (occ > kAttnMaxCtasPerSm) occ = kAttnMaxCtasPerSm;
  long long n = static_cast<long long>(num_sms) * occ;
  if (n > ap.W) n = ap.W;
  if (n < 1) n = 1;
  ap.N = static_cast<int>(n);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ap.N));
  cfg.blockDim = dim3(kStepThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  err = cudaLaunchKernelEx(&cfg, k4, km, vm, sp, ap, st);
  if (err == cudaErrorCooperativeLaunchTooLarge) {
    (void)cudaGetLastError();  // not every CTA fits now: the caller takes two launches
    return cudaSuccess;
  }
  if (err == cudaSuccess) *launched = true;
  return err;
}

}  // namespace

size_t decode_step_workspace_bytes(int B, int Hq, int Hkv, int D, int T, int bs, int num_sms) {
  return select_workspace_bytes(B, Hkv, T, bs) + attn_workspace_bytes(B, Hq, Hkv, D, num_sms);
}

cudaError_t launch_decode_step(const SelectArgs &sa, const uint16_t *K, const AttnArgs &aa,
                               void *ws, int num_sms, cudaStream_t stream) {
  const size_t sel_bytes = select_workspace_bytes(sa.B, sa.Hkv, sa.T, sa.bs);
  void *ws_att = static_cast<uint8_t *>(ws) + sel_bytes;
  const int nb_max = (sa.T + sa.bs - 1) / sa.bs;
  if (nb_max <= kMaxFusedBlocks) {
    const size_t rows = static_cast<size_t>(sa.B) * sa.Hkv;
    const size_t lead = ((rows + 2) * sizeof(int32_t) + 255) & ~static_cast<size_t>(255);
    ScoreDev sp;
    memset(&sp, 0, sizeof sp);
    sp.a = sa;
    sp.K = K;
    sp.keys = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) + lead);
    sp.prow = sel::kPieceBytes / (sa.D * (sa.sbf16 ? 2 : 4));
    sp.pieces = (nb_max + sp.prow - 1) / sp.prow;
    sp.units = static_cast<long long>(rows) * sp.pieces;
    sp.N = 1;
    StepDev st;
    st.ready = static_cast<uint32_t *>(ws);
    st.bar = st.ready + rows;
    CUtensorMap km, vm;
    AttnDev ap;
    int mode = 0;
    if (!att::attn_prepare(aa, ws_att, &km, &vm, &ap, &mode)) return cudaErrorInvalidValue;
    bool launched = false;
    cudaError_t err;
    if (sa.D == 128)
      err = sa.sbf16 ? launch_fused<128, true>(km, vm, sp, ap, st, nb_max, num_sms, stream, &launched)
                     : launch_fused<128, false>(km, vm, sp, ap, st, nb_max, num_sms, stream, &launched);
    else
      err = sa.sbf16 ? launch_fused<64, true>(km, vm, sp, ap, st, nb_max, num_sms, stream, &launched)
                     : launch_fused<64, false>(km, vm, sp, ap, st, nb_max, num_sms, stream, &launched);
    if (err != cudaSuccess || launched) return err;
  }
  // long rows (or no room for a cooperative grid): the two-launch form, same results
  cudaError_t err = launch_select_blocks(sa, K, ws, num_sms, stream);
  if (err != cudaSuccess) return err;
  return launch_sparse_decode_attn(aa, ws_att, num_sms, stream);
}

}  // namespace ksa
