// select_blocks.cu -- block scoring and top-k block selection.
//
// Kinetics (block top-k section): every block's mean key is scored against the
// query and the K' most relevant blocks are kept.  Reading of the relevance
// (the source gives no formula): the dot product of the block mean with the
// sum of the kv-group's query heads, one selection per kv-head.
//
// Two launches:
//  1. scoring, persistent.  The summaries of every (row b, kv-head g) are cut
//     into pieces of 8 KB (2048 / D consecutive blocks of D fp32, or 4096 / D
//     of D bf16, contiguous); each row is padded to the same number of pieces
//     and the grid's warps take equal contiguous slices of the flat piece
//     sequence, so a warp streams one region front to back and forms each
//     row's group query sum once.  (A partition over the rows' real pieces
//     only, which evens out warps' bytes when lengths differ, measured 3 us
//     slower on the 16K-32K batch.)  A warp pulls a whole piece into registers with 16-byte
//     loads (all in flight at once), then scores it -- 8 lanes per summary
//     row, warp shuffles -- and stores order-preserving uint32 keys in the
//     workspace.  No shared memory, no barriers.  Pieces of rows with at most
//     k blocks are skipped: nothing is read.
//  2. ranking: one CTA per (row, kv-head) holds the row's keys (just written,
//     in L2) in registers and runs fast_topk: histogram passes over shrinking
//     key ranges (usually two) find the k best, ties at the threshold going
//     to the lower block, and a bitmap of the winners gives their places in
//     ascending block order.  Rows with at most k blocks keep every block.
//
// With a key cache given (the fused decode-step entry point), the last block
// of every row is first re-averaged from the keys -- the per-step maintenance
// of the block representation: by the warp whose piece holds it, before it
// reads the piece (so the fresh value is scored), or by the ranking warp or
// CTA for rows whose blocks are all kept.
#include <string.h>

#include "ksa_device.cuh"
#include "ksa_internal.h"
#include "select_device.cuh"

namespace ksa {

using namespace sel;

namespace {

// The scoring kernel's format for fp8 summaries: fp8 at D = 128; other head
// sizes never reach it (the API refuses fp8 there), so they map to fp32.
template <int D>
constexpr int kFp8For = D == 128 ? KSA_SUMMARIES_FP8 : KSA_SUMMARIES_F32;

// Scoring.  The grid's warps take equal contiguous slices of the flat piece
// sequence: a warp streams one region of the summaries front to back (the
// pattern the DRAM serves best, measured against round-robin and
// counter-driven orders) and forms each row's group query sum once.
template <int D, int FMT>
__global__ void __launch_bounds__(kScThreads) score_blocks_kernel(const ScoreDev p) {
  constexpr int kWarps = kScThreads / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, sub = lane & 7;
  pdl_wait();
  pdl_launch_dependents();
  uint32_t bad = 0u;
  int qrow = -1;  // row whose group query sum qv holds
  float4 qv[D / 32];
  const long long NW = static_cast<long long>(p.N) * kWarps;
  const long long gw = static_cast<long long>(blockIdx.x) * kWarps + warp;
  const long long s0 = gw * p.units / NW, s1 = (gw + 1) * p.units / NW;
  for (long long u = s0; u < s1; ++u) {  // warp-uniform control flow throughout
    const Piece x = piece_of(p, u);
    if (x.n == 0) continue;
    if (x.row != qrow) {
      qrow = x.row;
      load_qsum<D, FMT>(p.a, x.b, x.g, sub, qv);
    }
    score_piece<D, FMT>(p, x, qv, bad);
  }
  bad = __reduce_or_sync(0xffffffffu, bad);
  if (bad != 0u && lane == 0) flag_status(p.a.status, bad);
}

// Ranking, one CTA of NT threads per (row, kv-head): the row's keys (just
// written, in L2) go into registers and fast_topk keeps the k best.  Rows with
// at most k blocks keep every block.
template <int D, int NT, int KPL>
__global__ void __launch_bounds__(NT) rank_rows_kernel(const ScoreDev p) {
  __shared__ __align__(16) uint32_t sm[fast_topk_words<NT, KPL>()];
  pdl_wait();
  pdl_launch_dependents();
  const SelectArgs &a = p.a;
  const int row = blockIdx.x;
  const int nb_max = (a.T + a.bs - 1) / a.bs;
  const int L = clamp_len(a.seq_lens[row / a.Hkv], a.T, threadIdx.x == 0 ? a.status : nullptr);
  const int nb = (L + a.bs - 1) / a.bs;
  if (nb <= a.k) {
    if (threadIdx.x < 32) keep_all_blocks<D>(p, row, L, nb);
    return;
  }
  fast_topk<NT, KPL>(p.keys + static_cast<size_t>(row) * nb_max, nb, a.k,
                     a.block_idx + static_cast<size_t>(row) * a.k, sm);
  if (threadIdx.x == 0) a.num_sel[row] = a.k;
}

// Local attention as a block selection: every (row, kv-head) keeps its last
// min(k, NB_b) blocks, ascending, -1 padded.  One thread per output slot.
__global__ void __launch_bounds__(256) window_blocks_kernel(const SelectArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= static_cast<long long>(a.B) * a.Hkv * a.k) return;
  const int row = static_cast<int>(e / a.k), i = static_cast<int>(e % a.k);
  const int b = row / a.Hkv;
  const int L = clamp_len(a.seq_lens[b], a.T,
                          (i == 0 && row == b * a.Hkv) ? a.status : nullptr);
  const int nb = (L + a.bs - 1) / a.bs;
  const int n = min(a.k, nb);
  a.block_idx[e] = i < n ? nb - n + i : -1;
  if (i == 0) a.num_sel[row] = n;
}

template <int D>
cudaError_t launch_select(const ScoreDev &p0, int num_sms, cudaStream_t stream) {
  ScoreDev p = p0;
  const SelectArgs &a = p.a;
  const int nb_max = (a.T + a.bs - 1) / a.bs;
  const int rows = a.B * a.Hkv;
  cudaError_t err;
  if (nb_max > a.k) {  // otherwise no row has a block to score
    const auto kern = a.sfmt == KSA_SUMMARIES_BF16 ? score_blocks_kernel<D, KSA_SUMMARIES_BF16>
                      : a.sfmt == KSA_SUMMARIES_FP8 ? score_blocks_kernel<D, kFp8For<D>>
                                                    : score_blocks_kernel<D, KSA_SUMMARIES_F32>;
    int per_sm = 0;
    err = kernel_occupancy(reinterpret_cast<const void *>(kern), kScThreads, 0, &per_sm);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) per_sm = 1;
    constexpr int kWarps = kScThreads / 32;
    long long n = static_cast<long long>(num_sms) * per_sm;
    const long long need = (p.units + kWarps - 1) / kWarps;
    if (n > need) n = need;
    p.N = static_cast<int>(n);
    err = launch_pdl(kern, dim3(static_cast<unsigned>(p.N)), dim3(kScThreads), 0, stream, p);
    if (err != cudaSuccess) return err;
  }
  // one CTA per row; its threads hold the row's keys in registers
  const dim3 grid(static_cast<unsigned>(rows));
  if (nb_max <= 512) return launch_pdl(rank_rows_kernel<D, 128, 4>, grid, dim3(128), 0, stream, p);
  if (nb_max <= 1024) return launch_pdl(rank_rows_kernel<D, 128, 8>, grid, dim3(128), 0, stream, p);
  if (nb_max <= 2048) return launch_pdl(rank_rows_kernel<D, 256, 8>, grid, dim3(256), 0, stream, p);
  if (nb_max <= 4096) return launch_pdl(rank_rows_kernel<D, 256, 16>, grid, dim3(256), 0, stream, p);
  if (nb_max <= 8192) return launch_pdl(rank_rows_kernel<D, 256, 32>, grid, dim3(256), 0, stream, p);
  // (nb_max <= 16384 is checked by the API)
  return launch_pdl(rank_rows_kernel<D, 256, 64>, grid, dim3(256), 0, stream, p);
}

}  // namespace

// workspace: a leading region of one word per row plus two (reserved: zero)
// + score keys [B*Hkv, nb_max]
cudaError_t launch_select_window(const SelectArgs &a, cudaStream_t stream) {
  const long long n = static_cast<long long>(a.B) * a.Hkv * a.k;
  return launch_pdl(window_blocks_kernel, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256),
                    0, stream, a);
}

size_t select_workspace_bytes(int B, int Hkv, int T, int bs) {
  const size_t rows = static_cast<size_t>(B) * Hkv;
  const size_t nb_max = static_cast<size_t>((T + bs - 1) / bs);
  const size_t sems = ((rows + 2) * sizeof(int32_t) + 255) & ~static_cast<size_t>(255);
  const size_t keys = (rows * nb_max * sizeof(uint32_t) + 255) & ~static_cast<size_t>(255);
  return sems + keys;
}

cudaError_t launch_select_blocks(const SelectArgs &a, const uint16_t *K, void *ws, int num_sms,
                                 cudaStream_t stream) {
  const int nb_max = (a.T + a.bs - 1) / a.bs;
  const size_t rows = static_cast<size_t>(a.B) * a.Hkv;
  const size_t sems = ((rows + 2) * sizeof(int32_t) + 255) & ~static_cast<size_t>(255);
  ScoreDev p;
  memset(&p, 0, sizeof(p));
  p.a = a;
  p.K = K;
  p.keys = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) + sems);
  p.prow = kPieceBytes / (a.D * (a.sfmt == KSA_SUMMARIES_F32    ? 4
                                  : a.sfmt == KSA_SUMMARIES_BF16 ? 2
                                                                 : 1));
  p.pieces = (nb_max + p.prow - 1) / p.prow;
  p.units = static_cast<long long>(rows) * p.pieces;
  p.N = 1;
  return a.D == 128 ? launch_select<128>(p, num_sms, stream) : launch_select<64>(p, num_sms, stream);
}

}  // namespace ksa
