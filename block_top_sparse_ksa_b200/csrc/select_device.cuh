// select_device.cuh -- device pieces of block scoring and top-k selection,
// shared by the two-launch selection (select_blocks.cu) and the one-launch
// decode step (decode_step.cu).
//
// Kinetics (block top-k section): every block's mean key is scored against
// the query and the K' most relevant blocks are kept.  Reading of the
// relevance (the source gives no formula): the dot product of the block mean
// with the sum of the kv-group's query heads, one selection per kv-head.
#pragma once

#include "ksa_device.cuh"
#include "ksa_internal.h"

namespace ksa {
namespace sel {

constexpr int kPieceBytes = 8192;  // one piece: 2048 / D fp32 or 4096 / D bf16 summary rows
constexpr int kScThreads = 256;
constexpr int kRankWarpThreads = 128;
constexpr int kRankThreads = 256;

struct ScoreDev {
  SelectArgs a;
  const uint16_t *K;  // non-null: refresh the last block of each scored row from K
  uint32_t *keys;     // workspace [B*Hkv, nb_max]
  int prow;           // summary rows per piece
  int pieces;         // pieces per row: ceil(nb_max / prow)
  long long units;    // rows * pieces
  int N;              // CTAs in the grid
};

struct Piece {
  int row, b, g, L, nb, j0, n;  // blocks [j0, j0 + n) of the row; n == 0: nothing to score
};

// `report`: flag an out-of-range sequence length in the status word (once per row).
static __device__ __forceinline__ Piece piece_of(const ScoreDev &p, long long u, bool report = false) {
  Piece x;
  x.row = static_cast<int>(u / p.pieces);
  const int piece = static_cast<int>(u - static_cast<long long>(x.row) * p.pieces);
  x.b = x.row / p.a.Hkv;
  x.g = x.row - x.b * p.a.Hkv;
  x.L = clamp_len(p.a.seq_lens[x.b], p.a.T, (report && piece == 0) ? p.a.status : nullptr);
  x.nb = (x.L + p.a.bs - 1) / p.a.bs;
  x.j0 = piece * p.prow;
  x.n = (x.nb > p.a.k && x.j0 < x.nb) ? min(p.prow, x.nb - x.j0) : 0;
  return x;
}

// Re-averages block nb-1 of `row` from K and stores it in the summaries.
// Lanes l < D/8 get dims [8 (l % (D/8)), +8) in mean[] and return true.
// One whole warp.
template <int D>
__device__ __forceinline__ bool refresh_last_block(const SelectArgs &a, const uint16_t *K,
                                                   int row, int L, int nb, float (&mean)[8]) {
  const int nb_max = (a.T + a.bs - 1) / a.bs;
  const int jl = nb - 1;
  const int b = row / a.Hkv;
  const long long row0 = kv_row(a.kv, b, row - b * a.Hkv, a.Hkv, a.T,
                                static_cast<long long>(jl) * a.bs);
  bool mine;
  if (row0 < 0) {  // a page id that names no page: flagged, the block reads as zeros
    if ((threadIdx.x & 31) == 0) flag_status(a.status, KSA_FLAG_INDEX_SKIPPED);
#pragma unroll
    for (int i = 0; i < 8; ++i) mean[i] = 0.f;
    mine = (threadIdx.x & 31) < D / 8;
  } else {
    mine = warp_block_mean<D>(K + static_cast<size_t>(row0) * D, L - jl * a.bs, mean);
  }
  if (mine)
    store_mean8(a.S, a.sbf16, (static_cast<size_t>(row) * nb_max + jl) * D,
                ((threadIdx.x & 31) % (D / 8)) * 8, mean);
  return mine;
}

// Exact top-k of one row's nb (k < nb <= 32 KPL) score keys by one warp, the
// keys held in registers: lane l holds blocks l, l + 32, l + 64, ... so that
// (slot, lane) order is block order.  Radix select for the k-th largest key
// tau, 8 bits a pass from the highest bit in which the row's keys differ (the
// bits above are common to all): a 256-bin shared-memory histogram of the
// keys that match the digits fixed so far, then the bin where the count from
// the top reaches the number still to take.  Every key above tau is kept, and
// of the keys equal to tau the lowest-index ones, k in all; ballots give each
// winner its place, so out[0..k) comes out in ascending block order.
// `hist`: 256 words of this warp's shared memory, 16-byte aligned.
template <int KPL>
__device__ __forceinline__ void warp_topk(const uint32_t *krow, int nb, int k, int32_t *out,
                                          uint32_t *hist) {
  static_assert(KPL >= 1 && KPL <= 32, "the live-slot mask is one 32-bit word");
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;  // lanes below this one
  uint32_t key[KPL];
  uint32_t live = 0u;  // bit e: block lane + 32 e exists
  uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    const bool ok = lane + 32 * e < nb;
    key[e] = ok ? __ldcg(krow + lane + 32 * e) : 0u;
    live |= ok ? (1u << e) : 0u;
    if (ok) {
      kmin = min(kmin, key[e]);
      kmax = max(kmax, key[e]);
    }
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  uint32_t tau = kmin;                            // every key equal: tau is that key
  uint32_t remaining = static_cast<uint32_t>(k);  // keys still to take at or below tau
  if (kmin != kmax) {
    const int hb = 31 - __clz(kmin ^ kmax);  // highest bit in which keys differ
    uint32_t pmask = hb == 31 ? 0u : ~((2u << hb) - 1u);  // bits fixed so far
    uint32_t prefix = kmin & pmask;
    for (int shift = hb - 7;; shift -= 8) {
      const int sh = shift > 0 ? shift : 0;
      reinterpret_cast<uint4 *>(hist)[2 * lane] = make_uint4(0u, 0u, 0u, 0u);
      reinterpret_cast<uint4 *>(hist)[2 * lane + 1] = make_uint4(0u, 0u, 0u, 0u);
      __syncwarp();
#pragma unroll
      for (int e = 0; e < KPL; ++e) {
        if (((live >> e) & 1u) && (key[e] & pmask) == prefix)
          atomicAdd(&hist[(key[e] >> sh) & 255u], 1u);
      }
      __syncwarp();
      // lane l owns bins [8l, 8l + 8); counts from the top bin down
      const uint4 h0 = reinterpret_cast<const uint4 *>(hist)[2 * lane];
      const uint4 h1 = reinterpret_cast<const uint4 *>(hist)[2 * lane + 1];
      const uint32_t c[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
      const uint32_t tot = c[0] + c[1] + c[2] + c[3] + c[4] + c[5] + c[6] + c[7];
      uint32_t incl = tot;  // keys in the bins of lanes >= this lane
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, incl, off);
        if (lane + off < 32) incl += y;
      }
      uint32_t run = incl - tot, digit = 0u, above = 0u;
      bool found = false;
#pragma unroll
      for (int j = 7; j >= 0; --j) {
        const uint32_t before = run;
        run += c[j];
        if (before < remaining && run >= remaining) {
          found = true;
          digit = static_cast<uint32_t>(lane * 8 + j);
          above = before;
        }
      }
      const int src = __ffs(__ballot_sync(0xffffffffu, found)) - 1;
      digit = __shfl_sync(0xffffffffu, digit, src);
      above = __shfl_sync(0xffffffffu, above, src);
      remaining -= above;
      prefix = (prefix & ~(255u << sh)) | (digit << sh);
      pmask |= 255u << sh;
      __syncwarp();  // the bins are read before the next pass clears them
      if (sh == 0) break;
    }
    tau = prefix;
  }
  const uint32_t take_eq = remaining;  // k minus the keys above tau
  uint32_t base = 0u, eq_seen = 0u;
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    const bool ok = (live >> e) & 1u;
    const bool gt = ok && key[e] > tau, eq = ok && key[e] == tau;
    const uint32_t eb = __ballot_sync(0xffffffffu, eq);
    const bool sel = gt || (eq && eq_seen + __popc(eb & lt) < take_eq);
    eq_seen += __popc(eb);
    const uint32_t sb = __ballot_sync(0xffffffffu, sel);
    if (sel) out[base + __popc(sb & lt)] = lane + 32 * e;
    base += __popc(sb);
  }
}

// Exact top-k of one row's nb (k < nb <= NT KPL) score keys by a whole CTA
// of NT threads, keys in registers (thread t holds blocks t, t + NT, ... so
// that (slot, thread) order is block order).  The same radix select as
// warp_topk, block-wide: per pass, per-warp 256-bin shared histograms (fewer
// same-address atomics), summed by warp 0, which finds the digit.  Output: per
// slot, ballots and one exchange of per-warp counts give every winner its
// place, ascending.  Shared memory `sm`, 16-byte aligned: block_topk_words<NT>
// words (per-warp histograms, then two words per warp and two more).  All NT
// threads call it.
template <int NT>
__host__ __device__ constexpr int block_topk_words() {
  return (NT / 32) * 256 + 2 * (NT / 32) + 2;
}

template <int NT, int KPL>
__device__ __forceinline__ void block_topk(const uint32_t *krow, int nb, int k, int32_t *out,
                                           uint32_t *sm) {
  constexpr int NW = NT / 32;
  uint32_t(*hist)[256] = reinterpret_cast<uint32_t(*)[256]>(sm);
  uint32_t(*red)[NW] = reinterpret_cast<uint32_t(*)[NW]>(sm + NW * 256);
  uint32_t *xinfo = sm + NW * 256 + 2 * NW;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t key[KPL];
  uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    const int j = tid + NT * e;
    key[e] = j < nb ? __ldcg(krow + j) : 0u;
    if (j < nb) {
      kmin = min(kmin, key[e]);
      kmax = max(kmax, key[e]);
    }
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if (lane == 0) {
    red[0][warp] = kmin;
    red[1][warp] = kmax;
  }
  __syncthreads();
  kmin = red[0][0];
  kmax = red[1][0];
#pragma unroll
  for (int w = 1; w < NW; ++w) {
    kmin = min(kmin, red[0][w]);
    kmax = max(kmax, red[1][w]);
  }
  uint32_t tau = kmin;
  uint32_t remaining = static_cast<uint32_t>(k);  // keys still to take at or below tau
  if (kmin != kmax) {
    const int hb = 31 - __clz(kmin ^ kmax);
    uint32_t pmask = hb == 31 ? 0u : ~((2u << hb) - 1u);
    uint32_t prefix = kmin & pmask;
    for (int shift = hb - 7;; shift -= 8) {
      const int sh = shift > 0 ? shift : 0;
      for (int i = tid; i < NW * 256; i += NT) (&hist[0][0])[i] = 0u;
      __syncthreads();
#pragma unroll
      for (int e = 0; e < KPL; ++e) {
        if (tid + NT * e < nb && (key[e] & pmask) == prefix)
          atomicAdd(&hist[warp][(key[e] >> sh) & 255u], 1u);
      }
      __syncthreads();
      if (warp == 0) {  // lane l owns bins [8l, 8l + 8); counts from the top bin down
        uint32_t c[8];
        uint32_t tot = 0u;
#pragma unroll
        for (int jb = 0; jb < 8; ++jb) {
          uint32_t v = 0u;
#pragma unroll
          for (int w = 0; w < NW; ++w) v += hist[w][lane * 8 + jb];
          c[jb] = v;
          tot += v;
        }
        uint32_t incl = tot;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const uint32_t y = __shfl_down_sync(0xffffffffu, incl, off);
          if (lane + off < 32) incl += y;
        }
        uint32_t run = incl - tot;
#pragma unroll
        for (int jb = 7; jb >= 0; --jb) {
          const uint32_t before = run;
          run += c[jb];
          if (before < remaining && run >= remaining) {
            xinfo[0] = static_cast<uint32_t>(lane * 8 + jb);
            xinfo[1] = before;
          }
        }
      }
      __syncthreads();
      const uint32_t digit = xinfo[0];
      remaining -= xinfo[1];
      prefix = (prefix & ~(255u << sh)) | (digit << sh);
      pmask |= 255u << sh;
      __syncthreads();  // xinfo and the bins are read before the next pass
      if (sh == 0) break;
    }
    tau = prefix;
  }
  const uint32_t take_eq = remaining;
  uint32_t base = 0u, eq_seen = 0u;
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    const int j = tid + NT * e;
    const bool ok = j < nb;
    const bool gt = ok && key[e] > tau, eq = ok && key[e] == tau;
    const uint32_t eb = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) red[0][warp] = __popc(eb);
    __syncthreads();
    uint32_t eq_below = 0u, eq_tot = 0u;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const uint32_t v = red[0][w];
      eq_below += w < warp ? v : 0u;
      eq_tot += v;
    }
    const bool sel = gt || (eq && eq_seen + eq_below + __popc(eb & lt) < take_eq);
    eq_seen += eq_tot;
    const uint32_t sb = __ballot_sync(0xffffffffu, sel);
    if (lane == 0) red[1][warp] = __popc(sb);
    __syncthreads();
    uint32_t sel_below = 0u, sel_tot = 0u;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const uint32_t v = red[1][w];
      sel_below += w < warp ? v : 0u;
      sel_tot += v;
    }
    if (sel) out[base + sel_below + __popc(sb & lt)] = j;
    base += sel_tot;
  }
}

// A row with at most k blocks keeps them all (and -1 pads the list).
template <int D>
__device__ __forceinline__ void keep_all_blocks(const ScoreDev &p, int row, int L, int nb) {
  const int lane = threadIdx.x & 31;
  const SelectArgs &a = p.a;
  int32_t *out = a.block_idx + static_cast<size_t>(row) * a.k;
  for (int i = lane; i < a.k; i += 32) out[i] = i < nb ? i : -1;
  if (lane == 0) a.num_sel[row] = nb;
  if (p.K != nullptr && nb > 0) {
    float mean[8];
    refresh_last_block<D>(a, p.K, row, L, nb, mean);  // the step's maintenance still runs
  }
}

// Group query sum of kv-head g of batch row b over this lane's columns,
// summed over the heads in order.  The lane reads 16-byte chunks sub + 8 j of
// a summary row: 4 fp32 dims each (qv[j]), or with bf16 summaries 8 dims each
// (qv[2j], qv[2j+1]).  Either way qv covers D/8 dims in D/32 float4.
template <int D, bool SBF>
__device__ __forceinline__ void load_qsum(const SelectArgs &a, int b, int g, int sub,
                                          float4 (&qv)[D / 32]) {
  constexpr int NQ = D / 32;
  const int G = a.Hq / a.Hkv;
#pragma unroll
  for (int j = 0; j < NQ; ++j) qv[j] = make_float4(0.f, 0.f, 0.f, 0.f);
  const uint16_t *qg = a.q + (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(g) * G) * D;
#pragma unroll 4
  for (int h = 0; h < G; ++h) {
#pragma unroll
    for (int j = 0; j < NQ; ++j) {
      // dims 4 c .. 4 c + 3 with c the 4-dim group of qv[j]
      const int c4 = SBF ? 2 * (sub + 8 * (j >> 1)) + (j & 1) : sub + 8 * j;
      const uint32_t *q2 =
          reinterpret_cast<const uint32_t *>(qg + static_cast<size_t>(h) * D + 4 * c4);
      const uint32_t w0 = __ldg(q2), w1 = __ldg(q2 + 1);
      qv[j].x += bf16_lo(w0);
      qv[j].y += bf16_hi(w0);
      qv[j].z += bf16_lo(w1);
      qv[j].w += bf16_hi(w1);
    }
  }
}

// Scores piece x (x.n > 0) against the group query sum qv: the whole 8 KB
// piece is pulled into registers at once (lane (r, sub) holds chunks sub + 8 j
// of rows 4 it + r), each summary row is reduced over its 8 lanes, and the
// keys are stored.  With a key cache given, the piece holding the row's last
// block first re-averages that block, so the fresh value is the one scored.
template <int D, bool SBF>
__device__ __forceinline__ void score_piece(const ScoreDev &p, const Piece &x,
                                            const float4 (&qv)[D / 32], uint32_t &bad) {
  constexpr int RB = D * (SBF ? 2 : 4);  // bytes per summary row
  constexpr int R = kPieceBytes / RB;     // rows per piece
  constexpr int PER = RB / 16 / 8;        // 16-byte chunks per lane and row
  constexpr int IT = R / 4;
  const SelectArgs &a = p.a;
  const int lane = threadIdx.x & 31, sub = lane & 7;
  const int nb_max = (a.T + a.bs - 1) / a.bs;
  if (p.K != nullptr && x.j0 + x.n == x.nb) {
    float mean[8];
    refresh_last_block<D>(a, p.K, x.row, x.L, x.nb, mean);
    __syncwarp();  // the fresh summary is visible to the whole warp's loads below
  }
  const uint4 *src = reinterpret_cast<const uint4 *>(
      static_cast<const uint8_t *>(a.S) + (static_cast<size_t>(x.row) * nb_max + x.j0) * RB);
  uint4 v[IT][PER];
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int jr = it * 4 + (lane >> 3);
#pragma unroll
    for (int j = 0; j < PER; ++j)
      v[it][j] = jr < x.n ? __ldcg(src + jr * (RB / 16) + sub + 8 * j) : make_uint4(0u, 0u, 0u, 0u);
  }
  uint32_t *krow = p.keys + static_cast<size_t>(x.row) * nb_max + x.j0;
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int jr = it * 4 + (lane >> 3);
    float sc = 0.f;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const uint4 w = v[it][j];
      if (SBF) {
        const float4 qa = qv[2 * j], qb = qv[2 * j + 1];
        sc = fmaf(qa.x, bf16_lo(w.x), sc);
        sc = fmaf(qa.y, bf16_hi(w.x), sc);
        sc = fmaf(qa.z, bf16_lo(w.y), sc);
        sc = fmaf(qa.w, bf16_hi(w.y), sc);
        sc = fmaf(qb.x, bf16_lo(w.z), sc);
        sc = fmaf(qb.y, bf16_hi(w.z), sc);
        sc = fmaf(qb.z, bf16_lo(w.w), sc);
        sc = fmaf(qb.w, bf16_hi(w.w), sc);
      } else {
        sc = fmaf(qv[j].x, __uint_as_float(w.x), sc);
        sc = fmaf(qv[j].y, __uint_as_float(w.y), sc);
        sc = fmaf(qv[j].z, __uint_as_float(w.z), sc);
        sc = fmaf(qv[j].w, __uint_as_float(w.w), sc);
      }
    }
    sc += __shfl_xor_sync(0xffffffffu, sc, 1);
    sc += __shfl_xor_sync(0xffffffffu, sc, 2);
    sc += __shfl_xor_sync(0xffffffffu, sc, 4);
    if (jr < x.n && sub == 0) {
      bool nan;
      krow[jr] = score_key(sc, nan);
      bad |= nan ? KSA_FLAG_NONFINITE_SCORE : 0u;
    }
  }
}

}  // namespace sel
}  // namespace ksa
