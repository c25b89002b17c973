// select_device.cuh -- device pieces of block scoring and top-k selection.
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
// FMT: the summaries' storage format (a.sfmt), or -1 to read it at run time.
template <int D, int FMT = -1>
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
  const size_t n_blocks = static_cast<size_t>(a.B) * a.Hkv * nb_max;
  const size_t blk = static_cast<size_t>(row) * nb_max + jl;
  if (FMT < 0)
    store_block_mean_any<D>(a.S, a.sfmt, n_blocks, blk, mine, mean);
  else
    store_block_mean<D, (FMT < 0 ? 0 : FMT)>(a.S, n_blocks, blk, mine, mean);
  return mine;
}

// Shared-memory words of fast_topk<NT, KPL>: a 1024-bin histogram, the
// selected and the tied-candidate bitmaps (one bit per block), and 64 words
// for reductions and broadcasts.
template <int NT, int KPL>
__host__ __device__ constexpr int fast_topk_words() {
  return 1024 + 2 * ((NT * KPL + 31) / 32) + 64;  // misc: 8 + 3 * (NT / 32) <= 64 words
}

// The score an order-preserving key stands for (score_key's inverse); the key
// of a NaN score (0) gives -inf.
__device__ __forceinline__ float key_score(uint32_t key) {
  if (key == 0u) return -INFINITY;
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// Exact top-k of one row's n (k < n <= NT KPL) uint32 score keys by a CTA of
// NT threads (all of them call it), the keys in registers: thread t holds
// blocks t, t + NT, t + 2 NT, ...  Selection by shrinking ranges: a pass drops
// the live keys into 1024 buckets, the bucket holding the k-th largest live
// key is found from a histogram, keys in higher buckets are selected, in lower
// ones dropped, and the bucket's keys stay live.  The first pass buckets by
// score value over [min, max] (linear in the score, so continuous scores
// spread over many buckets and the boundary one holds a few); later passes
// bucket the live keys' range [lo, hi] by key bits, 2^s wide ((hi - lo) >> s <
// 1024), each 1024 times narrower.  Every bucket map is monotone in the key,
// so a higher bucket means a higher score.  Done when the live keys are
// exactly the ones still needed (usually after two passes), or all equal: then
// the lowest-index ones are taken (ties go to the lower block).  At most five
// passes.  The winners are written to out[0..k) in ascending block order
// through a bitmap of the selection and one prefix count over its words.
// `sm`: fast_topk_words words of shared memory, 16-byte aligned.
template <int NT, int KPL>
__device__ __forceinline__ void fast_topk(const uint32_t *krow, int n, int k, int32_t *out,
                                          uint32_t *sm) {
  static_assert(NT % 32 == 0 && NT >= 64 && NT <= 1024, "whole warps");
  static_assert(KPL >= 1 && KPL <= 64, "a 64-bit slot mask per thread");
  static_assert(8 + 3 * (NT / 32) <= 64, "the reduction words fit in misc");
  constexpr int NW = NT / 32;
  constexpr int W = (NT * KPL + 31) / 32;  // bitmap words; block j is bit j % 32 of word j / 32
  uint32_t *hist = sm;
  uint32_t *selw = sm + 1024;
  uint32_t *livew = selw + W;
  uint32_t *misc = livew + W;  // [0..3) the pass's bucket, count above, count in it; [8..) reductions
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t key[KPL];
  uint64_t live = 0ull, sel = 0ull;
  uint32_t lo = 0xffffffffu, hi = 0u, lo_real = 0xffffffffu;  // lo_real: over keys of real scores
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    const int j = tid + NT * e;
    key[e] = j < n ? __ldcg(krow + j) : 0u;
    if (j < n) {
      live |= 1ull << e;
      lo = min(lo, key[e]);
      hi = max(hi, key[e]);
      if (key[e] != 0u) lo_real = min(lo_real, key[e]);
    }
  }
  uint32_t remaining = static_cast<uint32_t>(k);  // winners still to find among the live keys
  for (int pass = 0;; ++pass) {
    // range of the live keys, block-wide
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    if (pass == 0) lo_real = __reduce_min_sync(0xffffffffu, lo_real);
    if (lane == 0) {
      misc[8 + warp] = lo;
      misc[8 + NW + warp] = hi;
      misc[8 + 2 * NW + warp] = lo_real;
    }
    __syncthreads();
    lo = misc[8];
    hi = misc[8 + NW];
    if (pass == 0) lo_real = misc[8 + 2 * NW];
#pragma unroll
    for (int w = 1; w < NW; ++w) {
      lo = min(lo, misc[8 + w]);
      hi = max(hi, misc[8 + NW + w]);
      if (pass == 0) lo_real = min(lo_real, misc[8 + 2 * NW + w]);
    }
    if (lo == hi || pass == 5) break;  // all live keys equal: the index rule decides
    // pass 0 by score value when the real scores span a finite, non-empty range
    const float v0 = key_score(lo_real), v1 = key_score(hi);
    const float vscale = 1024.f / (v1 - v0);
    const bool by_value = pass == 0 && lo_real < hi && isfinite(vscale) && vscale > 0.f;
    const int bits = 32 - __clz(hi - lo);
    const int sh = bits > 10 ? bits - 10 : 0;
    for (int i = tid; i < 1024; i += NT) hist[i] = 0u;
    __syncthreads();
#pragma unroll
    for (int e = 0; e < KPL; ++e) {
      if (!((live >> e) & 1ull)) continue;
      uint32_t bk;
      if (by_value) {  // NaN keys (0) and the lowest scores share bucket 0
        const float f = (key_score(key[e]) - v0) * vscale;
        bk = key[e] == 0u ? 0u : static_cast<uint32_t>(fminf(fmaxf(f, 0.f), 1023.f));
      } else {
        bk = (key[e] - lo) >> sh;
      }
      atomicAdd(&hist[bk], 1u);
    }
    __syncthreads();
    if (warp == 0) {  // lane l owns buckets [32 l, 32 l + 32); count from the top down
      uint32_t tot = 0u;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint4 v = reinterpret_cast<const uint4 *>(hist + 32 * lane)[q];
        tot += v.x + v.y + v.z + v.w;
      }
      uint32_t incl = tot;  // keys in the buckets of lanes >= this one
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, incl, off);
        if (lane + off < 32) incl += y;
      }
      // the one lane whose buckets hold the k-th live key; then the whole warp walks that
      // lane's 32 buckets from the top, one bucket per lane, with a prefix sum
      const int owner = __ffs(__ballot_sync(0xffffffffu, incl - tot < remaining &&
                                                             incl >= remaining)) - 1;
      const uint32_t above_owner = __shfl_sync(0xffffffffu, incl - tot, owner);
      const uint32_t c = hist[32 * owner + 31 - lane];
      uint32_t pre = c;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, pre, off);
        if (lane >= off) pre += y;
      }
      const int j = __ffs(__ballot_sync(0xffffffffu, above_owner + pre >= remaining)) - 1;
      if (lane == j) {
        misc[0] = static_cast<uint32_t>(32 * owner + 31 - j);
        misc[1] = above_owner + pre - c;
        misc[2] = c;
      }
    }
    __syncthreads();
    const uint32_t bstar = misc[0], above = misc[1], inb = misc[2];
    remaining -= above;
    const bool exact = inb == remaining;  // every live key of the bucket is needed
    const uint32_t base = lo;
    lo = 0xffffffffu;
    hi = 0u;
#pragma unroll
    for (int e = 0; e < KPL; ++e) {
      if (!((live >> e) & 1ull)) continue;
      uint32_t bk;
      if (by_value) {
        const float f = (key_score(key[e]) - v0) * vscale;
        bk = key[e] == 0u ? 0u : static_cast<uint32_t>(fminf(fmaxf(f, 0.f), 1023.f));
      } else {
        bk = (key[e] - base) >> sh;
      }
      if (bk > bstar || (bk == bstar && exact)) {
        sel |= 1ull << e;
        live &= ~(1ull << e);
      } else if (bk < bstar) {
        live &= ~(1ull << e);
      } else {
        lo = min(lo, key[e]);
        hi = max(hi, key[e]);
      }
    }
    __syncthreads();  // misc and the histogram are rewritten by the next pass
    if (exact) {
      remaining = 0u;
      break;
    }
  }
  // bitmaps of the selected and of the still-live (all equal) keys, in block order
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    const uint32_t sb = __ballot_sync(0xffffffffu, (sel >> e) & 1ull);
    const uint32_t lb = __ballot_sync(0xffffffffu, (live >> e) & 1ull);
    if (lane == 0) {
      selw[warp + NW * e] = sb;
      livew[warp + NW * e] = lb;
    }
  }
  __syncthreads();
  if (warp == 0) {
    // lane l owns words [WPL l, WPL l + WPL): the lowest-index `remaining` live keys join the
    // selection (written back into selw); then each word's place in the output (livew)
    constexpr int WPL = (W + 31) / 32;
    const int w0 = lane * WPL, w1 = min(w0 + WPL, W);
    uint32_t nl = 0u;
    for (int w = w0; w < w1; ++w) nl += __popc(livew[w]);
    uint32_t pl = nl;  // inclusive prefix of live bits over the lanes
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, pl, off);
      if (lane >= off) pl += y;
    }
    pl -= nl;
    uint32_t ns = 0u;
    for (int w = w0; w < w1; ++w) {
      uint32_t take = 0u, x = livew[w];
      if (pl + __popc(x) <= remaining) {  // the whole word
        take = x;
        pl += __popc(x);
        x = 0u;
      }
      while (x != 0u && pl < remaining) {  // lowest set bits first: ascending blocks
        const uint32_t b = x & (0u - x);
        take |= b;
        x ^= b;
        ++pl;
      }
      pl += __popc(x);
      const uint32_t sw = selw[w] | take;
      selw[w] = sw;
      ns += __popc(sw);
    }
    uint32_t ps = ns;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, ps, off);
      if (lane >= off) ps += y;
    }
    ps -= ns;
    for (int w = w0; w < w1; ++w) {
      livew[w] = ps;
      ps += __popc(selw[w]);
    }
  }
  __syncthreads();
  for (int w = tid; w < W; w += NT) {  // every thread writes the winners of its words
    uint32_t x = selw[w], pos = livew[w];
    while (x != 0u) {
      out[pos++] = 32 * w + (__ffs(x) - 1);
      x &= x - 1u;
    }
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
// a summary row: 4 fp32 dims each (qv[j]), with bf16 summaries 8 dims each
// (qv[2j], qv[2j+1]), with fp8 ones (D = 128: one chunk) 16 dims (qv[0..3]).
// Either way qv covers D/8 dims in D/32 float4.
template <int D, int FMT>
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
      const int c4 = FMT == KSA_SUMMARIES_FP8    ? 4 * sub + j
                     : FMT == KSA_SUMMARIES_BF16 ? 2 * (sub + 8 * (j >> 1)) + (j & 1)
                                                 : sub + 8 * j;
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
template <int D, int FMT>
__device__ __forceinline__ void score_piece(const ScoreDev &p, const Piece &x,
                                            const float4 (&qv)[D / 32], uint32_t &bad) {
  static_assert(FMT != KSA_SUMMARIES_FP8 || D == 128, "fp8 rows are one 16-byte chunk per lane");
  constexpr int RB = D * (FMT == KSA_SUMMARIES_F32 ? 4 : FMT == KSA_SUMMARIES_BF16 ? 2 : 1);
  constexpr int R = kPieceBytes / RB;     // rows per piece
  constexpr int PER = RB / 16 / 8;        // 16-byte chunks per lane and row
  constexpr int IT = R / 4;
  const SelectArgs &a = p.a;
  const int lane = threadIdx.x & 31, sub = lane & 7;
  const int nb_max = (a.T + a.bs - 1) / a.bs;
  if (p.K != nullptr && x.j0 + x.n == x.nb) {
    float mean[8];
    refresh_last_block<D, FMT>(a, p.K, x.row, x.L, x.nb, mean);
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
  // fp8: the piece's block scales, row jr's in lane jr % 32 of sa (jr < 32) or sb
  float sa = 1.f, sb = 1.f;
  if (FMT == KSA_SUMMARIES_FP8) {
    const float *scales = reinterpret_cast<const float *>(
        static_cast<const uint8_t *>(a.S) + static_cast<size_t>(a.B) * a.Hkv * nb_max * D);
    const size_t s0 = static_cast<size_t>(x.row) * nb_max + x.j0;
    if (lane < x.n) sa = __ldcg(scales + s0 + lane);
    if (32 + lane < x.n) sb = __ldcg(scales + s0 + 32 + lane);
  }
  uint32_t *krow = p.keys + static_cast<size_t>(x.row) * nb_max + x.j0;
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int jr = it * 4 + (lane >> 3);
    float sc = 0.f;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const uint4 w = v[it][j];
      if (FMT == KSA_SUMMARIES_FP8) {
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {  // dims 16 sub + 4 c .. + 3
          const float2 lo = e4m3x2_to_float2(static_cast<uint16_t>(ww[c] & 0xffffu));
          const float2 hi = e4m3x2_to_float2(static_cast<uint16_t>(ww[c] >> 16));
          sc = fmaf(qv[c].x, lo.x, sc);
          sc = fmaf(qv[c].y, lo.y, sc);
          sc = fmaf(qv[c].z, hi.x, sc);
          sc = fmaf(qv[c].w, hi.y, sc);
        }
      } else if (FMT == KSA_SUMMARIES_BF16) {
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
    if (FMT == KSA_SUMMARIES_FP8) {  // the stored values times the block's scale (exact)
      const float ga = __shfl_sync(0xffffffffu, sa, jr & 31);
      const float gb = __shfl_sync(0xffffffffu, sb, jr & 31);
      sc *= jr < 32 ? ga : gb;
    }
    if (jr < x.n && sub == 0) {
      bool nan;
      krow[jr] = score_key(sc, nan);
      bad |= nan ? KSA_FLAG_NONFINITE_SCORE : 0u;
    }
  }
}

}  // namespace sel
}  // namespace ksa
