// unified_select.cu -- LessIsMore unified token selection.
//
// LessIsMore (unified head selection, stable recency window; token selection
// layer): every query head ranks all cached tokens, each head votes for its
// top tokens, the votes are pooled into one token set shared by all heads,
// and the budget is split between voted tokens and the most recent tokens.
//
// Launches on the caller's stream (four when every row has at most 24576 tokens:
// the votes get a kernel of their own; three otherwise):
//  1. scores: one CTA per (row, kv-head, 1024-token chunk).  A producer warp
//     streams the chunk's keys with TMA (128B swizzle); four consumer warps
//     form S^T = K_tile q^T for the kv-group's G heads with mma.sync
//     (fp32 accumulate) and store order-preserving uint32 score keys
//     [B, Hq, T].  The g == 0 CTAs also clear the vote table.
//  2. per-head picks: one CTA per (row, query head).  Exact radix select of the
//     P-th largest key over the row's L keys, ties at the threshold to the
//     lower token.  Rows of up to 24576 tokens keep their keys in registers,
//     run an adaptive radix (each pass starts at the highest bit in which the
//     remaining candidates differ) and write the picks as bit sets, from which
//     a per-token kernel then counts the votes (2b); longer rows stage the keys
//     in shared memory and add one atomic vote per pick.
//  3. shared set: one CTA per row.  Radix select on the vote counts of
//     [0, L - R) for the (budget - R) most voted tokens (ties to the lower
//     token), written ascending, followed by the window [L - R, L).
#include <string.h>

#include "ksa_device.cuh"
#include "ksa_internal.h"

namespace ksa {

namespace {

constexpr int kTok = 32;            // tokens per pipeline stage
constexpr int kChunk = 1024;        // tokens per scoring CTA
constexpr int kScoreThreads = 160;  // 4 consumer warps + 1 producer warp
constexpr int kPickThreads = 512;
constexpr int kPickRegThreads = 256;  // picks with the row's keys in registers
constexpr int kPickRegMaxKeys = 96;   // keys per thread of that kernel (rows <= 24576 tokens)
constexpr int kSetThreads = 1024;
constexpr int kSmemKeys = 40960;    // keys of one head staged in shared memory

template <int D>
struct SCfg {
  static constexpr int kHalves = D / 64;
  static constexpr int kHalfBytes = kTok * 128;
  static constexpr int kStageBytes = kHalves * kHalfBytes;
  static constexpr int kStages = 8;  // multiple of the 4 consumer warps: one owner per buffer
  static_assert(kStages % 4 == 0, "stage buffers must map to one consumer warp each");
  static constexpr size_t kSmemBytes =
      1024 + static_cast<size_t>(kStages) * kStageBytes + 16 * kStages + 64;
};

template <int D>
__global__ void __launch_bounds__(kScoreThreads, 2)
    unified_scores_kernel(const __grid_constant__ CUtensorMap kmap, const UnifiedArgs a,
                          int n_chunks) {
  using C = SCfg<D>;
  constexpr int NS = C::kStages;
  constexpr int KT = D / 16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + static_cast<size_t>(NS) * C::kStageBytes);
  uint64_t *empty = full + NS;
  uint32_t *timed_out = reinterpret_cast<uint32_t *>(empty + NS);

  const int row = blockIdx.x / n_chunks, chunk = blockIdx.x % n_chunks;
  const int b = row / a.Hkv, g = row % a.Hkv;
  const int G = a.Hq / a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();
  pdl_launch_dependents();
  const int L = clamp_len(a.seq_lens[b], a.T,
                          (g == 0 && chunk == 0 && tid == 0) ? a.status : nullptr);
  if (L <= a.budget) return;  // every token is selected; no scores needed
  const int t_begin = chunk * kChunk;
  if (t_begin >= L) return;
  const int t_end = min(L, t_begin + kChunk);
  const int n_stage = (t_end - t_begin + kTok - 1) / kTok;

  if (g == 0) {
    for (int t = t_begin + tid; t < t_end; t += kScoreThreads)
      a.votes[static_cast<size_t>(b) * a.T + t] = 0;
  }
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1u);
      mbar_init(&empty[s], 1u);
    }
    *timed_out = 0u;
    fence_mbar_init();
  }
  __syncthreads();

  uint32_t bad = 0u;
  int issued = 0;
  if (warp == 4) {
    if (lane == 0) {
      for (int i = 0; i < n_stage; ++i) {
        const int buf = i % NS;
        if (i >= NS && !mbar_wait(&empty[buf], static_cast<uint32_t>((i / NS) - 1) & 1u)) {
          bad |= KSA_FLAG_WAIT_TIMEOUT;
          break;
        }
        issued = i + 1;
        uint8_t *dst = smem + static_cast<size_t>(buf) * C::kStageBytes;
        mbar_arrive_expect_tx(&full[buf], C::kStageBytes);
        const int y = static_cast<int>(static_cast<long long>(row) * a.T + t_begin + i * kTok);
#pragma unroll
        for (int h = 0; h < C::kHalves; ++h)
          tma_load_2d(dst + h * C::kHalfBytes, &kmap, h * 64, y, &full[buf]);
      }
    }
  } else {
    const int gid = lane >> 2, tig = lane & 3;
    uint32_t qb[KT][2];
    const uint16_t *qrow =
        a.q + (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(g) * G + gid) * D;
#pragma unroll
    for (int ks = 0; ks < KT; ++ks) {
      qb[ks][0] = gid < G ? *reinterpret_cast<const uint32_t *>(qrow + ks * 16 + tig * 2) : 0u;
      qb[ks][1] = gid < G ? *reinterpret_cast<const uint32_t *>(qrow + ks * 16 + 8 + tig * 2) : 0u;
    }
    const int mi = lane >> 3, lr = lane & 7;
    for (int i = warp; i < n_stage; i += 4) {
      const int buf = i % NS;
      if (!__all_sync(0xffffffffu, mbar_wait(&full[buf], static_cast<uint32_t>(i / NS) & 1u))) {
        bad |= KSA_FLAG_WAIT_TIMEOUT;
        break;
      }
      const uint32_t kbase = smem_addr(smem + static_cast<size_t>(buf) * C::kStageBytes);
      float s[2][4];
#pragma unroll
      for (int tile = 0; tile < 2; ++tile) {
        s[tile][0] = s[tile][1] = s[tile][2] = s[tile][3] = 0.f;
        const int r = tile * 16 + lr + ((mi & 1) << 3);
#pragma unroll
        for (int ks = 0; ks < KT; ++ks) {
          const int d = ks * 16 + ((mi >> 1) << 3);
          uint32_t af[4];
          ldsm_x4(af, kbase + (d >> 6) * C::kHalfBytes + swz128(r, (d & 63) >> 3));
          mma_16816(s[tile], af, qb[ks][0], qb[ks][1]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[buf]);
      const int t0 = t_begin + i * kTok;
#pragma unroll
      for (int tile = 0; tile < 2; ++tile) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int hh = tig * 2 + (c & 1);
          const int t = t0 + tile * 16 + gid + ((c >> 1) << 3);
          if (hh < G && t < t_end) {
            bool nan;
            const uint32_t key = score_key(s[tile][c], nan);
            bad |= nan ? KSA_FLAG_NONFINITE_SCORE : 0u;
            a.keys[(static_cast<size_t>(b) * a.Hq + static_cast<size_t>(g) * G + hh) * a.T + t] = key;
          }
        }
      }
    }
  }
  flag_status(a.status, bad);
  if (bad & KSA_FLAG_WAIT_TIMEOUT) atomicExch(timed_out, 1u);
  __syncthreads();
  if (*timed_out != 0u && warp == 4 && lane == 0) {
    // a wait gave up: let the issued copies land before the CTA exits (bounded)
    for (int buf = 0; buf < NS && buf < issued; ++buf)
      mbar_wait(&full[buf], static_cast<uint32_t>((issued - 1 - buf) / NS) & 1u);
  }
}

// Per-head pick and vote: CTA per (row, query head).
__global__ void __launch_bounds__(kPickThreads) unified_pick_kernel(const UnifiedArgs a,
                                                                     int stage_in_smem) {
  extern __shared__ uint32_t skeys[];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t info[4];
  __shared__ uint32_t scratch[33];
  const int b = blockIdx.x / a.Hq, h = blockIdx.x % a.Hq;
  pdl_wait();
  pdl_launch_dependents();
  const int L = clamp_len(a.seq_lens[b], a.T, nullptr);
  if (L <= a.budget) return;
  int32_t *votes = a.votes + static_cast<size_t>(b) * a.T;
  if (a.P >= L) {
    for (int t = threadIdx.x; t < L; t += kPickThreads) atomicAdd(&votes[t], 1);
    return;
  }
  const uint32_t *gkeys = a.keys + (static_cast<size_t>(b) * a.Hq + h) * a.T;
  const uint32_t *keys = gkeys;
  if (stage_in_smem) {
    for (int t = threadIdx.x; t < L; t += kPickThreads) skeys[t] = gkeys[t];
    __syncthreads();
    keys = skeys;
  }
  uint32_t tau, n_gt, n_eq;
  radix_select_desc<kPickThreads>(keys, L, a.P, 32, hist, info, tau, n_gt, n_eq);
  select_ascending<kPickThreads>(keys, L, tau, n_gt, n_eq, a.P, nullptr, scratch,
                                 [&](int t) { atomicAdd(&votes[t], 1); });
}

// Per-head picks for rows that fit in registers (L <= kPickRegThreads * KPL):
// CTA per (row, query head), thread t holds tokens t, t + NT, ...  The P-th
// largest key is found by a radix select that, before every 8-bit pass,
// recomputes the min and max of the keys still in play and starts the pass at
// their highest differing bit: bits all candidates share cost nothing, and a
// pass never piles equal digits of tied keys into one bin (scores on a coarse
// grid tie a lot).  Once the candidates are all equal the threshold is found.
// Keys above it vote; of the keys equal to it the lowest-index ones vote
// (ballots and per-warp counts, in token order).  Slots past the row's end
// hold key 0, the lowest key there is, and take part like real keys: the
// P-th largest is a real key (P < L), and where it is 0 the real zeros come
// first in token order, so a padding slot never votes.
template <int KPL>
__global__ void __launch_bounds__(kPickRegThreads) unified_pick_reg_kernel(const UnifiedArgs a) {
  constexpr int NT = kPickRegThreads, NW = NT / 32;
  __shared__ __align__(16) uint32_t hist[NW][256];
  __shared__ uint32_t spare[NT];  // the non-candidates' adds (never read)
  __shared__ uint32_t red[3][NW];
  __shared__ uint32_t xinfo[3];
  const int b = blockIdx.x / a.Hq, h = blockIdx.x % a.Hq;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  pdl_wait();
  pdl_launch_dependents();
  const int L = clamp_len(a.seq_lens[b], a.T, nullptr);
  if (L <= a.budget) return;
  if (a.P >= L) {  // the head picks every token
    const int W32 = (a.T + 31) / 32;
    uint32_t *bits = a.bits + (static_cast<size_t>(b) * a.Hq + h) * W32;
    for (int w = tid; w < (L + 31) / 32; w += NT)
      bits[w] = (w + 1) * 32 <= L ? 0xffffffffu : ((1u << (L - w * 32)) - 1u);
    return;
  }
  const uint32_t *gkeys = a.keys + (static_cast<size_t>(b) * a.Hq + h) * a.T;
  uint32_t key[KPL];
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    const int j = tid + NT * e;
    key[e] = j < L ? __ldcg(gkeys + j) : 0u;
  }
  uint32_t prefix = 0u, pmask = 0u;
  uint32_t remaining = static_cast<uint32_t>(a.P);  // still to take among the candidates
  uint32_t tau = 0u, n_eq = 0u;
  // min / max / count of the candidates, block-wide (every thread gets them)
  auto block_range = [&](uint32_t &kmin, uint32_t &kmax, uint32_t &cnt) {
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (lane == 0) {
      red[0][warp] = kmin;
      red[1][warp] = kmax;
      red[2][warp] = cnt;
    }
    __syncthreads();
    kmin = red[0][0];
    kmax = red[1][0];
    cnt = red[2][0];
#pragma unroll
    for (int w = 1; w < NW; ++w) {
      kmin = min(kmin, red[0][w]);
      kmax = max(kmax, red[1][w]);
      cnt += red[2][w];
    }
  };
  // the first pass's candidates are all the slots
  uint32_t kmin = 0xffffffffu, kmax = 0u, cnt = KPL;
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    kmin = min(kmin, key[e]);
    kmax = max(kmax, key[e]);
  }
  block_range(kmin, kmax, cnt);
  for (int pass = 0; pass < 5; ++pass) {  // at most 4 passes of 8 bits, then all equal
    if (kmin == kmax) {  // every candidate equal: the threshold
      tau = kmin;
      n_eq = cnt;
      break;
    }
    const int hb = 31 - __clz(kmin ^ kmax);  // candidates share every bit above hb
    const uint32_t above = hb == 31 ? 0u : ~((2u << hb) - 1u);
    prefix = kmin & above;
    pmask = above;
    const int sh = hb >= 7 ? hb - 7 : 0;
    for (int i = tid; i < NW * 256; i += NT) (&hist[0][0])[i] = 0u;
    __syncthreads();  // also: red was read by everyone
#pragma unroll
    for (int e = 0; e < KPL; ++e) {
      // every slot adds: non-candidates to a spare word of their own (a
      // conditional add here costs the compiler a register per key)
      const bool c = (key[e] & pmask) == prefix;
      atomicAdd(c ? &hist[warp][(key[e] >> sh) & 255u] : &spare[tid], 1u);
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
          xinfo[2] = c[jb];
        }
      }
    }
    __syncthreads();
    remaining -= xinfo[1];
    prefix = (prefix & ~(255u << sh)) | (xinfo[0] << sh);
    pmask |= 255u << sh;
    n_eq = xinfo[2];
    tau = prefix;
    __syncthreads();  // xinfo, hist and red are rewritten by the next pass
    if (sh == 0) break;  // every bit fixed
    // the next pass's candidates: keys matching the digits fixed so far
    kmin = 0xffffffffu;
    kmax = 0u;
    cnt = 0u;
#pragma unroll
    for (int e = 0; e < KPL; ++e) {
      if ((key[e] & pmask) == prefix) {
        kmin = min(kmin, key[e]);
        kmax = max(kmax, key[e]);
        ++cnt;
      }
    }
    block_range(kmin, kmax, cnt);
  }
  __syncthreads();  // red is read above before it is rewritten below
  const uint32_t take_eq = remaining;  // keys equal to tau to take, lowest token first
  const bool all_eq = take_eq == n_eq;  // block-uniform
  uint32_t *pre = &hist[0][0];          // [KPL][NW] exclusive counts of tied keys, token order
  if (!all_eq) {
#pragma unroll
    for (int e = 0; e < KPL; ++e) {
      const bool eq = key[e] == tau;
      const uint32_t eb = __ballot_sync(0xffffffffu, eq);
      if (lane == 0) pre[e * NW + warp] = __popc(eb);
    }
    __syncthreads();
    if (warp == 0) {  // exclusive scan of the KPL * NW counts, slot-major = token order
      constexpr int N = KPL * NW, PERL = (N + 31) / 32;
      uint32_t v[PERL];
      uint32_t s = 0u;
#pragma unroll
      for (int i = 0; i < PERL; ++i) {
        const int x = lane * PERL + i;
        v[i] = x < N ? pre[x] : 0u;
        s += v[i];
      }
      uint32_t incl = s;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      uint32_t run = incl - s;
#pragma unroll
      for (int i = 0; i < PERL; ++i) {
        const int x = lane * PERL + i;
        if (x < N) pre[x] = run;
        run += v[i];
      }
    }
    __syncthreads();
  }
  const int W32 = (a.T + 31) / 32;
  const int nwords = (L + 31) / 32;
  uint32_t *bits = a.bits + (static_cast<size_t>(b) * a.Hq + h) * W32;
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    const bool gt = key[e] > tau, eq = key[e] == tau;
    bool sel = gt || eq;
    if (!all_eq) {
      const uint32_t eb = __ballot_sync(0xffffffffu, eq);
      sel = gt || (eq && pre[e * NW + warp] + __popc(eb & lt) < take_eq);
    }
    const uint32_t sb = __ballot_sync(0xffffffffu, sel);
    const int word = NW * e + warp;  // tokens NT e + 32 warp + [0, 32)
    if (lane == 0 && word < nwords) bits[word] = sb;
  }
}

// Votes from the pick bit sets (rows whose picks were written as bits): one
// thread per token, votes[t] = number of heads whose bit t is set.  A warp's
// 32 tokens share one word per head, read once per warp.
__global__ void __launch_bounds__(256) unified_votes_kernel(const UnifiedArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const int W32 = (a.T + 31) / 32;
  const long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int b = static_cast<int>(e / (static_cast<long long>(W32) * 32));
  const int t = static_cast<int>(e - static_cast<long long>(b) * W32 * 32);
  if (b >= a.B) return;
  const int L = clamp_len(a.seq_lens[b], a.T, nullptr);
  if (L <= a.budget || t >= L) return;  // warp-uniform up to the row's last word
  const uint32_t *bits = a.bits + static_cast<size_t>(b) * a.Hq * W32 + (t >> 5);
  int v = 0;
#pragma unroll 16
  for (int h = 0; h < a.Hq; ++h) v += (__ldcg(bits + static_cast<size_t>(h) * W32) >> (t & 31)) & 1u;
  a.votes[static_cast<size_t>(b) * a.T + t] = v;
}

// Per-head token top-k lists: CTA per (row, query head), the k highest score
// keys (ties to the lower token) listed ascending with -1 padding; rows with
// L <= k keep every token.  Keys staged in shared memory when they fit.
__global__ void __launch_bounds__(kPickThreads) unified_topk_list_kernel(const UnifiedArgs a,
                                                                          int stage_in_smem) {
  extern __shared__ uint32_t skeys[];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t info[4];
  __shared__ uint32_t scratch[33];
  const int b = blockIdx.x / a.Hq, h = blockIdx.x % a.Hq;
  pdl_wait();
  pdl_launch_dependents();
  const int L = clamp_len(a.seq_lens[b], a.T, (h == 0 && threadIdx.x == 0) ? a.status : nullptr);
  const int k = a.P;
  int32_t *out = a.token_idx + (static_cast<size_t>(b) * a.Hq + h) * k;
  if (L <= k) {
    for (int i = threadIdx.x; i < k; i += kPickThreads) out[i] = i < L ? i : -1;
    if (threadIdx.x == 0) a.num_sel[static_cast<size_t>(b) * a.Hq + h] = L;
    return;
  }
  const uint32_t *gkeys = a.keys + (static_cast<size_t>(b) * a.Hq + h) * a.T;
  const uint32_t *keys = gkeys;
  if (stage_in_smem) {
    for (int t = threadIdx.x; t < L; t += kPickThreads) skeys[t] = gkeys[t];
    __syncthreads();
    keys = skeys;
  }
  uint32_t tau, n_gt, n_eq;
  radix_select_desc<kPickThreads>(keys, L, k, 32, hist, info, tau, n_gt, n_eq);
  select_ascending<kPickThreads>(keys, L, tau, n_gt, n_eq, k, out, scratch, [](int) {});
  if (threadIdx.x == 0) a.num_sel[static_cast<size_t>(b) * a.Hq + h] = k;
}

// Exclusive prefix sum of v over the block (thread order) and the total.
// `scan` holds NT / 32 + 1 words of shared memory.  All threads must call.
template <int NT>
__device__ __forceinline__ uint32_t block_exclusive_sum(uint32_t v, uint32_t *scan,
                                                        uint32_t &total) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) scan[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = lane < NW ? scan[lane] : 0u;
    uint32_t wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += y;
    }
    if (lane < NW) scan[lane] = wi - w;
    if (lane == 31) scan[NW] = wi;
  }
  __syncthreads();
  const uint32_t r = scan[warp] + incl - v;
  total = scan[NW];
  __syncthreads();  // scan is reused by the next call
  return r;
}

// Full adder on 32 bit lanes at once: a + b + c = 2 hi + lo in every lane.
__device__ __forceinline__ void csa(uint32_t &hi, uint32_t &lo, uint32_t a, uint32_t b,
                                    uint32_t c) {
  const uint32_t u = a ^ b;
  hi = (a & b) | (u & c);
  lo = u ^ c;
}

// Shared set straight from the per-head pick bit sets (the register-pick path,
// fewer than 64 heads): CTA per row, thread t owns the 32 candidates of bit
// word t.  It adds the row's Hq words into six bit planes (a counter per token
// lane, so plane i holds bit i of every token's vote count: carry-save adders
// take sixteen heads at a time, ripple-carry adds the rest),
// counts the tokens of each vote value from the planes, finds the threshold
// vote from the top value down, then -- with masks of the tokens above it and
// equal to it, again from the planes -- one block scan gives each thread its
// share of the tied tokens (lowest first) and its output position, and it
// writes its picks in token order.  The same set as the votes kernel followed
// by unified_set_kernel, in one launch.
__global__ void __launch_bounds__(kSetThreads, 1) unified_set_bits_kernel(const UnifiedArgs a) {
  constexpr int NT = kSetThreads, NW = NT / 32;
  __shared__ uint32_t hist[NW][64];
  __shared__ uint32_t scan[NW + 1];
  __shared__ uint32_t info[2];
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();
  pdl_launch_dependents();
  const int L = clamp_len(a.seq_lens[b], a.T, nullptr);
  int32_t *out = a.token_idx + static_cast<size_t>(b) * a.budget;
  if (L <= a.budget) {
    for (int i = tid; i < a.budget; i += NT) out[i] = i < L ? i : -1;
    if (tid == 0) a.num_sel[b] = L;
    return;
  }
  const int n = L - a.R;  // candidates [0, L - R)
  const int k = a.budget - a.R;
  if (k > 0) {
    // this thread's candidates: tokens 32 tid + j, j set in vm
    const int base = tid * 32;
    const uint32_t vm = base + 32 <= n ? 0xffffffffu : (base < n ? (1u << (n - base)) - 1u : 0u);
    uint32_t c[6] = {0u, 0u, 0u, 0u, 0u, 0u};  // bit planes of the vote counts
    if (vm != 0u) {  // (words past the candidates are not read: they may be stale)
      const int W32 = (a.T + 31) / 32;
      const uint32_t *bits = a.bits + static_cast<size_t>(b) * a.Hq * W32 + tid;
      int h = 0;
      // sixteen heads at a time through a tree of carry-save adders: c[0..3]
      // take the weights 1..8 and the tree's weight-16 output adds into c[4],
      // c[5] (a count stays below 64, so nothing carries past c[5])
      for (; h + 16 <= a.Hq; h += 16) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i] = __ldcg(bits + static_cast<size_t>(h + i) * W32);
        uint32_t t2a, t2b, f4a, f4b, e8a, e8b, s16;
        csa(t2a, c[0], c[0], w[0], w[1]);
        csa(t2b, c[0], c[0], w[2], w[3]);
        csa(f4a, c[1], c[1], t2a, t2b);
        csa(t2a, c[0], c[0], w[4], w[5]);
        csa(t2b, c[0], c[0], w[6], w[7]);
        csa(f4b, c[1], c[1], t2a, t2b);
        csa(e8a, c[2], c[2], f4a, f4b);
        csa(t2a, c[0], c[0], w[8], w[9]);
        csa(t2b, c[0], c[0], w[10], w[11]);
        csa(f4a, c[1], c[1], t2a, t2b);
        csa(t2a, c[0], c[0], w[12], w[13]);
        csa(t2b, c[0], c[0], w[14], w[15]);
        csa(f4b, c[1], c[1], t2a, t2b);
        csa(e8b, c[2], c[2], f4a, f4b);
        csa(s16, c[3], c[3], e8a, e8b);
        const uint32_t t = c[4] & s16;
        c[4] ^= s16;
        c[5] ^= t;
      }
      for (; h < a.Hq; ++h) {  // the rest one at a time: a ripple-carry add
        uint32_t carry = __ldcg(bits + static_cast<size_t>(h) * W32);
#pragma unroll
        for (int i = 0; i < 6; ++i) {
          const uint32_t t = c[i] & carry;
          c[i] ^= carry;
          carry = t;
        }
      }
    }
    // tokens of each vote value, per warp (warps past the candidates count none)
    if (__any_sync(0xffffffffu, vm != 0u)) {
      for (int v = 0; v <= a.Hq; ++v) {
        uint32_t m = vm;
#pragma unroll
        for (int i = 0; i < 6; ++i) m &= ((v >> i) & 1) ? c[i] : ~c[i];
        const uint32_t cnt = __reduce_add_sync(0xffffffffu, static_cast<uint32_t>(__popc(m)));
        if (lane == 0) hist[warp][v] = cnt;
      }
    } else {
      for (int v = lane; v <= a.Hq; v += 32) hist[warp][v] = 0u;
    }
    __syncthreads();
    if (tid < 64) {
      uint32_t t = 0u;
      for (int w = 0; w < NW; ++w) t += tid <= a.Hq ? hist[w][tid] : 0u;
      hist[0][tid] = t;
    }
    __syncthreads();
    if (warp == 0) {  // lane l owns values 2l, 2l + 1; counts from the top value down
      const uint32_t c1 = hist[0][2 * lane + 1], c0 = hist[0][2 * lane];
      const uint32_t tot = c0 + c1;
      uint32_t incl = tot;  // over lanes >= this one
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, incl, off);
        if (lane + off < 32) incl += y;
      }
      const uint32_t above = incl - tot;
      const uint32_t kk = static_cast<uint32_t>(k);
      if (above < kk && above + c1 >= kk) {
        info[0] = 2u * lane + 1u;
        info[1] = above;
      } else if (above + c1 < kk && above + tot >= kk) {
        info[0] = 2u * lane;
        info[1] = above + c1;
      }
    }
    __syncthreads();
    const uint32_t tau = info[0];
    const uint32_t take_eq = static_cast<uint32_t>(k) - info[1];  // tied picks, lowest first
    // masks of this thread's tokens with votes above tau and equal to it
    uint32_t gt = 0u, eq = 0xffffffffu;
#pragma unroll
    for (int i = 5; i >= 0; --i) {
      if ((tau >> i) & 1u) {
        eq &= c[i];
      } else {
        gt |= eq & c[i];
        eq &= ~c[i];
      }
    }
    gt &= vm;
    eq &= vm;
    // one scan of the packed counts (each total is at most 32 NT < 2^16): the tied
    // tokens before this thread, and those above tau; the kept tied tokens before it
    // are the first take_eq of the row's, so its first output slot follows from both
    uint32_t tot;
    const uint32_t my_eq = static_cast<uint32_t>(__popc(eq));
    const uint32_t before = block_exclusive_sum<NT>(
        (static_cast<uint32_t>(__popc(gt)) << 16) | my_eq, scan, tot);
    const uint32_t eq_before = before & 0xffffu, gt_before = before >> 16;
    const uint32_t eq_take = eq_before >= take_eq ? 0u : min(my_eq, take_eq - eq_before);
    uint32_t keep = 0u, rest = eq;  // the lowest eq_take tied tokens
    for (uint32_t q = 0u; q < eq_take; ++q) {
      const uint32_t low = rest & (~rest + 1u);
      keep |= low;
      rest ^= low;
    }
    uint32_t sel = gt | keep;
    uint32_t pos = gt_before + min(eq_before, take_eq);
    while (sel != 0u) {
      out[pos++] = base + __ffs(sel) - 1;
      sel &= sel - 1u;
    }
  }
  for (int i = tid; i < a.R; i += NT) out[k + i] = n + i;
  if (tid == 0) a.num_sel[b] = a.budget;
}

// Shared set: CTA per row.
__global__ void __launch_bounds__(kSetThreads) unified_set_kernel(const UnifiedArgs a) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t info[4];
  __shared__ uint32_t scratch[33];
  const int b = blockIdx.x;
  pdl_wait();
  pdl_launch_dependents();
  const int L = clamp_len(a.seq_lens[b], a.T, nullptr);
  int32_t *out = a.token_idx + static_cast<size_t>(b) * a.budget;
  if (L <= a.budget) {
    for (int i = threadIdx.x; i < a.budget; i += kSetThreads) out[i] = i < L ? i : -1;
    if (threadIdx.x == 0) a.num_sel[b] = L;
    return;
  }
  const int n = L - a.R;       // candidates [0, L - R)
  const int k = a.budget - a.R;
  if (k > 0) {
    const uint32_t *keys = reinterpret_cast<const uint32_t *>(a.votes + static_cast<size_t>(b) * a.T);
    const int nbits = a.Hq < 256 ? 8 : 16;
    uint32_t tau, n_gt, n_eq;
    radix_select_desc<kSetThreads>(keys, n, k, nbits, hist, info, tau, n_gt, n_eq);
    select_ascending<kSetThreads>(keys, n, tau, n_gt, n_eq, k, out, scratch, [](int) {});
  }
  for (int i = threadIdx.x; i < a.R; i += kSetThreads) out[k + i] = n + i;
  if (threadIdx.x == 0) a.num_sel[b] = a.budget;
}

template <int D>
cudaError_t launch_scores(const UnifiedArgs &a, cudaStream_t stream) {
  CUtensorMap km;
  memset(&km, 0, sizeof km);
  if (!encode_kv_tensor_map(&km, a.K, static_cast<uint64_t>(a.B) * a.Hkv * a.T, D, kTok))
    return cudaErrorInvalidValue;
  const int n_chunks = (a.T + kChunk - 1) / kChunk;
  const size_t smem = SCfg<D>::kSmemBytes;
  int occ = 0;  // (the memo raises the kernel's shared-memory limit once per device)
  const cudaError_t err = kernel_occupancy(reinterpret_cast<const void *>(unified_scores_kernel<D>),
                                           kScoreThreads, smem, &occ);
  if (err != cudaSuccess) return err;
  const unsigned grid = static_cast<unsigned>(a.B) * a.Hkv * n_chunks;
  return launch_pdl(unified_scores_kernel<D>, dim3(grid), dim3(kScoreThreads), smem, stream, km,
                    a, n_chunks);
}

// Random-head aggregation's last step: row b's set is query head head[b]'s
// list and count.  One thread per list entry (and per count).
__global__ void __launch_bounds__(256) gather_head_lists_kernel(const int32_t *lists,
                                                                const int32_t *counts,
                                                                const int32_t *head, int B,
                                                                int Hq, int k, int32_t *token_idx,
                                                                int32_t *num_sel) {
  pdl_wait();
  pdl_launch_dependents();
  const long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long n = static_cast<long long>(B) * k;
  if (e < n) {
    const int b = static_cast<int>(e / k), i = static_cast<int>(e - static_cast<long long>(b) * k);
    const size_t src = static_cast<size_t>(b) * Hq + head[b];
    token_idx[e] = lists[src * k + i];
  } else if (e < n + B) {
    const int b = static_cast<int>(e - n);
    num_sel[b] = counts[static_cast<size_t>(b) * Hq + head[b]];
  }
}

}  // namespace

size_t unified_workspace_bytes(int B, int Hq, int T) {
  const size_t keys = (static_cast<size_t>(B) * Hq * T * sizeof(uint32_t) + 255) & ~static_cast<size_t>(255);
  const size_t votes = (static_cast<size_t>(B) * T * sizeof(int32_t) + 255) & ~static_cast<size_t>(255);
  const size_t bits =
      (static_cast<size_t>(B) * Hq * ((T + 31) / 32) * sizeof(uint32_t) + 255) & ~static_cast<size_t>(255);
  return keys + votes + bits;
}

cudaError_t launch_gather_head_lists(const int32_t *lists, const int32_t *counts,
                                     const int32_t *head, int B, int Hq, int k,
                                     int32_t *token_idx, int32_t *num_sel, cudaStream_t stream) {
  const long long n = static_cast<long long>(B) * k + B;
  return launch_pdl(gather_head_lists_kernel, dim3(static_cast<unsigned>((n + 255) / 256)),
                    dim3(256), 0, stream, lists, counts, head, B, Hq, k, token_idx, num_sel);
}

cudaError_t launch_tokens_per_head(const UnifiedArgs &a, cudaStream_t stream) {
  // the scoring launch skips rows with L <= budget: here the budget is k
  cudaError_t err = a.D == 128 ? launch_scores<128>(a, stream) : launch_scores<64>(a, stream);
  if (err != cudaSuccess) return err;
  const int in_smem = a.T <= kSmemKeys ? 1 : 0;
  const size_t smem = in_smem ? static_cast<size_t>(a.T) * sizeof(uint32_t) : 0;
  int occ = 0;
  err = kernel_occupancy(reinterpret_cast<const void *>(unified_topk_list_kernel), kPickThreads,
                         smem, &occ);
  if (err != cudaSuccess) return err;
  return launch_pdl(unified_topk_list_kernel, dim3(static_cast<unsigned>(a.B) * a.Hq),
                    dim3(kPickThreads), smem, stream, a, in_smem);
}

cudaError_t launch_unified_select(const UnifiedArgs &a, int num_sms, cudaStream_t stream) {
  (void)num_sms;
  cudaError_t err = a.D == 128 ? launch_scores<128>(a, stream) : launch_scores<64>(a, stream);
  if (err != cudaSuccess) return err;
  const dim3 pgrid(static_cast<unsigned>(a.B) * a.Hq);
  const int per = (a.T + kPickRegThreads - 1) / kPickRegThreads;  // keys per thread
  if (per <= kPickRegMaxKeys) {
    const dim3 pblock(kPickRegThreads);
    if (per <= 16) err = launch_pdl(unified_pick_reg_kernel<16>, pgrid, pblock, 0, stream, a);
    else if (per <= 32) err = launch_pdl(unified_pick_reg_kernel<32>, pgrid, pblock, 0, stream, a);
    else if (per <= 48) err = launch_pdl(unified_pick_reg_kernel<48>, pgrid, pblock, 0, stream, a);
    else if (per <= 64) err = launch_pdl(unified_pick_reg_kernel<64>, pgrid, pblock, 0, stream, a);
    else if (per <= 80) err = launch_pdl(unified_pick_reg_kernel<80>, pgrid, pblock, 0, stream, a);
    else err = launch_pdl(unified_pick_reg_kernel<96>, pgrid, pblock, 0, stream, a);
    if (err != cudaSuccess) return err;
    if (a.Hq < 64 && (a.T + 31) / 32 <= kSetThreads)  // the set straight from the bit sets
      return launch_pdl(unified_set_bits_kernel, dim3(static_cast<unsigned>(a.B)),
                        dim3(kSetThreads), 0, stream, a);
    const long long nt = static_cast<long long>(a.B) * ((a.T + 31) / 32) * 32;
    err = launch_pdl(unified_votes_kernel, dim3(static_cast<unsigned>((nt + 255) / 256)),
                     dim3(256), 0, stream, a);
  } else {  // longer rows: keys staged in shared memory (or read from L2)
    const int in_smem = a.T <= kSmemKeys ? 1 : 0;
    const size_t pick_smem = in_smem ? static_cast<size_t>(a.T) * sizeof(uint32_t) : 0;
    int occ = 0;
    err = kernel_occupancy(reinterpret_cast<const void *>(unified_pick_kernel), kPickThreads,
                           pick_smem, &occ);
    if (err != cudaSuccess) return err;
    err = launch_pdl(unified_pick_kernel, pgrid, dim3(kPickThreads), pick_smem, stream, a,
                     in_smem);
  }
  if (err != cudaSuccess) return err;
  return launch_pdl(unified_set_kernel, dim3(static_cast<unsigned>(a.B)), dim3(kSetThreads), 0,
                    stream, a);
}

}  // namespace ksa
