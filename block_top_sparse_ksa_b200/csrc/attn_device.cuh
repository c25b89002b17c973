// attn_device.cuh -- device pieces of the gathered split-KV flash-decode (the
// attention kernel's body and its helpers) and the host-side preparation of an
// attention launch.  The design is described at the top of decode_attn.cu.
#pragma once

#include "ksa_device.cuh"
#include "ksa_internal.h"

namespace ksa {
namespace att {

constexpr int kStageTok = 16;  // tokens per pipeline stage (16 or 32: one or two mma tiles)
constexpr int kTiles = kStageTok / 16;
constexpr uint32_t kFullMask = kStageTok >= 32 ? 0xffffffffu : ((1u << kStageTok) - 1u);
constexpr int kConsumers = 4;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kMergeParts = 4;  // split-row partials combined per round of loads

enum { kModeDense = 0, kModeTma = 1, kModeCp = 2 };

// Token lists take two producer warps (stages alternate between them): their
// 16-byte copies are issued by the warps themselves, and one warp per CTA set
// the pace.
template <int MODE>
__host__ __device__ constexpr int attn_producers() {
  return MODE == kModeCp ? 2 : 1;
}
template <int MODE>
__host__ __device__ constexpr int attn_threads() {
  return (kConsumers + attn_producers<MODE>()) * 32;
}

template <int D, bool DEEP = false>
struct Cfg {
  static constexpr int kHalves = D / 64;              // 64-column (128-byte) halves of a row
  static constexpr int kHalfBytes = kStageTok * 128;  // one 64-column half of a stage tile
  static constexpr int kTileBytes = kHalves * kHalfBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;  // K tile + V tile
  // A multiple of the consumer-warp count: stage i lives in buffer i % kStages
  // and is consumed by warp i % kConsumers, so every buffer always belongs to
  // the same warp and that warp awaits the buffer's phases strictly in order.
  // (With buffers shared between warps a fast warp could wait on a phase two
  // ahead of the barrier, which a parity wait cannot tell from a finished one.)
  // Two buffers per warp: a warp computes on one while its next stage lands;
  // three in the deep form (two CTAs per SM, one per row: more bytes in flight
  // per CTA).
  static constexpr int kStages = (kStageTok == 16 ? (DEEP ? 12 : 8) : 4) * (D == 128 ? 1 : 2);
  static_assert(kStages % kConsumers == 0, "stage buffers must map to one consumer warp each");
  static constexpr int kKT = D / 16;
  // stage buffers, 2 mbarriers + 1 mask per stage, flags; plus 1 KB alignment slack
  static constexpr size_t kBarrierOffset = static_cast<size_t>(kStages) * kStageBytes;
  static constexpr size_t kMergeOffset = kBarrierOffset + 2 * 8 * kStages + 4 * kStages + 64;
  static constexpr size_t kFixedSmem = 1024 + kMergeOffset;
};

struct AttnDev {
  AttnArgs a;
  int rpb;        // rows per batch row: Hkv, or Hq with per-query-head lists
  int gw;         // query heads per row: G, or 1 with per-query-head lists
  int V;          // stages each row is padded to
  long long W;    // rows * V
  int N;          // CTAs in the grid
  int slot;       // floats of one partial: m[G], l[G], o[G][D]
  float *part;    // workspace partials [N][2][slot]
  int32_t *sem;   // workspace semaphores [rows], zero between calls
  float scale_log2;
};

static __device__ __forceinline__ long long cta_start(long long c, long long W, int N) {
  return c * W / N;
}
// The CTA whose slice holds virtual stage v: the largest c with cta_start(c) <= v.
static __device__ __forceinline__ int cta_of(long long v, long long W, int N) {
  return static_cast<int>(((v + 1) * N + W - 1) / W - 1);
}

static __device__ __forceinline__ void consumer_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumers * 32) : "memory");
}

// Row r of the work: batch row b, kv-head g, and its query heads qh0 .. qh0 + gw - 1
// (the G heads of kv-head g, or with per-query-head lists the one head h).
struct RowGeom {
  int b, g, qh0;
};
static __device__ __forceinline__ RowGeom row_geom(const AttnDev &p, int r) {
  RowGeom x;
  x.b = r / p.rpb;
  const int i = r - x.b * p.rpb;
  if (p.gw == 1 && p.rpb == p.a.Hq) {  // per-query-head rows
    x.g = i / (p.a.Hq / p.a.Hkv);
    x.qh0 = i;
  } else {
    x.g = i;
    x.qh0 = i * p.gw;
  }
  return x;
}

struct RowInfo {
  int L;
  const int32_t *list;
  int n_idx;
  int n_st;  // real stages of the row
};

template <int MODE>
__device__ __forceinline__ RowInfo row_info(const AttnArgs &a, int r, int b, uint32_t *flag_sink) {
  RowInfo ri;
  ri.L = clamp_len(a.seq_lens[b], a.T, flag_sink);
  ri.list = nullptr;
  ri.n_idx = 0;
  if (MODE == kModeDense) {
    ri.n_st = (ri.L + kStageTok - 1) / kStageTok;
    return ri;
  }
  ri.list = a.shared == 1 ? a.idx + static_cast<size_t>(b) * a.cap
                          : a.idx + static_cast<size_t>(r) * a.cap;
  int n = a.shared == 1 ? a.num_idx[b] : a.num_idx[r];  // 0: per kv-head, 2: per query head rows
  if (n < 0 || n > a.cap) {
    flag_status(flag_sink, KSA_FLAG_INDEX_SKIPPED);
    n = n < 0 ? 0 : a.cap;
  }
  ri.n_idx = n;
  if (a.tpi >= kStageTok)
    ri.n_st = n * (a.tpi / kStageTok);
  else
    ri.n_st = static_cast<int>((static_cast<long long>(n) * a.tpi + kStageTok - 1) / kStageTok);
  return ri;
}

static __device__ __forceinline__ void store_out(const AttnArgs &a, size_t oi, float v) {
  if (a.out_f32 != nullptr)
    a.out_f32[oi] = v;
  else
    a.out_bf16[oi] = f32_to_bf16_bits(v);
}

// Merges the partials (m, l, o per head) that the CTAs sharing row r left in
// the workspace and writes the row's output and lse.  The 128 consumer
// threads take two output elements each per round and issue every load for
// them (up to kMergeParts partials) before combining, so a row split between a
// few CTAs costs one round trip to L2.
template <int D>
__device__ __forceinline__ void merge_partials(const AttnDev &p, int r, int tid) {
  const AttnArgs &a = p.a;
  const int G = p.gw;  // query heads of the row
  const int SL = p.slot;
  const RowGeom rg = row_geom(p, r);
  const long long rv0 = static_cast<long long>(r) * p.V;
  const int c_first = cta_of(rv0, p.W, p.N);
  const int c_last = cta_of(rv0 + p.V - 1, p.W, p.N);
  const size_t obase = static_cast<size_t>(rg.b) * a.Hq + rg.qh0;
  constexpr int NT = kConsumers * 32;
  for (int e0 = tid; e0 < G * D; e0 += 2 * NT) {
    float M[2] = {-INFINITY, -INFINITY}, o[2] = {0.f, 0.f}, l[2] = {0.f, 0.f};
    for (int cq0 = c_first; cq0 <= c_last; cq0 += kMergeParts) {
      float mv[2][kMergeParts], lv[2][kMergeParts], ov[2][kMergeParts];
#pragma unroll
      for (int i = 0; i < kMergeParts; ++i) {
        const int cq = cq0 + i;
        const float *sl = nullptr;
        if (cq <= c_last) {
          const int wq = (r == static_cast<int>(cta_start(cq, p.W, p.N) / p.V)) ? 0 : 1;
          sl = p.part + (static_cast<size_t>(cq) * 2 + wq) * SL;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int e = e0 + h * NT;
          const bool ok = sl != nullptr && e < G * D;
          const int hh = e / D, d = e % D;
          mv[h][i] = ok ? __ldcg(sl + hh) : -INFINITY;
          lv[h][i] = ok ? __ldcg(sl + G + hh) : 0.f;
          ov[h][i] = ok ? __ldcg(sl + 2 * G + hh * D + d) : 0.f;
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float Mn = M[h];
#pragma unroll
        for (int i = 0; i < kMergeParts; ++i) Mn = fmaxf(Mn, mv[h][i]);
        const float base = (Mn == -INFINITY) ? 0.f : Mn;
        const float sc = fast_exp2(M[h] - base);  // rescale what was summed so far
        o[h] *= sc;
        l[h] *= sc;
#pragma unroll
        for (int i = 0; i < kMergeParts; ++i) {
          const float f = fast_exp2(mv[h][i] - base);
          o[h] += f * ov[h][i];
          l[h] += f * lv[h][i];
        }
        M[h] = Mn;
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int e = e0 + h * NT;
      if (e < G * D) {
        const int hh = e / D, d = e % D;
        store_out(a, (obase + hh) * D + d, l[h] > 0.f ? o[h] / l[h] : 0.f);
        if (d == 0 && a.lse != nullptr)
          a.lse[obase + hh] = l[h] > 0.f ? (M[h] + log2f(l[h])) * kLn2 : -INFINITY;
      }
    }
  }
}

// One CTA's share of the attention (the body of the attention kernel).
template <int D, int MODE, bool DEEP = false>
__device__ __forceinline__ void attn_cta(const CUtensorMap &kmap, const CUtensorMap &vmap,
                                         const AttnDev &p, uint8_t *smem_raw) {
  using C = Cfg<D, DEEP>;
  constexpr int NS = C::kStages;
  constexpr int KT = C::kKT;
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *stages = smem;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarrierOffset);
  uint64_t *empty = full + NS;
  uint32_t *stage_mask = reinterpret_cast<uint32_t *>(empty + NS);
  volatile uint32_t *abort_flag = stage_mask + NS;
  volatile int32_t *last_flag = reinterpret_cast<volatile int32_t *>(stage_mask + NS + 1);
  float *merge = reinterpret_cast<float *>(smem + C::kMergeOffset);  // [4][2G + G*D]

  const AttnArgs &a = p.a;
  const int G = p.gw;  // query heads per row
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = blockIdx.x;
  const long long s0 = cta_start(c, p.W, p.N), s1 = cta_start(c + 1, p.W, p.N);
  if (s0 >= s1) return;
  const int r_first = static_cast<int>(s0 / p.V), r_last = static_cast<int>((s1 - 1) / p.V);
  const int tpi = a.tpi;

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], MODE == kModeCp ? 33u : 1u);
      mbar_init(&empty[s], 1u);
    }
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (MODE != kModeCp && tid == kConsumers * 32) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }
  pdl_wait();
  pdl_launch_dependents();
  __syncthreads();

  int issued = 0;  // stages the producer filled (TMA modes: uses of the lane's own buffer)

  if (warp >= kConsumers) {
    // ------------------------------------------------------------ producer
    uint32_t skipped = 0u;
    if (MODE != kModeCp) {
      // TMA modes, lane-parallel: lane l < NS owns stage buffer l and fills the
      // CTA's stages l, l + NS, l + 2 NS, ...  Each lane runs its own chain
      // (wait for the buffer, read the block index, arm the barrier, issue the
      // boxes), so up to NS such chains are in flight at once.
      if (lane < NS) {
        const int seg = (MODE == kModeDense || tpi >= kStageTok) ? kStageTok : tpi;
        const int nseg = kStageTok / seg;                        // 1 or 2 segments
        const int spe = tpi >= kStageTok ? tpi / kStageTok : 1;  // stages per entry
        int r = r_first;
        long long rv0 = static_cast<long long>(r) * p.V;
        RowGeom rg = row_geom(p, r);
        RowInfo ri = row_info<MODE>(a, r, rg.b, (lane == 0 && rv0 >= s0) ? a.status : nullptr);
        int ja = static_cast<int>((s0 > rv0 ? s0 : rv0) - rv0);
        int jb = min(static_cast<int>((s1 < rv0 + p.V ? s1 : rv0 + p.V) - rv0), ri.n_st);
        int cnt = jb > ja ? jb - ja : 0;
        int row_base = 0;  // CTA ordinal of the row's first stage
        for (int i = lane;; i += NS) {
          while (i >= row_base + cnt && r <= r_last) {
            row_base += cnt;
            if (++r > r_last) break;
            rv0 = static_cast<long long>(r) * p.V;
            rg = row_geom(p, r);
            ri = row_info<MODE>(a, r, rg.b, (lane == 0 && rv0 >= s0) ? a.status : nullptr);
            ja = static_cast<int>((s0 > rv0 ? s0 : rv0) - rv0);
            jb = min(static_cast<int>((s1 < rv0 + p.V ? s1 : rv0 + p.V) - rv0), ri.n_st);
            cnt = jb > ja ? jb - ja : 0;
          }
          if (r > r_last) break;
          const int j = ja + (i - row_base);
          long long t0[kTiles], yr[kTiles];
          int nv[kTiles];
          uint32_t mask = 0u, bytes = 0u;
#pragma unroll
          for (int u = 0; u < kTiles; ++u) {  // nseg <= kTiles segments
            nv[u] = 0;
            t0[u] = 0;
            yr[u] = 0;
            if (u >= nseg) continue;
            bool ok = true;
            if (MODE == kModeDense) {
              t0[u] = static_cast<long long>(j) * kStageTok;
            } else {
              const int e = (tpi >= kStageTok) ? j / spe : j * nseg + u;
              const int part = (tpi >= kStageTok) ? j % spe : 0;
              // read the entry without waiting for the count (any e < cap is in
              // bounds): one dependent round trip fewer per row
              const int id_any = e < a.cap ? __ldg(ri.list + e) : -1;
              const int id = e < ri.n_idx ? id_any : -1;
              ok = e < ri.n_idx && id >= 0;
              t0[u] = static_cast<long long>(id) * tpi + static_cast<long long>(part) * kStageTok;
              if (e < ri.n_idx && (id < 0 || (part == 0 && t0[u] >= ri.L)))
                skipped = KSA_FLAG_INDEX_SKIPPED;
            }
            const long long left = ri.L - t0[u];
            nv[u] = (!ok || left <= 0) ? 0 : (left < seg ? static_cast<int>(left) : seg);
            if (nv[u] > 0) {  // the segment's first K/V row (its page, when paged)
              yr[u] = kv_row(a.kv, rg.b, rg.g, a.Hkv, a.T, t0[u]);
              if (yr[u] < 0) {
                nv[u] = 0;
                skipped = KSA_FLAG_INDEX_SKIPPED;
              }
            }
            if (nv[u] > 0) {
              mask |= (nv[u] >= 32 ? 0xffffffffu : ((1u << nv[u]) - 1u)) << (u * seg);
              bytes += static_cast<uint32_t>(seg) * 128u * C::kHalves * 2u;
            }
          }
          if (issued > 0 &&
              !mbar_wait(&empty[lane], static_cast<uint32_t>(issued - 1) & 1u)) {
            *abort_flag = 1u;
            flag_status(a.status, KSA_FLAG_WAIT_TIMEOUT);
            break;
          }
          ++issued;  // uses of this lane's buffer
          uint8_t *sK = stages + static_cast<size_t>(lane) * C::kStageBytes;
          uint8_t *sV = sK + C::kTileBytes;
          stage_mask[lane] = mask;
          mbar_arrive_expect_tx(&full[lane], bytes);
#pragma unroll
          for (int u = 0; u < kTiles; ++u) {
            if (nv[u] <= 0) continue;
            const int yrow = static_cast<int>(yr[u]);
#pragma unroll
            for (int h = 0; h < C::kHalves; ++h) {
              tma_load_2d(sK + h * C::kHalfBytes + u * seg * 128, &kmap, h * 64, yrow, &full[lane]);
              tma_load_2d(sV + h * C::kHalfBytes + u * seg * 128, &vmap, h * 64, yrow, &full[lane]);
            }
          }
        }
      }
    } else {
      // token lists: each producer warp fills its stages one at a time with
      // 16-byte cp.async (row u of a stage <- list entry j*eps + u/tpi, token
      // offset u%tpi); producer pw takes the CTA's stages i = pw (mod 2), so it
      // only ever fills the buffers of that parity (kStages is even).  The list
      // is read 32 entries at a time, one per lane, the next 32 in flight.
      constexpr int NP = attn_producers<MODE>();
      static_assert(NS % NP == 0, "a buffer belongs to one producer");
      const int pw = warp - kConsumers;
      bool stop = false;
      int i = 0;
      for (int r = r_first; r <= r_last && !stop; ++r) {
        const long long rv0 = static_cast<long long>(r) * p.V;
        const bool reporter = lane == 0 && rv0 >= s0;
        const RowGeom rg = row_geom(p, r);
        const RowInfo ri = row_info<MODE>(a, r, rg.b, reporter ? a.status : nullptr);
        const int ja = static_cast<int>((s0 > rv0 ? s0 : rv0) - rv0);
        const int jb = min(static_cast<int>((s1 < rv0 + p.V ? s1 : rv0 + p.V) - rv0), ri.n_st);
        const int eps = kStageTok / tpi;  // entries per stage
        int wbase = 0, cur = -1, nxt = -1;
        if (ja < jb) {
          wbase = (ja * eps) & ~31;
          // entries are read before the count is known (any index < cap is in bounds)
          const int c0 = (wbase + lane < a.cap) ? ri.list[wbase + lane] : -1;
          const int c1 =
              (wbase + 32 + lane < a.cap) ? ri.list[wbase + 32 + lane] : -1;
          cur = (wbase + lane < ri.n_idx) ? c0 : -1;
          nxt = (wbase + 32 + lane < ri.n_idx) ? c1 : -1;
        }
        for (int j = ja; j < jb; ++j, ++i) {
          if (j * eps >= wbase + 32) {  // stages advance by at most one window
            wbase += 32;
            cur = nxt;
            nxt = (wbase + 32 + lane < ri.n_idx) ? ri.list[wbase + 32 + lane] : -1;
          }
          if (i % NP != pw) continue;  // the other producer's stage
          const int buf = i % NS;
          if (i >= NS &&
              !__all_sync(0xffffffffu,
                          mbar_wait(&empty[buf], static_cast<uint32_t>((i / NS) - 1) & 1u))) {
            if (lane == 0) {
              *abort_flag = 1u;
              flag_status(a.status, KSA_FLAG_WAIT_TIMEOUT);
            }
            stop = true;
            break;
          }
          issued = i + 1;
          uint8_t *sK = stages + static_cast<size_t>(buf) * C::kStageBytes;
          uint8_t *sV = sK + C::kTileBytes;
          const int e = j * eps + lane / tpi;
          const int id = __shfl_sync(0xffffffffu, cur, (e - wbase) & 31);
          bool valid = false;
          long long trow = 0;  // the token's K/V row
          if (lane < kStageTok && e < ri.n_idx) {
            const long long t = static_cast<long long>(id) * tpi + (lane % tpi);
            valid = id >= 0 && t < ri.L;
            if (!valid && (lane % tpi) == 0 &&
                (id < 0 || static_cast<long long>(id) * tpi >= ri.L))
              skipped = KSA_FLAG_INDEX_SKIPPED;
            if (valid) {
              trow = kv_row(a.kv, rg.b, rg.g, a.Hkv, a.T, t);
              if (trow < 0) {  // its page id names no page
                valid = false;
                skipped = KSA_FLAG_INDEX_SKIPPED;
              }
            }
          }
          const uint32_t mask = __ballot_sync(0xffffffffu, valid);
          constexpr int CH = D / 8;     // 16-byte chunks per row
          constexpr int RPW = 32 / CH;  // rows per warp instruction
          const int my_c = lane % CH;
          for (int q0 = 0; q0 < kStageTok; q0 += RPW) {
            const int u = q0 + lane / CH;
            const int uv = __shfl_sync(0xffffffffu, static_cast<int>(valid), u);
            const long long ur = __shfl_sync(0xffffffffu, trow, u);
            if (uv) {
              const size_t src = static_cast<size_t>(ur) * D + my_c * 8;
              const uint32_t off = (my_c >> 3) * C::kHalfBytes + swz128(u, my_c & 7);
              cp_async_16(sK + off, a.K + src);
              cp_async_16(sV + off, a.V + src);
            }
          }
          if (lane == 0) {
            stage_mask[buf] = mask;
            mbar_arrive(&full[buf]);
          }
          cp_async_arrive_noinc(&full[buf]);
        }
      }
    }
    __syncwarp();
    skipped = __reduce_or_sync(0xffffffffu, skipped);
    if (skipped && lane == 0) flag_status(a.status, skipped);
  } else {
    // ------------------------------------------------------------ consumers
    const int gid = lane >> 2, tig = lane & 3;
    const int mi = lane >> 3, lr = lane & 7;
    const float sl2 = p.scale_log2;
    const int SL = p.slot;
    float *wm = merge;          // [4][G]
    float *wl = merge + 4 * G;  // [4][G]
    float *wo = merge + 8 * G;  // [4][G][D]
    int i = 0;                  // ordinal of the next stage of this CTA
    for (int r = r_first; r <= r_last; ++r) {
      const RowGeom rg = row_geom(p, r);
      const long long rv0 = static_cast<long long>(r) * p.V;
      const RowInfo ri = row_info<MODE>(a, r, rg.b, nullptr);
      const int ja = static_cast<int>((s0 > rv0 ? s0 : rv0) - rv0);
      const int jb = min(static_cast<int>((s1 < rv0 + p.V ? s1 : rv0 + p.V) - rv0), ri.n_st);
      const int cnt = jb > ja ? jb - ja : 0;

      uint32_t qb[KT][2];
      {
        const uint16_t *qrow =
            a.q + (static_cast<size_t>(rg.b) * a.Hq + rg.qh0 + gid) * D;
#pragma unroll
        for (int ks = 0; ks < KT; ++ks) {
          qb[ks][0] =
              gid < G ? *reinterpret_cast<const uint32_t *>(qrow + ks * 16 + tig * 2) : 0u;
          qb[ks][1] =
              gid < G ? *reinterpret_cast<const uint32_t *>(qrow + ks * 16 + 8 + tig * 2) : 0u;
        }
      }
      // online-softmax state for the lane's two heads 2*(lane%4), 2*(lane%4)+1
      float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
      float acc[KT][4];
#pragma unroll
      for (int mt = 0; mt < KT; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;

      // this warp takes the row's stages whose CTA ordinal is = warp (mod 4)
      for (int k = ((warp - i) % kConsumers + kConsumers) % kConsumers; k < cnt;
           k += kConsumers) {
        const int ii = i + k;
        const int buf = ii % NS;
        if (__any_sync(0xffffffffu, *abort_flag != 0u)) break;
        if (!__all_sync(0xffffffffu,
                        mbar_wait(&full[buf], static_cast<uint32_t>(ii / NS) & 1u))) {
          if (lane == 0) {
            *abort_flag = 1u;
            flag_status(a.status, KSA_FLAG_WAIT_TIMEOUT);
          }
          break;
        }
        const uint32_t mask = stage_mask[buf];
        uint8_t *sK = stages + static_cast<size_t>(buf) * C::kStageBytes;
        uint8_t *sV = sK + C::kTileBytes;
        if (mask != kFullMask) {
          // rows past L / skipped entries: zero V so that p = 0 meets finite values
          for (int u = 0; u < kStageTok; ++u) {
            if (!((mask >> u) & 1u) && lane < C::kHalves * 8) {
              *reinterpret_cast<uint4 *>(sV + (lane >> 3) * C::kHalfBytes + u * 128 +
                                         (lane & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
            }
          }
          if (MODE != kModeCp) fence_proxy_async_smem();
          __syncwarp();
        }
        const uint32_t kbase = smem_addr(sK), vbase = smem_addr(sV);
#pragma unroll
        for (int tile = 0; tile < kTiles; ++tile) {
          float s[4] = {0.f, 0.f, 0.f, 0.f};
          {
            const int rr = tile * 16 + lr + ((mi & 1) << 3);
#pragma unroll
            for (int ks = 0; ks < KT; ++ks) {
              const int d = ks * 16 + ((mi >> 1) << 3);
              uint32_t af[4];
              ldsm_x4(af, kbase + (d >> 6) * C::kHalfBytes + swz128(rr, (d & 63) >> 3));
              mma_16816(s, af, qb[ks][0], qb[ks][1]);
            }
          }
          const int r0 = tile * 16 + gid;
          const bool v0 = (mask >> r0) & 1u, v1 = (mask >> (r0 + 8)) & 1u;
          const float z0 = v0 ? s[0] * sl2 : -INFINITY;
          const float z1 = v0 ? s[1] * sl2 : -INFINITY;
          const float z2 = v1 ? s[2] * sl2 : -INFINITY;
          const float z3 = v1 ? s[3] * sl2 : -INFINITY;
          float mx0 = fmaxf(z0, z2), mx1 = fmaxf(z1, z3);
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
          }
          const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
          const float base0 = (mn0 == -INFINITY) ? 0.f : mn0;
          const float base1 = (mn1 == -INFINITY) ? 0.f : mn1;
          const float al0 = fast_exp2(m0 - base0), al1 = fast_exp2(m1 - base1);
          const float p0 = fast_exp2(z0 - base0), p1 = fast_exp2(z1 - base1);
          const float p2 = fast_exp2(z2 - base0), p3 = fast_exp2(z3 - base1);
          l0 = l0 * al0 + (p0 + p2);
          l1 = l1 * al1 + (p1 + p3);
          m0 = mn0;
          m1 = mn1;
          if (!__all_sync(0xffffffffu, al0 == 1.f && al1 == 1.f)) {
#pragma unroll
            for (int mt = 0; mt < KT; ++mt) {
              acc[mt][0] *= al0;
              acc[mt][1] *= al1;
              acc[mt][2] *= al0;
              acc[mt][3] *= al1;
            }
          }
          // P^T fragments (tokens x heads) as bf16 hi + lo, transposed in registers
          const uint32_t ha = pack_bf16x2(p0, p1), hb = pack_bf16x2(p2, p3);
          const uint32_t la = pack_bf16x2(p0 - bf16_lo(ha), p1 - bf16_hi(ha));
          const uint32_t lb = pack_bf16x2(p2 - bf16_lo(hb), p3 - bf16_hi(hb));
          const uint32_t b0h = movmatrix_trans(ha), b1h = movmatrix_trans(hb);
          const uint32_t b0l = movmatrix_trans(la), b1l = movmatrix_trans(lb);
          {
            const int rr = tile * 16 + ((mi >> 1) << 3) + lr;
#pragma unroll
            for (int mt = 0; mt < KT; ++mt) {
              const int d = mt * 16 + ((mi & 1) << 3);
              uint32_t vf[4];
              ldsm_x4_trans(vf, vbase + (d >> 6) * C::kHalfBytes + swz128(rr, (d & 63) >> 3));
              mma_16816(acc[mt], vf, b0h, b1h);
              mma_16816(acc[mt], vf, b0l, b1l);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[buf]);
      }
      i += cnt;

      // ---- end of row: merge the four warp states in shared memory
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, off);
        l1 += __shfl_xor_sync(0xffffffffu, l1, off);
      }
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int hh = tig * 2 + cc;
        if (hh < G) {
          if (gid == 0) {
            wm[warp * G + hh] = cc ? m1 : m0;
            wl[warp * G + hh] = cc ? l1 : l0;
          }
#pragma unroll
          for (int mt = 0; mt < KT; ++mt) {
            wo[(warp * G + hh) * D + mt * 16 + gid] = acc[mt][cc];
            wo[(warp * G + hh) * D + mt * 16 + gid + 8] = acc[mt][2 + cc];
          }
        }
      }
      consumer_bar();
      const int c_first = cta_of(rv0, p.W, p.N);
      const int c_last = cta_of(rv0 + p.V - 1, p.W, p.N);
      const bool whole = (c_first == c_last);
      float *myslot = nullptr;
      if (!whole) {
        const int which = (r == static_cast<int>(s0 / p.V)) ? 0 : 1;
        myslot = p.part + (static_cast<size_t>(c) * 2 + which) * SL;
      }
      const size_t obase = static_cast<size_t>(rg.b) * a.Hq + rg.qh0;
      for (int e = tid; e < G * D; e += kConsumers * 32) {
        const int hh = e / D, d = e % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, wm[w * G + hh]);
        const float base = (M == -INFINITY) ? 0.f : M;
        float o = 0.f, l = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumers; ++w) {
          const float f = fast_exp2(wm[w * G + hh] - base);
          o += f * wo[(w * G + hh) * D + d];
          l += f * wl[w * G + hh];
        }
        if (whole) {
          store_out(a, (obase + hh) * D + d, l > 0.f ? o / l : 0.f);
          if (d == 0 && a.lse != nullptr)
            a.lse[obase + hh] = l > 0.f ? (M + log2f(l)) * kLn2 : -INFINITY;
        } else {
          if (d == 0) {
            myslot[hh] = M;
            myslot[G + hh] = l;
          }
          myslot[2 * G + hh * D + d] = o;
        }
      }
      if (!whole) {
        __threadfence();  // this thread's partial stores before the count
        consumer_bar();
        if (tid == 0) {
          const int old = atomicAdd(&p.sem[r], 1);
          *last_flag = (old == c_last - c_first) ? 1 : 0;
        }
        consumer_bar();
        if (*last_flag) {  // this CTA completes the row: merge the partials
          __threadfence();
          merge_partials<D>(p, r, tid);
          if (tid == 0) p.sem[r] = 0;  // ready for the next call
        }
      }
      consumer_bar();  // the merge area is reused by the next row
    }
  }

  __syncthreads();
  if (*abort_flag != 0u && warp >= kConsumers) {
    // a wait gave up: let every copy the producers issued land before the CTA
    // exits (each wait bounded again); a token-list producer waits for its own
    // buffers, those of its stages' parity
    if (MODE != kModeCp) {
      if (lane < NS && issued > 0) mbar_wait(&full[lane], static_cast<uint32_t>(issued - 1) & 1u);
    } else if (lane == 0) {
      constexpr int NP = attn_producers<MODE>();
      for (int buf = warp - kConsumers; buf < NS && buf < issued; buf += NP) {
        const int uses = (issued - 1 - buf) / NS + 1;
        mbar_wait(&full[buf], static_cast<uint32_t>(uses - 1) & 1u);
      }
    }
  }
}

// Host side: the TMA maps and kernel arguments of an attention call over the
// workspace `ws` (p->N is left at 1 for the launcher to set); *mode is the
// kernel form (kModeDense, kModeTma or kModeCp).  False if a map cannot be
// encoded.
bool attn_prepare(const AttnArgs &a, void *ws, CUtensorMap *km, CUtensorMap *vm, AttnDev *p,
                  int *mode);
// Dynamic shared memory of the attention CTA for G query heads per row (deep:
// the form with three stage buffers per consumer warp).
size_t attn_smem_bytes(int D, int G, bool deep = false);

}  // namespace att
}  // namespace ksa
