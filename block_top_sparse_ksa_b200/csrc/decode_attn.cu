// decode_attn.cu -- gathered split-KV flash-decode over a selected token set.
//
// Kinetics (block top-k section): attention runs over the selected blocks'
// tokens only.  LessIsMore (implementation section): one shared token set per
// GQA group, so the G query heads of a kv-head read each K/V row once.
//
// Design (B200, sm_100a):
//  * one thread-block cluster of C CTAs per (row b, kv-head g); CTA rank r
//    takes a contiguous 1/C share of the row's 32-token stages (split-KV);
//  * warp 4 is the producer: per stage it issues TMA tile loads (128B swizzle,
//    no multicast) of the selected K and V rows -- whole blocks / dense runs --
//    or, for token lists, 16-byte cp.async into the same swizzled layout; each
//    stage buffer has a full and an empty mbarrier (bounded waits);
//  * warps 0-3 consume stages round-robin.  The G (<= 8) query heads of the
//    group form the N dimension of mma.sync m16n8k16 tiles: S^T = K_tile q^T
//    (16 tokens x 8 heads, fp32 accumulate), online softmax in fp32 registers,
//    then O^T += V_tile^T P^T with P split into bf16 hi + lo parts (p is
//    carried to ~2^-17 relative), so both contractions run on tensor cores
//    while the kernel stays bound by HBM;
//  * the four warp partials (m, l, o) merge in shared memory, the C CTA
//    partials merge through distributed shared memory, and every CTA writes a
//    1/C slice of the final output (and lse).  No workspace, one launch.
#include <string.h>

#include "ksa_device.cuh"
#include "ksa_internal.h"

namespace ksa {

namespace {

constexpr int kStageTok = 32;
constexpr int kConsumers = 4;
constexpr int kAttnThreads = (kConsumers + 1) * 32;
constexpr float kLn2 = 0.6931471805599453f;

enum { kModeDense = 0, kModeTma = 1, kModeCp = 2 };

template <int D>
struct Cfg {
  static constexpr int kHalves = D / 64;                // 64-column (128-byte) halves of a row
  static constexpr int kHalfBytes = kStageTok * 128;    // one half of a 32-row tile
  static constexpr int kTileBytes = kHalves * kHalfBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;    // K tile + V tile
  static constexpr int kStages = (D == 128) ? 6 : 12;
  static constexpr int kKT = D / 16;
  static constexpr size_t kSmemBytes =
      1024 + static_cast<size_t>(kStages) * kStageBytes + 2 * 8 * kStages + 4 * kStages + 64;
};

struct AttnDev {
  AttnArgs a;
  int csize;
  float scale_log2;
};

struct StageSpan {
  long long t0;  // first token of the segment
  int nvalid;    // rows of the segment below L
  bool entry;    // the segment comes from a real list entry
};

// Segment u (one per lane) of stage `stage` of a row.  Dense and TMA modes.
__device__ __forceinline__ StageSpan stage_segment(int mode, int stage, int u, int tpi, int L,
                                                   const int32_t *list, int n_idx) {
  StageSpan sp{0, 0, false};
  if (mode == kModeDense) {
    if (u == 0) {
      sp.t0 = static_cast<long long>(stage) * kStageTok;
      sp.nvalid = static_cast<int>(min(static_cast<long long>(kStageTok), L - sp.t0));
      sp.entry = true;
    }
    return sp;
  }
  const int seg = tpi < kStageTok ? tpi : kStageTok;
  const int nseg = kStageTok / seg;
  if (u >= nseg) return sp;
  int e, part;
  if (tpi >= kStageTok) {
    e = stage / (tpi / kStageTok);
    part = stage % (tpi / kStageTok);
  } else {
    e = stage * nseg + u;
    part = 0;
  }
  if (e >= n_idx) return sp;
  const int id = list[e];
  sp.entry = true;
  if (id < 0) return sp;
  sp.t0 = static_cast<long long>(id) * tpi + static_cast<long long>(part) * kStageTok;
  const long long left = L - sp.t0;
  sp.nvalid = static_cast<int>(left <= 0 ? 0 : (left < seg ? left : seg));
  return sp;
}

template <int D, int MODE>
__global__ void __launch_bounds__(kAttnThreads, 2)
    sparse_decode_attn_kernel(const __grid_constant__ CUtensorMap kmap,
                              const __grid_constant__ CUtensorMap vmap, const AttnDev p) {
  using C = Cfg<D>;
  constexpr int NS = C::kStages;
  constexpr int KT = C::kKT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *stages = smem;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + static_cast<size_t>(NS) * C::kStageBytes);
  uint64_t *empty = full + NS;
  uint32_t *stage_mask = reinterpret_cast<uint32_t *>(empty + NS);
  uint32_t *abort_flag = stage_mask + NS;

  const AttnArgs &a = p.a;
  cg::cluster_group cluster = cg::this_cluster();
  const int csize = p.csize;
  const int rank = static_cast<int>(cluster.block_rank());
  const int row = blockIdx.x / csize;
  const int b = row / a.Hkv, g = row % a.Hkv;
  const int G = a.Hq / a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  const bool lead = (rank == 0 && tid == 0);
  const int L = clamp_len(a.seq_lens[b], a.T, lead ? a.status : nullptr);
  const int32_t *list = nullptr;
  int n_idx = 0;
  const int tpi = a.tpi;
  if (MODE != kModeDense) {
    list = a.shared ? a.idx + static_cast<size_t>(b) * a.cap
                    : a.idx + static_cast<size_t>(row) * a.cap;
    n_idx = a.shared ? a.num_idx[b] : a.num_idx[row];
    if (n_idx < 0 || n_idx > a.cap) {
      if (lead) flag_status(a.status, KSA_FLAG_INDEX_SKIPPED);
      n_idx = n_idx < 0 ? 0 : a.cap;
    }
  }
  long long n_st;
  if (MODE == kModeDense)
    n_st = (L + kStageTok - 1) / kStageTok;
  else if (tpi >= kStageTok)
    n_st = static_cast<long long>(n_idx) * (tpi / kStageTok);
  else
    n_st = (static_cast<long long>(n_idx) * tpi + kStageTok - 1) / kStageTok;
  const int s_begin = static_cast<int>(n_st * rank / csize);
  const int n_my = static_cast<int>(n_st * (rank + 1) / csize) - s_begin;

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], MODE == kModeCp ? 33u : 1u);
      mbar_init(&empty[s], 1u);
    }
    *abort_flag = 0u;
    fence_mbar_init();
  }
  __syncthreads();

  // per-warp online-softmax state (consumers only): running max m, sum l and
  // O^T accumulators for the lane's two heads 2*(lane%4), 2*(lane%4)+1
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float acc[KT][4];
#pragma unroll
  for (int mt = 0; mt < KT; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;

  int issued = 0;  // stages the producer filled

  if (warp == kConsumers) {
    // ------------------------------------------------------------ producer
    if (MODE != kModeCp && lane == 0) {
      prefetch_tensormap(&kmap);
      prefetch_tensormap(&vmap);
    }
    uint32_t skipped = 0u;
    for (int i = 0; i < n_my; ++i) {
      const int buf = i % NS;
      if (i >= NS &&
          !__all_sync(0xffffffffu,
                      mbar_wait(&empty[buf], static_cast<uint32_t>((i / NS) - 1) & 1u))) {
        if (lane == 0) {
          atomicExch(abort_flag, 1u);
          flag_status(a.status, KSA_FLAG_WAIT_TIMEOUT);
        }
        break;
      }
      issued = i + 1;
      const int stage = s_begin + i;
      uint8_t *sK = stages + static_cast<size_t>(buf) * C::kStageBytes;
      uint8_t *sV = sK + C::kTileBytes;
      if (MODE != kModeCp) {
        const StageSpan sp = stage_segment(MODE, stage, lane, tpi, L, list, n_idx);
        const int seg = (MODE == kModeDense || tpi >= kStageTok) ? kStageTok : tpi;
        if (sp.entry && sp.nvalid == 0 && (MODE == kModeDense || sp.t0 % tpi == 0))
          skipped = KSA_FLAG_INDEX_SKIPPED;
        uint32_t bits = 0u;
        if (sp.nvalid > 0)
          bits = (sp.nvalid >= 32 ? 0xffffffffu : ((1u << sp.nvalid) - 1u)) << (lane * seg);
        const uint32_t mask = __reduce_or_sync(0xffffffffu, bits);
        const uint32_t issuing = __ballot_sync(0xffffffffu, sp.nvalid > 0);
        const uint32_t bytes = static_cast<uint32_t>(__popc(issuing)) * seg * 128u * C::kHalves * 2u;
        if (lane == 0) {
          stage_mask[buf] = mask;
          mbar_arrive_expect_tx(&full[buf], bytes);
        }
        __syncwarp();
        if (sp.nvalid > 0) {
          const int yrow = static_cast<int>(static_cast<long long>(row) * a.T + sp.t0);
#pragma unroll
          for (int h = 0; h < C::kHalves; ++h) {
            tma_load_2d(sK + h * C::kHalfBytes + lane * seg * 128, &kmap, h * 64, yrow, &full[buf]);
            tma_load_2d(sV + h * C::kHalfBytes + lane * seg * 128, &vmap, h * 64, yrow, &full[buf]);
          }
        }
      } else {
        // token lists: row r of the stage <- entry stage*32/tpi + r/tpi, token offset r%tpi
        const int per = kStageTok / tpi;
        const int e = stage * per + lane / tpi;
        bool valid = false;
        long long t = 0;
        if (e < n_idx) {
          const int id = list[e];
          t = static_cast<long long>(id) * tpi + (lane % tpi);
          valid = id >= 0 && t < L;
          if (!valid && (lane % tpi) == 0 && (id < 0 || static_cast<long long>(id) * tpi >= L))
            skipped = KSA_FLAG_INDEX_SKIPPED;
        }
        const uint32_t mask = __ballot_sync(0xffffffffu, valid);
        constexpr int CH = D / 8;          // 16-byte chunks per row
        constexpr int RPW = 32 / CH;       // rows per warp instruction
        const int my_c = lane % CH;
        for (int r0 = 0; r0 < kStageTok; r0 += RPW) {
          const int r = r0 + lane / CH;
          const int rv = __shfl_sync(0xffffffffu, static_cast<int>(valid), r);
          const long long rt = __shfl_sync(0xffffffffu, t, r);
          if (rv) {
            const size_t src = (static_cast<size_t>(row) * a.T + rt) * D + my_c * 8;
            const uint32_t off = (my_c >> 3) * C::kHalfBytes + swz128(r, my_c & 7);
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
    if (skipped && lane == 0) flag_status(a.status, skipped);
  } else {
    // ------------------------------------------------------------ consumers
    const int gid = lane >> 2, tig = lane & 3;
    uint32_t qb[KT][2];
    {
      const uint16_t *qrow = a.q + (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(g) * G + gid) * D;
#pragma unroll
      for (int ks = 0; ks < KT; ++ks) {
        if (gid < G) {
          qb[ks][0] = *reinterpret_cast<const uint32_t *>(qrow + ks * 16 + tig * 2);
          qb[ks][1] = *reinterpret_cast<const uint32_t *>(qrow + ks * 16 + 8 + tig * 2);
        } else {
          qb[ks][0] = 0u;
          qb[ks][1] = 0u;
        }
      }
    }
    const float sl2 = p.scale_log2;

    const int mi = lane >> 3, lr = lane & 7;
    for (int i = warp; i < n_my; i += kConsumers) {
      const int buf = i % NS;
      if (!__all_sync(0xffffffffu, mbar_wait(&full[buf], static_cast<uint32_t>(i / NS) & 1u))) {
        if (lane == 0) {
          atomicExch(abort_flag, 1u);
          flag_status(a.status, KSA_FLAG_WAIT_TIMEOUT);
        }
        break;
      }
      const uint32_t mask = stage_mask[buf];
      uint8_t *sK = stages + static_cast<size_t>(buf) * C::kStageBytes;
      uint8_t *sV = sK + C::kTileBytes;
      if (mask != 0xffffffffu) {
        // rows past L / skipped entries: zero V so that p = 0 meets finite values
        for (int r = 0; r < kStageTok; ++r) {
          if (!((mask >> r) & 1u) && lane < C::kHalves * 8) {
            *reinterpret_cast<uint4 *>(sV + (lane >> 3) * C::kHalfBytes + r * 128 + (lane & 7) * 16) =
                make_uint4(0u, 0u, 0u, 0u);
          }
        }
        if (MODE != kModeCp) fence_proxy_async_smem();
        __syncwarp();
      }
      const uint32_t kbase = smem_addr(sK), vbase = smem_addr(sV);
#pragma unroll
      for (int tile = 0; tile < 2; ++tile) {
        float s[4] = {0.f, 0.f, 0.f, 0.f};
        {
          const int r = tile * 16 + lr + ((mi & 1) << 3);
#pragma unroll
          for (int ks = 0; ks < KT; ++ks) {
            const int d = ks * 16 + ((mi >> 1) << 3);
            uint32_t af[4];
            ldsm_x4(af, kbase + (d >> 6) * C::kHalfBytes + swz128(r, (d & 63) >> 3));
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
          const int r = tile * 16 + ((mi >> 1) << 3) + lr;
#pragma unroll
          for (int mt = 0; mt < KT; ++mt) {
            const int d = mt * 16 + ((mi & 1) << 3);
            uint32_t vf[4];
            ldsm_x4_trans(vf, vbase + (d >> 6) * C::kHalfBytes + swz128(r, (d & 63) >> 3));
            mma_16816(acc[mt], vf, b0h, b1h);
            mma_16816(acc[mt], vf, b0l, b1l);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[buf]);
    }
    // lane-partial sums -> per-head sums (lanes with equal tig share heads)
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, off);
      l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
  }
  // every warp has left its stage loop
  __syncthreads();
  if (*abort_flag != 0u) {
    // a wait gave up: let every copy the producer issued land before the stage
    // memory is reused or the CTA exits (each wait bounded again)
    if (warp == kConsumers && lane == 0) {
      for (int buf = 0; buf < NS && buf < issued; ++buf) {
        const int uses = (issued - 1 - buf) / NS + 1;
        mbar_wait(&full[buf], static_cast<uint32_t>(uses - 1) & 1u);
      }
    }
    __syncthreads();
  }
  // stage memory is free for the merge
  if (warp < kConsumers) {
    float *part = reinterpret_cast<float *>(stages);
    float *wm = part;       // [4][8]
    float *wl = part + 32;  // [4][8]
    float *wo = part + 64;  // [4][8][D]
    const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int hh = tig * 2 + c;
      if (hh < G) {
        if (gid == 0) {
          wm[warp * 8 + hh] = c ? m1 : m0;
          wl[warp * 8 + hh] = c ? l1 : l0;
        }
#pragma unroll
        for (int mt = 0; mt < KT; ++mt) {
          wo[(warp * 8 + hh) * D + mt * 16 + gid] = acc[mt][c];
          wo[(warp * 8 + hh) * D + mt * 16 + gid + 8] = acc[mt][2 + c];
        }
      }
    }
  }
  __syncthreads();

  // ------------------------------------------------------------ merge
  {
    float *part = reinterpret_cast<float *>(stages);
    const float *wm = part, *wl = part + 32, *wo = part + 64;
    float *cm = part + 64 + 4 * 8 * D;  // [8]
    float *cl = cm + 8;                 // [8]
    float *co = cl + 8;                 // [8][D]
    for (int e = tid; e < G * D; e += kAttnThreads) {
      const int hh = e / D, d = e % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, wm[w * 8 + hh]);
      const float base = (M == -INFINITY) ? 0.f : M;
      float o = 0.f, l = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumers; ++w) {
        const float f = fast_exp2(wm[w * 8 + hh] - base);
        o += f * wo[(w * 8 + hh) * D + d];
        l += f * wl[w * 8 + hh];
      }
      co[hh * D + d] = o;
      if (d == 0) {
        cm[hh] = M;
        cl[hh] = l;
      }
    }
    cluster.sync();  // every CTA partial of the row is ready
    const int GD = G * D;
    const int e0 = static_cast<int>(static_cast<long long>(GD) * rank / csize);
    const int e1 = static_cast<int>(static_cast<long long>(GD) * (rank + 1) / csize);
    for (int e = e0 + tid; e < e1; e += kAttnThreads) {
      const int hh = e / D, d = e % D;
      float M = -INFINITY;
      for (int q = 0; q < csize; ++q) M = fmaxf(M, *cluster.map_shared_rank(cm + hh, q));
      const float base = (M == -INFINITY) ? 0.f : M;
      float o = 0.f, l = 0.f;
      for (int q = 0; q < csize; ++q) {
        const float f = fast_exp2(*cluster.map_shared_rank(cm + hh, q) - base);
        o += f * *cluster.map_shared_rank(co + hh * D + d, q);
        l += f * *cluster.map_shared_rank(cl + hh, q);
      }
      const float res = l > 0.f ? o / l : 0.f;
      const size_t oi = (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(g) * G + hh) * D + d;
      if (a.out_f32 != nullptr)
        a.out_f32[oi] = res;
      else
        a.out_bf16[oi] = f32_to_bf16_bits(res);
      if (d == 0 && a.lse != nullptr)
        a.lse[static_cast<size_t>(b) * a.Hq + static_cast<size_t>(g) * G + hh] =
            l > 0.f ? (M + log2f(l)) * kLn2 : -INFINITY;
    }
    cluster.sync();  // remote reads done before any CTA of the cluster exits
  }
}

template <int D, int MODE>
cudaError_t launch_one(const CUtensorMap &km, const CUtensorMap &vm, const AttnDev &p, int grid,
                       cudaStream_t stream) {
  const size_t smem = Cfg<D>::kSmemBytes;
  cudaError_t err = cudaFuncSetAttribute(sparse_decode_attn_kernel<D, MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kAttnThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, sparse_decode_attn_kernel<D, MODE>, km, vm, p);
}

}  // namespace

cudaError_t launch_sparse_decode_attn(const AttnArgs &a, int num_sms, cudaStream_t stream) {
  const int mode = a.idx == nullptr ? kModeDense : (a.tpi >= 16 ? kModeTma : kModeCp);
  CUtensorMap km, vm;
  memset(&km, 0, sizeof km);
  memset(&vm, 0, sizeof vm);
  if (mode != kModeCp) {
    const int box_rows = (mode == kModeDense || a.tpi >= kStageTok) ? kStageTok : a.tpi;
    const uint64_t rows = static_cast<uint64_t>(a.B) * a.Hkv * a.T;
    if (!encode_kv_tensor_map(&km, a.K, rows, a.D, box_rows) ||
        !encode_kv_tensor_map(&vm, a.V, rows, a.D, box_rows))
      return cudaErrorInvalidValue;
  }
  const long long rows_bg = static_cast<long long>(a.B) * a.Hkv;
  long long n_st_max;
  if (mode == kModeDense)
    n_st_max = (a.T + kStageTok - 1) / kStageTok;
  else if (a.tpi >= kStageTok)
    n_st_max = static_cast<long long>(a.cap) * (a.tpi / kStageTok);
  else
    n_st_max = (static_cast<long long>(a.cap) * a.tpi + kStageTok - 1) / kStageTok;
  long long csize = (8LL * num_sms + rows_bg - 1) / rows_bg;
  if (csize > n_st_max / 2) csize = n_st_max / 2;
  csize = csize < 1 ? 1 : (csize > 8 ? 8 : csize);
  AttnDev p;
  p.a = a;
  p.csize = static_cast<int>(csize);
  p.scale_log2 = static_cast<float>(static_cast<double>(a.scale) * 1.4426950408889634);
  const int grid = static_cast<int>(rows_bg * csize);
  if (a.D == 128) {
    if (mode == kModeDense) return launch_one<128, kModeDense>(km, vm, p, grid, stream);
    if (mode == kModeTma) return launch_one<128, kModeTma>(km, vm, p, grid, stream);
    return launch_one<128, kModeCp>(km, vm, p, grid, stream);
  }
  if (mode == kModeDense) return launch_one<64, kModeDense>(km, vm, p, grid, stream);
  if (mode == kModeTma) return launch_one<64, kModeTma>(km, vm, p, grid, stream);
  return launch_one<64, kModeCp>(km, vm, p, grid, stream);
}

}  // namespace ksa
