// decode_attn.cu -- gathered split-KV flash-decode over a selected token set.
//
// Kinetics (block top-k section): attention runs over the selected blocks'
// tokens only.  LessIsMore (implementation section): one shared token set per
// GQA group, so the G query heads of a kv-head read each K/V row once.
//
// Design (B200, sm_100a):
//  * persistent, stream-K split: the work is the flat sequence of 16-token
//    stages of all (row b, kv-head g) pairs, each row padded to V stages (the
//    most any row can hold); a fixed grid of (SMs x resident CTAs) CTAs takes
//    equal contiguous slices of it, so every CTA streams about the same number
//    of bytes and there is no tail wave (with index lists and between half
//    and all of that many rows, one CTA per row instead: no row is split);
//  * warp 4 is the producer: per stage it issues TMA tile loads (128B swizzle,
//    no multicast) of the selected K and V rows -- whole blocks / dense runs --
//    or, for token lists, 16-byte cp.async into the same swizzled layout; each
//    stage buffer has a full and an empty mbarrier (bounded waits) and belongs
//    to one consumer warp (two buffers per warp, so loads overlap compute);
//  * warps 0-3 consume the stages round-robin.  The G (<= 8) query heads of
//    the group form the N dimension of mma.sync m16n8k16 tiles: S^T = K_tile q^T
//    (16 tokens x 8 heads, fp32 accumulate), online softmax in fp32 registers,
//    then O^T += V_tile^T P^T with P split into bf16 hi + lo parts (p carried to
//    ~2^-17 relative), so both contractions run on tensor cores while the
//    kernel stays bound by HBM;
//  * at the end of each row the four warp states (m, l, o) merge in shared
//    memory (named barrier of the consumer warps only: the producer keeps
//    prefetching the next row).  A row held by one CTA is written out at once;
//    a row split between CTAs leaves a partial in the workspace and bumps the
//    row's semaphore, and the CTA that arrives last merges the partials,
//    writes the output and resets the semaphore to zero.
#include <string.h>

#include "attn_device.cuh"
#include "ksa_device.cuh"
#include "ksa_internal.h"

namespace ksa {

using namespace att;

namespace {

template <int D, int MODE, bool DEEP = false>
__global__ void __launch_bounds__(attn_threads<MODE>(), DEEP ? 2 : 3)
    sparse_decode_attn_kernel(const __grid_constant__ CUtensorMap kmap,
                              const __grid_constant__ CUtensorMap vmap, const AttnDev p) {
  extern __shared__ uint8_t smem_raw[];
  attn_cta<D, MODE, DEEP>(kmap, vmap, p, smem_raw);
}

template <int D, int MODE, bool DEEP>
cudaError_t resident_ctas(const AttnDev &p, int num_sms, long long *n) {
  int occ = 0;
  const cudaError_t err = kernel_occupancy(
      reinterpret_cast<const void *>(sparse_decode_attn_kernel<D, MODE, DEEP>),
      attn_threads<MODE>(), attn_smem_bytes(D, p.gw, DEEP), &occ);
  if (err != cudaSuccess) return err;
  occ = occ < 1 ? 1 : (occ > kAttnMaxCtasPerSm ? kAttnMaxCtasPerSm : occ);
  *n = static_cast<long long>(num_sms) * occ;
  return cudaSuccess;
}

template <int D, int MODE>
cudaError_t launch_one(const CUtensorMap &km, const CUtensorMap &vm, AttnDev p, int num_sms,
                       cudaStream_t stream) {
  long long n = 0;
  cudaError_t err = resident_ctas<D, MODE, false>(p, num_sms, &n);
  if (err != cudaSuccess) return err;
  if (n > p.W) n = p.W;
  if (n < 1) n = 1;
  // With index lists (rows of equal padded length) and between half and all of the
  // resident CTAs' worth of rows, one CTA per row: slices then end on row boundaries, and
  // no row is split, so no CTA ends with a partial merge (measured on the Qwen3-8B shape,
  // 256 rows: attention 61.2 -> 55.0 us).  With block lists:
  //  * one CTA per row, where the rows also fit two deep CTAs per SM (three buffers per
  //    consumer warp), those run: the SMs that hold two rows set the time, and they then
  //    keep half as many bytes again in flight (Qwen3-8B step 100.2 -> 97.7 us);
  //  * more rows than resident CTAs but at most twice the deep grid, an even number,
  //    filling at least 85% of the deep grid with pairs: two whole rows per deep CTA (an
  //    SM holding two CTAs carries twice an SM holding one, so the fill bounds the
  //    imbalance).  Qwen3-0.6B shape, 512 rows in 256 CTAs: attention 57.1 -> 53.7 us.
  //    More rows per CTA measured slower than stream-K on the sweep shapes (80 rows per
  //    CTA at 4K/256: 441 -> 491 us; 4 rows in 160 CTAs at 128K/8192: 424 -> 532 us), and
  //    the 8-stage form with several rows per CTA gained nothing;
  //  * fewer than half the resident CTAs' worth of rows (token lists too): each row is cut
  //    into s = n / rows equal parts, one per CTA, so every CTA holds one piece of one row
  //    (128 rows of 250 stages: block lists 59.3 -> 53.0 us, token lists 59.3 -> 55.9 us;
  //    with one producer warp per CTA the token lists had measured slower this way).
  const long long rows = p.W / p.V;
  bool deep = false;
  if (MODE != kModeDense) {
    if (2 * rows >= n && rows <= n) {
      n = rows;
      if constexpr (MODE == kModeTma) {
        long long n_deep = 0;
        err = resident_ctas<D, MODE, true>(p, num_sms, &n_deep);
        if (err != cudaSuccess) return err;
        deep = rows <= n_deep;
      }
    } else if (2 * rows < n) {
      n = rows * (n / rows);
    } else if constexpr (MODE == kModeTma) {  // rows > n
      long long n_deep = 0;
      err = resident_ctas<D, MODE, true>(p, num_sms, &n_deep);
      if (err != cudaSuccess) return err;
      if (rows <= 2 * n_deep && rows % 2 == 0 && 20 * (rows / 2) >= 17 * n_deep) {
        n = rows / 2;
        deep = true;
      }
    }
  }
  p.N = static_cast<int>(n);
  // programmatic: the CTAs take their places and set up while the grid in
  // front (normally the small ranking launch) finishes
  if constexpr (MODE == kModeTma) {
    if (deep)
      return launch_programmatic(sparse_decode_attn_kernel<D, MODE, true>, dim3(p.N),
                                 dim3(attn_threads<MODE>()), attn_smem_bytes(D, p.gw, true),
                                 stream, km, vm, p);
  }
  return launch_programmatic(sparse_decode_attn_kernel<D, MODE, false>, dim3(p.N),
                             dim3(attn_threads<MODE>()), attn_smem_bytes(D, p.gw, false), stream,
                             km, vm, p);
}

}  // namespace

size_t attn_workspace_bytes(int B, int Hq, int Hkv, int D, int num_sms) {
  const int G = Hq / Hkv;
  const size_t slot = static_cast<size_t>(2 * G + G * D) * sizeof(float);
  const size_t parts = static_cast<size_t>(num_sms) * kAttnMaxCtasPerSm * 2 * slot;
  const size_t sems = static_cast<size_t>(B) * Hq * sizeof(int32_t);  // rows: B*Hkv, or B*Hq
  return ((sems + 255) & ~static_cast<size_t>(255)) + ((parts + 255) & ~static_cast<size_t>(255));
}

namespace att {

size_t attn_smem_bytes(int D, int G, bool deep) {
  const size_t fixed = deep ? (D == 128 ? Cfg<128, true>::kFixedSmem : Cfg<64, true>::kFixedSmem)
                            : (D == 128 ? Cfg<128>::kFixedSmem : Cfg<64>::kFixedSmem);
  return fixed + static_cast<size_t>(kConsumers) * (2 * G + G * D) * 4;
}

bool attn_prepare(const AttnArgs &a, void *ws, CUtensorMap *km, CUtensorMap *vm, AttnDev *pp,
                  int *mode_out) {
  const int mode = a.idx == nullptr ? kModeDense : (a.tpi >= 16 ? kModeTma : kModeCp);
  memset(km, 0, sizeof *km);
  memset(vm, 0, sizeof *vm);
  if (mode != kModeCp) {
    const int box_rows = (mode == kModeDense || a.tpi >= kStageTok) ? kStageTok : a.tpi;
    const uint64_t rows = a.kv.table != nullptr
                              ? static_cast<uint64_t>(a.kv.num_pages) * a.Hkv * a.kv.bs
                              : static_cast<uint64_t>(a.B) * a.Hkv * a.T;
    if (!encode_kv_tensor_map(km, a.K, rows, a.D, box_rows) ||
        !encode_kv_tensor_map(vm, a.V, rows, a.D, box_rows))
      return false;
  }
  long long V;
  if (mode == kModeDense)
    V = (a.T + kStageTok - 1) / kStageTok;
  else if (a.tpi >= kStageTok)
    V = static_cast<long long>(a.cap) * (a.tpi / kStageTok);
  else
    V = (static_cast<long long>(a.cap) * a.tpi + kStageTok - 1) / kStageTok;
  if (V < 1) V = 1;
  AttnDev &p = *pp;
  p.a = a;
  const bool per_q = a.shared == 2;  // one list per query head
  p.rpb = per_q ? a.Hq : a.Hkv;
  p.gw = per_q ? 1 : a.Hq / a.Hkv;
  const long long rows = static_cast<long long>(a.B) * p.rpb;
  p.V = static_cast<int>(V);
  p.W = rows * V;
  p.N = 1;
  p.slot = 2 * p.gw + p.gw * a.D;
  // the semaphore region is sized for B*Hq rows in either case (attn_workspace_bytes)
  const size_t sems = static_cast<size_t>(a.B) * a.Hq * sizeof(int32_t);
  p.sem = static_cast<int32_t *>(ws);
  p.part = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) +
                                     ((sems + 255) & ~static_cast<size_t>(255)));
  p.scale_log2 = static_cast<float>(static_cast<double>(a.scale) * 1.4426950408889634);
  *mode_out = mode;
  return true;
}

}  // namespace att

cudaError_t launch_sparse_decode_attn(const AttnArgs &a, void *ws, int num_sms,
                                      cudaStream_t stream) {
  CUtensorMap km, vm;
  AttnDev p;
  int mode = 0;
  if (!attn_prepare(a, ws, &km, &vm, &p, &mode)) return cudaErrorInvalidValue;
  if (a.D == 128) {
    if (mode == kModeDense) return launch_one<128, kModeDense>(km, vm, p, num_sms, stream);
    if (mode == kModeTma) return launch_one<128, kModeTma>(km, vm, p, num_sms, stream);
    return launch_one<128, kModeCp>(km, vm, p, num_sms, stream);
  }
  if (mode == kModeDense) return launch_one<64, kModeDense>(km, vm, p, num_sms, stream);
  if (mode == kModeTma) return launch_one<64, kModeTma>(km, vm, p, num_sms, stream);
  return launch_one<64, kModeCp>(km, vm, p, num_sms, stream);
}

}  // namespace ksa
