// ksa_device.cuh -- device helpers shared by the libksa kernels (sm_100a).
//
// Thin wrappers over PTX instructions (mbarrier, TMA / bulk copies, cp.async,
// ldmatrix, mma.sync, movmatrix) plus block-wide scan and radix select.
// Every wait on an mbarrier is bounded in time: on expiry the caller gets
// `false`, records KSA_FLAG_WAIT_TIMEOUT and leaves its loop, so no kernel can
// spin forever.
#pragma once

#include <cooperative_groups.h>
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ksa.h"

namespace ksa {

namespace cg = cooperative_groups;

constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // 2 s per wait, far above any real wait

// ---------------------------------------------------------------------------
// scalar helpers

__device__ __forceinline__ float bf16_lo(uint32_t packed) { return __uint_as_float(packed << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t packed) {
  return __uint_as_float(packed & 0xffff0000u);
}
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Packs two fp32 values as bf16x2 (round to nearest even): `lo` in bits 0..15.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float x) {
  return static_cast<uint16_t>(pack_bf16x2(x, 0.f) & 0xffffu);
}

// Packs two fp32 values as fp8 e4m3 (round to nearest even, held at +-448):
// `lo` in bits 0..7.
__device__ __forceinline__ uint16_t pack_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// The two fp8 e4m3 values of `v` (bits 0..7 -> .x), exactly, as fp32.
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t v) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(v));
  float lo, hi;
  asm("cvt.f32.f16 %0, %1;" : "=f"(lo) : "h"(static_cast<uint16_t>(h & 0xffffu)));
  asm("cvt.f32.f16 %0, %1;" : "=f"(hi) : "h"(static_cast<uint16_t>(h >> 16)));
  return make_float2(lo, hi);
}

// Scale exponent of an fp8 block: the smallest e with amax <= 448 * 2^e (448 =
// 0.875 * 2^9, so with amax = f 2^E, 0.5 <= f < 1: e = E - 9 if f <= 0.875,
// else E - 8); 0 for an all-zero block.
__device__ __forceinline__ int e4m3_scale_exp(float amax) {
  if (!(amax > 0.f)) return 0;
  int E;
  const float f = frexpf(amax, &E);
  return f <= 0.875f ? E - 9 : E - 8;
}

// 2^x with the hardware approximation (relative error ~2^-22); -inf -> +0.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Order-preserving map of an fp32 score to uint32: a > b  <=>  key(a) > key(b).
// -0.0 and +0.0 map to the same key.  NaN maps to 0 (ranked lowest).
__device__ __forceinline__ uint32_t score_key(float s, bool &is_nan) {
  uint32_t u = __float_as_uint(s);
  is_nan = (u & 0x7fffffffu) > 0x7f800000u;
  if (is_nan) return 0u;
  if ((u & 0x7fffffffu) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ void flag_status(uint32_t *status, uint32_t bits) {
  if (status != nullptr && bits != 0u) atomicOr(status, bits);
}

__device__ __forceinline__ int clamp_len(int len, int cap, uint32_t *status) {
  if (len < 1 || len > cap) {
    flag_status(status, KSA_FLAG_SEQ_LEN_CLAMPED);
    len = len < 0 ? 0 : (len > cap ? cap : len);
  }
  return len;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------------------
// programmatic dependent launch
//
// A kernel reads no input before pdl_wait(), which returns once the previous
// grid on the stream has finished and its memory is visible, and lets its
// dependents launch right after.  launch_pdl launches without the programmatic
// attribute (the calls are then no-ops); launch_programmatic sets it.  Measured
// on the decode step, it pays only where the grid in front is small: the
// attention launch behind the ranking launch (step 90.5 -> 88.3 us), whereas
// the ranking launch behind the scoring launch, or a whole step launched that
// way, got slower (resident early dependents take slots the grid in front
// still needs).

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

constexpr bool kProgrammaticLaunch = false;

template <typename Kernel, typename... Args>
inline cudaError_t launch_pdl(Kernel kernel, dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = kProgrammaticLaunch ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <typename Kernel, typename... Args>
inline cudaError_t launch_programmatic(Kernel kernel, dim3 grid, dim3 block, size_t smem,
                                       cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// ---------------------------------------------------------------------------
// mbarrier

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0u;
}

// Waits for the phase with the given parity to complete; false after the timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitTimeoutNs) return false;
  }
  return true;
}

// ---------------------------------------------------------------------------
// copies into shared memory

// TMA 2D tile load (no multicast): box at (x, y) of `map` into smem `dst`.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 16-byte asynchronous copy global -> shared (bypasses L1).
__device__ __forceinline__ void cp_async_16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src)
               : "memory");
}

// Arrive on `bar` once all cp.async issued so far by this thread have landed.
// Counts as one of the barrier's expected arrivals.
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy (TMA) writes to the same addresses.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tensor-core fragments (mma.sync m16n8k16, bf16 in, fp32 accumulate)

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Transposes an 8x8 b16 matrix held in the standard fragment layout
// (lane l: row l/4, columns 2*(l%4) and 2*(l%4)+1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// Byte offset of 16-byte chunk `c` (0..7) of 128-byte row `r` in a
// 128B-swizzled tile (the layout TMA SWIZZLE_128B writes): chunk ^ (row % 8).
__device__ __forceinline__ uint32_t swz128(int r, int c) {
  return static_cast<uint32_t>(r * 128 + (((c ^ r) & 7) << 4));
}

// ---------------------------------------------------------------------------
// block mean (the block summary of the method), one warp per block

// Mean of the n consecutive bf16 key rows starting at `rows` (row stride D),
// computed by one warp: lane l sums 16-byte chunk l % (D/8) of rows l / (D/8),
// l / (D/8) + 32 / (D/8), ... in row order (every row of the block is one
// in-flight load), partial sums meet by xor-shuffles, then one IEEE division.
// Lanes l < D/8 receive dims [8 (l % (D/8)), +8) in mean[] and return true.
// All 32 lanes must call it with the same arguments.
template <int D>
__device__ __forceinline__ bool warp_block_mean(const uint16_t *rows, int n, float (&mean)[8]) {
  constexpr int CH = D / 8;    // 16-byte chunks per key row
  constexpr int RP = 32 / CH;  // rows covered by one warp-wide load
  const int lane = threadIdx.x & 31;
  const int c = lane % CH, rp = lane / CH;
  const uint16_t *src = rows + c * 8;
#pragma unroll
  for (int i = 0; i < 8; ++i) mean[i] = 0.f;
#pragma unroll 8
  for (int t = rp; t < n; t += RP) {
    const uint4 x = __ldg(reinterpret_cast<const uint4 *>(src + static_cast<size_t>(t) * D));
    mean[0] += bf16_lo(x.x);
    mean[1] += bf16_hi(x.x);
    mean[2] += bf16_lo(x.y);
    mean[3] += bf16_hi(x.y);
    mean[4] += bf16_lo(x.z);
    mean[5] += bf16_hi(x.z);
    mean[6] += bf16_lo(x.w);
    mean[7] += bf16_hi(x.w);
  }
#pragma unroll
  for (int off = CH; off < 32; off <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) mean[i] += __shfl_xor_sync(0xffffffffu, mean[i], off);
  }
  const float fn = static_cast<float>(n);
#pragma unroll
  for (int i = 0; i < 8; ++i) mean[i] = mean[i] / fn;
  return rp == 0;
}

// Stores dims [c8, c8 + 8) of a block mean at element offset `row` of fp32
// summaries, or of bf16 ones (sfmt KSA_SUMMARIES_BF16: rounded to nearest
// even).
__device__ __forceinline__ void store_mean8(void *S, int sfmt, size_t row, int c8,
                                            const float (&m)[8]) {
  if (sfmt == KSA_SUMMARIES_BF16) {
    *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(S) + row + c8) =
        make_uint4(pack_bf16x2(m[0], m[1]), pack_bf16x2(m[2], m[3]), pack_bf16x2(m[4], m[5]),
                   pack_bf16x2(m[6], m[7]));
  } else {
    float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(S) + row + c8);
    dst[0] = make_float4(m[0], m[1], m[2], m[3]);
    dst[1] = make_float4(m[4], m[5], m[6], m[7]);
  }
}

// Stores the mean of block `blk` (flat index over the n_blocks blocks [B, Hkv,
// ceil(T/bs)] of the summaries), held by the lanes l < D/8 (`mine`: dims
// [8 (l % (D/8)), +8) in m[]).  Every writer of summaries goes through here,
// so all of them store the same bits.  fp32 and bf16: per lane.  fp8: the
// block's scale exponent e comes from the warp's largest |mean|, each lane
// stores round_e4m3(m 2^-e) as 8 bytes and lane 0 the scale 2^e (the scales
// follow the n_blocks * D value bytes).  All 32 lanes call it.
template <int D, int FMT>
__device__ __forceinline__ void store_block_mean(void *S, size_t n_blocks, size_t blk, bool mine,
                                                 const float (&m)[8]) {
  const int lane = threadIdx.x & 31;
  const int c8 = (lane % (D / 8)) * 8;
  if (FMT != KSA_SUMMARIES_FP8) {
    if (mine) store_mean8(S, FMT, blk * D, c8, m);
    return;
  }
  float amax = 0.f;
  if (mine) {
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(m[i]));
  }
  // non-negative floats order like their bit patterns
  amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
  const int e = e4m3_scale_exp(amax);
  if (mine) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = pack_e4m3x2(ldexpf(m[2 * i], -e), ldexpf(m[2 * i + 1], -e));
    *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(S) + blk * D + c8) =
        make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
  }
  if (lane == 0)
    reinterpret_cast<float *>(static_cast<uint8_t *>(S) + n_blocks * D)[blk] = ldexpf(1.f, e);
}

// store_block_mean with the format chosen at run time.
template <int D>
__device__ __forceinline__ void store_block_mean_any(void *S, int sfmt, size_t n_blocks,
                                                     size_t blk, bool mine, const float (&m)[8]) {
  if (sfmt == KSA_SUMMARIES_FP8)
    store_block_mean<D, KSA_SUMMARIES_FP8>(S, n_blocks, blk, mine, m);
  else if (sfmt == KSA_SUMMARIES_BF16)
    store_block_mean<D, KSA_SUMMARIES_BF16>(S, n_blocks, blk, mine, m);
  else
    store_block_mean<D, KSA_SUMMARIES_F32>(S, n_blocks, blk, mine, m);
}

// ---------------------------------------------------------------------------
// block-wide helpers

// Exclusive prefix count of `flag` over the block (thread order) plus the total.
// `scratch` holds >= 33 uint32 in shared memory.  All threads must call.
template <int NT>
__device__ __forceinline__ uint32_t block_exclusive_count(bool flag, uint32_t *scratch,
                                                          uint32_t &total) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t ballot = __ballot_sync(0xffffffffu, flag);
  const uint32_t in_warp = __popc(ballot & ((1u << lane) - 1u));
  if (lane == 0) scratch[warp] = __popc(ballot);
  __syncthreads();
  if (warp == 0) {
    uint32_t v = lane < NW ? scratch[lane] : 0u;
    uint32_t incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    if (lane < NW) scratch[lane] = incl - v;
    if (lane == 31) scratch[32] = incl;
  }
  __syncthreads();
  const uint32_t r = scratch[warp] + in_warp;
  total = scratch[32];
  __syncthreads();
  return r;
}

// Radix select on unsigned keys, largest first.  Given n > k >= 1 keys whose
// significant bits are [0, nbits) (nbits a multiple of 8), finds the k-th
// largest key `tau`, the number of keys strictly greater (`n_gt` < k) and the
// number equal to tau (`n_eq`).  keys may live in shared or global memory.
// `hist` holds 256 uint32 and `info` 4 uint32, both in shared memory.
template <int NT>
__device__ void radix_select_desc(const uint32_t *keys, int n, int k, int nbits,
                                  uint32_t *hist, uint32_t *info, uint32_t &tau,
                                  uint32_t &n_gt, uint32_t &n_eq) {
  const int tid = threadIdx.x, lane = tid & 31;
  uint32_t prefix = 0u, pmask = 0u;
  uint32_t remaining = static_cast<uint32_t>(k);  // keys still to take at/below the prefix
  uint32_t above = 0u;                             // keys already known to be greater
  uint32_t eq_count = 0u;
  for (int shift = nbits - 8; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += NT) hist[i] = 0u;
    __syncthreads();
    for (int base = 0; base < n; base += NT) {
      const int i = base + tid;
      bool live = false;
      uint32_t digit = 0u;
      if (i < n) {
        const uint32_t key = keys[i];
        live = (key & pmask) == prefix;
        digit = (key >> shift) & 255u;
      }
      // one atomic per distinct digit per warp
      const uint32_t lmask = __ballot_sync(0xffffffffu, live);
      if (live) {
        const uint32_t same = __match_any_sync(lmask, digit);
        if (lane == __ffs(same) - 1) atomicAdd(&hist[digit], __popc(same));
      }
    }
    __syncthreads();
    if (tid < 32) {
      // lane l owns bins [8l, 8l+8); suffix sums from the top bin down
      uint32_t c[8];
      uint32_t tot = 0u;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = hist[lane * 8 + j];
        tot += c[j];
      }
      uint32_t incl = tot;  // sum over lanes >= this lane
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, incl, off);
        if (lane + off < 32) incl += y;
      }
      uint32_t run = incl - tot;  // keys in bins above this lane's bins
#pragma unroll
      for (int j = 7; j >= 0; --j) {
        const uint32_t before = run;
        run += c[j];
        if (before < remaining && run >= remaining) {
          info[0] = static_cast<uint32_t>(lane * 8 + j);
          info[1] = before;
          info[2] = c[j];
        }
      }
    }
    __syncthreads();
    const uint32_t d = info[0];
    above += info[1];
    remaining -= info[1];
    eq_count = info[2];
    prefix |= d << shift;
    pmask |= 255u << shift;
    __syncthreads();
  }
  tau = prefix;
  n_gt = above;
  n_eq = eq_count;
}

// After radix_select_desc: writes, in ascending index order, the indices of the
// k selected keys (all keys > tau, then the lowest-index keys == tau) to
// out[0..k).  When `out` is null, calls `on_sel(i)` for each selected index
// instead (order unspecified within a chunk).  Returns k.
template <int NT, typename OnSel>
__device__ int select_ascending(const uint32_t *keys, int n, uint32_t tau, uint32_t n_gt,
                                uint32_t n_eq, int k, int32_t *out, uint32_t *scratch,
                                OnSel on_sel) {
  const int tid = threadIdx.x;
  const uint32_t take_eq = static_cast<uint32_t>(k) - n_gt;
  const bool all_eq = (take_eq == n_eq);
  uint32_t eq_seen = 0u, written = 0u;
  for (int base = 0; base < n; base += NT) {
    const int i = base + tid;
    uint32_t key = 0u;
    if (i < n) key = keys[i];
    const bool gt = (i < n) && key > tau;
    const bool eq = (i < n) && key == tau;
    bool sel;
    if (all_eq) {
      sel = gt || eq;
    } else {
      uint32_t tot_eq;
      const uint32_t eq_rank = block_exclusive_count<NT>(eq, scratch, tot_eq) + eq_seen;
      eq_seen += tot_eq;
      sel = gt || (eq && eq_rank < take_eq);
    }
    if (out != nullptr) {
      uint32_t tot_sel;
      const uint32_t pos = block_exclusive_count<NT>(sel, scratch, tot_sel) + written;
      written += tot_sel;
      if (sel) out[pos] = i;
    } else if (sel) {
      on_sel(i);
    }
  }
  return k;
}

}  // namespace ksa
