// ksa_noalloc.cu -- sparse decode attention without any allocation.
//
// ksa_sparse_decode_attn needs a caller-allocated workspace.  Some callers
// cannot allocate device memory: a serving loop that allows no new device
// memory after start-up (cudaMalloc synchronizes the device and can fragment a
// pre-sized pool), or an integration layer that is handed only its input and
// output buffers and owns no allocator.  For them this file keeps one fixed
// scratch area inside the library and runs the same attention kernel on it.
//
// The scratch is a file-scope __device__ array, so every GPU that loads the
// library holds kNoAllocScratchBytes of it until the process exits.  In host
// code the array's name only stands in for it: its device address is looked
// up with cudaGetSymbolAddress on a device's first call, and again whenever
// the device's current context has changed since (a device reset).
#include <mutex>

#include "../../include/ksa.h"
#include "ksa_internal.h"

namespace {

// Largest workspace the no-allocation entry point can serve (8 MiB).  The
// attention workspace is per-(row, kv-head) semaphores (4 bytes each) plus
// partial results of up to two rows per CTA; at G = 8, D = 128 on 148 SMs the
// partials take 4.9 MB, leaving room for semaphores of over 800K rows.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
// Device address of the scratch per device ordinal, with the context it was
// looked up in: after a device reset the primary context is a new one, the old
// address is stale, and the next call looks it up again.
struct ScratchAddr {
  CUcontext ctx;
  void *addr;
};
ScratchAddr g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext *);

// The driver's cuCtxGetCurrent, fetched through the runtime (no link to libcuda).
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of the scratch on the current device (looked up once per
// device and context).
ksa_status scratch_on_current_device(void **out) {
  int dev = -1;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess)
    return ksa::set_last_error(KSA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(err));
  if (dev < 0 || dev >= kMaxDevices)
    return ksa::set_last_error(KSA_ERR_UNSUPPORTED, "device ordinal %d above %d", dev,
                               kMaxDevices - 1);
  const CtxGetCurrentFn get = ctx_get_current();
  if (get == nullptr)
    return ksa::set_last_error(KSA_ERR_CUDA, "cuCtxGetCurrent is not available");
  CUcontext ctx = nullptr;  // null before the runtime has made the device's context
  if (get(&ctx) != CUDA_SUCCESS) ctx = nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchAddr &e = g_scratch_addr[dev];
  if (e.addr == nullptr || ctx == nullptr || e.ctx != ctx) {
    void *p = nullptr;  // (the lookup makes the context if there was none)
    err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (err != cudaSuccess || p == nullptr)
      return ksa::set_last_error(KSA_ERR_CUDA, "cudaGetSymbolAddress of the scratch: %s",
                                 cudaGetErrorString(err));
    if (get(&ctx) != CUDA_SUCCESS || ctx == nullptr)
      return ksa::set_last_error(KSA_ERR_CUDA, "no current CUDA context on device %d", dev);
    e.ctx = ctx;
    e.addr = p;
  }
  *out = e.addr;
  return KSA_OK;
}

}  // namespace

extern "C" ksa_status ksa_sparse_decode_attn_noalloc(
    const ksa_shape *shape, const uint16_t *q, const uint16_t *K, const uint16_t *V,
    const int32_t *seq_lens, const int32_t *idx, const int32_t *num_idx, int32_t idx_capacity,
    int32_t tokens_per_idx, int32_t idx_shared, float scale, int32_t out_dtype, void *out,
    float *lse, uint32_t *dev_status, void *stream) {
  if (shape == nullptr) return ksa::set_last_error(KSA_ERR_INVALID_ARG, "shape is NULL");
  const size_t need = ksa_sparse_decode_attn_workspace(shape, idx_capacity, tokens_per_idx);
  if (need == 0)  // the shape itself is invalid: let the full validation report why
    return ksa_sparse_decode_attn(shape, q, K, V, seq_lens, idx, num_idx, idx_capacity,
                                  tokens_per_idx, idx_shared, scale, out_dtype, out, lse, nullptr,
                                  0, dev_status, stream);
  if (need > kNoAllocScratchBytes)
    return ksa::set_last_error(
        KSA_ERR_UNSUPPORTED,
        "this shape needs %zu bytes of scratch; the no-allocation entry point has %zu "
        "(use ksa_sparse_decode_attn with a workspace)",
        need, kNoAllocScratchBytes);
  void *scratch = nullptr;
  const ksa_status st = scratch_on_current_device(&scratch);
  if (st != KSA_OK) return st;
  // The scratch keeps whatever the previous call left; the per-row semaphores
  // at its start must be zero when the kernel starts.
  // (the semaphore region covers B * Hq rows, the most any list mode uses)
  const size_t rows = static_cast<size_t>(shape->batch) * shape->num_q_heads;
  const size_t sem_bytes = (rows * sizeof(int32_t) + 255) & ~static_cast<size_t>(255);
  const cudaError_t err =
      cudaMemsetAsync(scratch, 0, sem_bytes, static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess)
    return ksa::set_last_error(KSA_ERR_CUDA, "clearing the scratch: %s", cudaGetErrorString(err));
  return ksa_sparse_decode_attn(shape, q, K, V, seq_lens, idx, num_idx, idx_capacity,
                                tokens_per_idx, idx_shared, scale, out_dtype, out, lse, scratch,
                                kNoAllocScratchBytes, dev_status, stream);
}
