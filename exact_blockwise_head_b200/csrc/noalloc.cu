// noalloc.cu -- split-KV forward for callers that cannot allocate device
// memory for a workspace.
//
// attn_fwd_splitkv writes its per-run partial results into a workspace that
// the caller allocates.  Some callers cannot do that: a host framework whose
// caching allocator owns all device memory and must not be bypassed with a
// cudaMalloc, a plugin interface that hands a library only its inputs and
// outputs, or a latency-critical loop where a cudaMalloc/cudaFree (which may
// synchronise the device) is not acceptable.  attn_fwd_splitkv_noalloc serves
// them from one fixed scratch array defined here, ATTN_NOALLOC_SCRATCH_BYTES
// long, which the CUDA runtime places on each device when it loads this
// library's device code there and which stays for the life of the process.
//
// The kernels need the scratch's device address, which belongs to the CUDA
// context it was looked up in.  The first call on a device looks it up
// (cudaGetSymbolAddress, with that device current) and keeps it together with
// the context's unique ID; a later call reuses it only while the same context
// is current, and looks it up again after the context changed (a
// cudaDeviceReset, or another context made current on that device).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <mutex>

#include "attn.h"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = ATTN_NOALLOC_SCRATCH_BYTES;
static_assert(kScratchBytes % 256 == 0, "scratch size must keep 256-byte alignment");

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;

struct ScratchEntry {
  unsigned long long ctx_id;  // unique ID of the context the address belongs to
  void* addr;
};

std::mutex g_scratch_mu;
ScratchEntry g_scratch[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// The driver's cuCtxGetCurrent and cuCtxGetId, found through the runtime once.
cudaError_t driver_fns(CtxGetCurrentFn* get_current, CtxGetIdFn* get_id) {
  static std::once_flag once;
  static CtxGetCurrentFn cur = nullptr;
  static CtxGetIdFn id = nullptr;
  static cudaError_t status = cudaSuccess;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    status = cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q);
    if (status == cudaSuccess && q != cudaDriverEntryPointSuccess) status = cudaErrorNotSupported;
    if (status != cudaSuccess) return;
    cur = reinterpret_cast<CtxGetCurrentFn>(p);
    status = cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q);
    if (status == cudaSuccess && q != cudaDriverEntryPointSuccess) status = cudaErrorNotSupported;
    if (status != cudaSuccess) return;
    id = reinterpret_cast<CtxGetIdFn>(p);
  });
  *get_current = cur;
  *get_id = id;
  return status;
}

// Unique ID of the context current on this thread (0 if none is current).
cudaError_t current_context_id(unsigned long long* ctx_id) {
  CtxGetCurrentFn get_current = nullptr;
  CtxGetIdFn get_id = nullptr;
  cudaError_t e = driver_fns(&get_current, &get_id);
  if (e != cudaSuccess) return e;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  *ctx_id = 0;
  if (ctx == nullptr) return cudaSuccess;
  return get_id(ctx, ctx_id) == CUDA_SUCCESS ? cudaSuccess : cudaErrorDeviceUninitialized;
}

// Device address of the scratch in the context current on this thread.
cudaError_t scratch_in_current_context(void** addr) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  unsigned long long ctx_id = 0;
  if ((e = current_context_id(&ctx_id)) != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchEntry& ent = g_scratch[dev];
  if (ctx_id == 0 || ent.addr == nullptr || ent.ctx_id != ctx_id) {
    // set-up: this makes the device's primary context current if no context
    // was, so the context ID is read again afterwards
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    if (ptr == nullptr) return cudaErrorInvalidSymbol;
    if ((e = current_context_id(&ctx_id)) != cudaSuccess) return e;
    if (ctx_id == 0) return cudaErrorDeviceUninitialized;
    ent.ctx_id = ctx_id;
    ent.addr = ptr;
  }
  *addr = ent.addr;
  return cudaSuccess;
}

}  // namespace

extern "C" int attn_fwd_splitkv_noalloc(const attn_params* p, int num_splits, void* stream) {
  // Every argument is checked exactly as attn_fwd_splitkv checks it, before
  // the scratch limit, so an invalid call reports what is wrong with it.
  int runs = 0, run_blocks = 0;
  const int st = ebh::splitkv_check(p, num_splits, &runs, &run_blocks);
  if (st != ATTN_OK) return st;
  if (runs == 1) return attn_fwd_ex(p, stream);  // one run: no partials, scratch untouched
  if (attn_splitkv_workspace_bytes(p->B, p->H, p->L, p->d, runs) > kScratchBytes)
    return ATTN_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  const cudaError_t e = scratch_in_current_context(&scratch);
  if (e != cudaSuccess) {
    ebh::set_last_cuda_error(e);
    return ATTN_ERR_CUDA;
  }
  // Nothing in the scratch needs to start at zero: the partial kernel writes
  // every (run, row) value that the merge then reads, in the same call.
  return attn_fwd_splitkv(p, num_splits, scratch, kScratchBytes, stream);
}
