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
// The kernels need the scratch's device address.  The first call on a device
// looks it up once (cudaGetSymbolAddress, with that device current) and
// keeps it; later calls on that device reuse it.
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
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch on the current device; looked up on the
// first call for that device.
cudaError_t scratch_on_current_device(void** addr) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    if (ptr == nullptr) return cudaErrorInvalidSymbol;
    g_scratch_addr[dev] = ptr;
  }
  *addr = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int attn_fwd_splitkv_noalloc(const attn_params* p, int num_splits, void* stream) {
  if (p == nullptr) return ATTN_ERR_INVALID;
  if (num_splits < 1 || num_splits > ebh::kMaxSplits) return ATTN_ERR_INVALID;
  if (p->B <= 0 || p->H <= 0 || p->L <= 0 || p->d <= 0) return ATTN_ERR_INVALID;
  if (p->block_n != 0 && p->block_n != 64 && p->block_n != 128) return ATTN_ERR_INVALID;
  // The number of runs attn_fwd_splitkv will use (whole key blocks per run)
  // and the scratch their partials take; one run needs no scratch.
  const long long bn = p->block_n == 0 ? 128 : p->block_n;
  const long long nkv = (static_cast<long long>(p->L) + bn - 1) / bn;
  const long long per_run = (nkv + num_splits - 1) / num_splits;
  const int runs = static_cast<int>((nkv + per_run - 1) / per_run);
  if (runs > 1 &&
      attn_splitkv_workspace_bytes(p->B, p->H, p->L, p->d, runs) > kScratchBytes)
    return ATTN_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  const cudaError_t e = scratch_on_current_device(&scratch);
  if (e != cudaSuccess) {
    ebh::set_last_cuda_error(e);
    return ATTN_ERR_CUDA;
  }
  // Nothing in the scratch needs to start at zero: the partial kernel writes
  // every (run, row) value that the merge then reads, in the same call.
  return attn_fwd_splitkv(p, num_splits, scratch, kScratchBytes, stream);
}
