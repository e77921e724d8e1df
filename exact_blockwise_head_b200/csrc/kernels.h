// kernels.h -- internal interface between the host API (api.cpp) and the
// CUDA translation units.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

namespace ebh {

// One validated forward problem (see include/attn.h for the meaning).
struct FwdArgs {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  float* lse;
  int B, H, L, d;
  float scale;
  int mask_kind;
  int window;       // already clamped to [0, L]
  int block_n;      // 64 or 128 on the bf16 path
  uint64_t timeout_ns;
};

// Each returns an ATTN_* status; on ATTN_ERR_CUDA *err holds the CUDA code.
int launch_fwd_bf16_sm100(const FwdArgs& a, cudaStream_t stream, cudaError_t* err);
int launch_fwd_f32(const FwdArgs& a, cudaStream_t stream, cudaError_t* err);
int launch_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t stream, cudaError_t* err);
int read_device_status(int device, int reset, cudaError_t* err);

}  // namespace ebh
