// kernels.h -- internal interface between the host API (api.cpp) and the
// CUDA translation units.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

#include "attn.h"

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
  // Query rows at an offset into the keys: q/out/lse have L rows, k/v have Lk
  // rows (0: Lk = L), and query row i sits at key position q_shift + i.
  int Lk = 0;
  int q_shift = 0;
  // Element strides (row, head, batch) of q, k, v and out on the bf16 path;
  // all zero: dense [B, H, rows, d].
  long long stride[4][3] = {};
  // split-KV partial mode (bf16 path): when o_part is set, the keys are cut
  // into num_splits runs of split_keys (a multiple of block_n) and the kernel
  // writes fp32 partial O [S,B,H,L,d] and partial LSE [S,B,H,L] instead of
  // out / lse.
  int num_splits = 1;
  int split_keys = 0;
  float* o_part = nullptr;
  float* lse_part = nullptr;
  // Programmatic dependent launch: the kernel may start while the previous
  // kernel on the stream finishes (its set-up overlaps that kernel's tail)
  // and waits for it before its first global memory access.
  bool dependent = false;
};

// Merge of split-KV partials: for every row, the splits whose key range
// [bounds[s], bounds[s+1]) holds an allowed key of the row are combined,
// O = sum_s e^(LSE_s - LSE) O_s, LSE = ln sum_s e^(LSE_s).
constexpr int kMaxSplits = 64;
struct MergeArgs {
  const float* o_part;
  const float* lse_part;
  int num_splits;
  int bounds[kMaxSplits + 1];  // key positions, from 0 to kv_len
  void* out;           // bf16 or fp32 [B,H,L,d]
  float* lse;          // fp32 [B,H,L] or nullptr
  bool out_f32;
  int BH, L, d;
  int mask_kind, window;
  // row i of the L rows sits at key position q_offset + i among kv_len keys
  // (0 and L for a plain split-KV merge)
  int kv_len = 0;
  int q_offset = 0;
  // launched as a dependent of the partial kernel before it on the stream
  // (programmatic dependent launch; the kernel waits for it first)
  bool dependent = false;
};

// Each returns an ATTN_* status; on ATTN_ERR_CUDA *err holds the CUDA code.
int launch_fwd_bf16_sm100(const FwdArgs& a, cudaStream_t stream, cudaError_t* err);
int launch_fwd_f32(const FwdArgs& a, cudaStream_t stream, cudaError_t* err);
int launch_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t stream, cudaError_t* err);
int launch_merge(const MergeArgs& m, cudaStream_t stream, cudaError_t* err);
int read_device_status(int device, int reset, cudaError_t* err);

// [S, BH, Ls, d] rank-major rows -> [BH, S Ls, d] (elem_bytes 2 or 4).
int launch_unshard(const void* src, void* dst, int S, int BH, int Ls, int d, int elem_bytes,
                   cudaStream_t stream, cudaError_t* err);

// Backward by recomputation (validated).
struct BwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* out;   // the forward's O
  const void* dout;  // dO, same dtype as q
  const float* lse;  // the forward's natural-log LSE
  float* D;          // workspace: [B, H, L] row dots <dO_i, O_i>
  float* dq;
  float* dk;
  float* dv;
  bool bf16;
  int B, H, L, d;
  float scale;
  int mask_kind, window;
  uint64_t timeout_ns = 10ull * 1000 * 1000 * 1000;  // limit on each wait (tensor-core path)
};
int launch_bwd(const BwdArgs& a, cudaStream_t stream, cudaError_t* err);
// dQ, dK, dV on the tensor cores (bf16, d in {64, 128}); a.D must already
// hold the row dots <dO_i, O_i>.  Defined with the forward kernel.
int launch_bwd_sm100(const BwdArgs& a, cudaStream_t stream, cudaError_t* err);

// The multi-head attention layer (validated).
struct MhaArgs {
  const void* x;       // bf16 [B, L, E]
  const void* w_qkv;   // bf16 [3E, E]
  const void* b_qkv;   // bf16 [3E] or nullptr
  const void* w_out;   // bf16 [E, E]
  const void* b_out;   // bf16 [E] or nullptr
  void* y;             // bf16 [B, L, E]
  int B, L, E, H;
  float scale;
  int mask_kind, window;
  uint64_t timeout_ns;
};
size_t mha_workspace_bytes(int B, int L, int E);
// Y[M, N] = X[M, K] W[N, K]^T + bias[N] (bias may be null), bf16 in and out,
// fp32 accumulation, on the tensor cores; N and K multiples of 8.  Defined
// with the attention kernels.
int launch_linear_bf16(const void* x, const void* w, const void* bias, void* y, int M, int N, int K,
                       uint64_t timeout_ns, cudaStream_t stream, cudaError_t* err,
                       bool dependent = false);
// On failure *err holds the CUDA error and *proj the failing projection (1 the
// qkv projection, 2 the output projection; 0 the attention).
int launch_mha(const MhaArgs& a, void* workspace, cudaStream_t stream, cudaError_t* err,
               int* proj);

// Every argument check of attn_fwd_splitkv except those on the workspace
// (defined in api.cpp).  On ATTN_OK, *runs is the number of key runs the call
// will use and *run_blocks the key blocks per run (the last run may be
// shorter); one run means the call is a plain forward and needs no workspace.
int splitkv_check(const attn_params* p, int num_splits, int* runs, int* run_blocks);

// Records e as this thread's attn_last_cuda_error() (defined in api.cpp).
void set_last_cuda_error(cudaError_t e);

}  // namespace ebh
