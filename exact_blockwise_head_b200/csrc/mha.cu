// mha.cu -- the multi-head attention layer around the attention kernel.
//
// "Transformer multi-head attention, 8-head parallel computation" (lshu.cn),
// sections 2.1 and 2.2, builds the layer as
//   qkv = x W_qkv^T + b_qkv            (one Linear(E, 3E))
//   q, k, v = the three E-wide thirds of qkv, each viewed [B, L, H, d] and
//             transposed to [B, H, L, d]  (d = E / H)
//   context = softmax(q k^T / sqrt(d) + mask) v, transposed back to [B, L, E]
//   y = context W_out^T + b_out        (one Linear(E, E))
// The two projections are dense GEMMs and run in this library's tcgen05 GEMM
// (launch_linear_bf16: bf16 operands, fp32 accumulation in tensor memory, the
// bias added in its epilogue).  The attention kernel reads q, k and v straight
// out of the projection's [B, L, 3, H, d] output through strided tensor maps
// and writes the context in [B, L, H, d], so the head split and merge cost no
// pass of their own.
#include <cuda_runtime.h>

#include <cstdint>

#include "attn.h"
#include "kernels.h"

namespace ebh {
namespace {

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

size_t mha_workspace_bytes(int B, int L, int E) {
  const size_t act = static_cast<size_t>(B) * L * E * 2;  // one [B, L, E] bf16 tensor
  return align256(3 * act) + align256(act);                 // qkv (3) + context (1)
}

int launch_mha(const MhaArgs& a, void* workspace, cudaStream_t stream, cudaError_t* err,
               int* proj) {
  *err = cudaSuccess;
  *proj = 0;
  const int d = a.E / a.H;
  const size_t act = static_cast<size_t>(a.B) * a.L * a.E * 2;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint16_t* qkv = reinterpret_cast<uint16_t*>(ws);
  ws += align256(3 * act);
  void* ctx = ws;
  const int M = a.B * a.L;
  int st = launch_linear_bf16(a.x, a.w_qkv, a.b_qkv, qkv, M, 3 * a.E, a.E, a.timeout_ns, stream,
                              err);
  if (st != ATTN_OK) {
    *proj = 1;
    return st;
  }
  // q, k, v: the three E-wide thirds of each qkv row, head h at columns h d
  FwdArgs f;
  f.q = qkv;
  f.k = qkv + a.E;
  f.v = qkv + 2 * a.E;
  f.out = ctx;
  f.lse = nullptr;
  f.B = a.B;
  f.H = a.H;
  f.L = a.L;
  f.d = d;
  f.scale = a.scale;
  f.mask_kind = a.mask_kind;
  f.window = a.window;
  f.block_n = 128;
  f.timeout_ns = a.timeout_ns;
  // the attention and the output projection start while the kernel before
  // them drains, and wait for it before reading its output
  f.dependent = true;
  const long long E3 = 3LL * a.E;
  for (int x = 0; x < 3; ++x) {
    f.stride[x][0] = E3;
    f.stride[x][1] = d;
    f.stride[x][2] = E3 * a.L;
  }
  f.stride[3][0] = a.E;  // context [B, L, H, d]
  f.stride[3][1] = d;
  f.stride[3][2] = static_cast<long long>(a.E) * a.L;
  st = launch_fwd_bf16_sm100(f, stream, err);
  if (st != ATTN_OK) return st;
  st = launch_linear_bf16(ctx, a.w_out, a.b_out, a.y, M, a.E, a.E, a.timeout_ns, stream, err,
                          /*dependent=*/true);
  if (st != ATTN_OK) *proj = 2;
  return st;
}

}  // namespace ebh
