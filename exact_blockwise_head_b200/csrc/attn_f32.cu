// attn_f32.cu -- exact blockwise attention forward in full fp32 on the CUDA
// cores (no tensor cores: TF32 would lose the precision this path exists for).
//
// Same method as the tensor-core path -- key tiles staged in shared memory, a
// running max and sum carried across them and the partial output rescaled
// whenever the max grows ("Mosaic multi-GPU sequence-sharded attention",
// section 3.2, with the missing rescale supplied) -- but every product and
// exponential is fp32 (expf).  The naive per-thread kernel of "Transformer
// multi-head attention, 8-head parallel computation" (lshu.cn), section 3.1,
// is the prior art: it dots q_i with k_i only and redoes the whole softmax in
// every thread; here each query row is owned by four threads that split the
// head dimension, and every key is read once per tile from shared memory.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "attn.h"
#include "kernels.h"
#include "tiles.h"

namespace ebh {
namespace {

constexpr int kRows = 64;      // query rows per CTA
constexpr int kParts = 4;      // threads per query row (split the head dim)
constexpr int kKeyTile = 32;   // keys per shared-memory tile
constexpr int kThreadsF32 = kRows * kParts;

// DPT = head-dim elements per thread; the head dim is padded to kParts * DPT.
template <int DPT>
__global__ void __launch_bounds__(kThreadsF32)
    attn_fwd_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                        const float* __restrict__ v, float* __restrict__ out,
                        float* __restrict__ lse, int L, int d, float scale, int mask_kind,
                        int window, int Lk, int q_shift) {
  constexpr int DP = kParts * DPT;
  extern __shared__ float sm[];
  float* Ks = sm;                   // [kKeyTile][DP]
  float* Vs = sm + kKeyTile * DP;   // [kKeyTile][DP]

  const int ntiles = (L + kRows - 1) / kRows;
  const int bh = blockIdx.x / ntiles;
  const int q_first = (blockIdx.x % ntiles) * kRows;
  const int q_last = min(q_first + kRows - 1, L - 1);
  const int r = threadIdx.x / kParts;
  const int part = threadIdx.x % kParts;
  const int row = q_first + r;
  const size_t head = static_cast<size_t>(bh) * L * d;      // q, out: L rows per head
  const size_t head_kv = static_cast<size_t>(bh) * Lk * d;  // k, v: Lk rows per head

  // this thread's slice of q: elements part, part + 4, part + 8, ...
  float qv[DPT], o[DPT];
#pragma unroll
  for (int i = 0; i < DPT; ++i) {
    const int c = part + kParts * i;
    qv[i] = (row < L && c < d) ? q[head + static_cast<size_t>(row) * d + c] : 0.f;
    o[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;

  int lo, hi;
  // query row r sits at key position r + q_shift
  kv_tile_range(Lk, q_first + q_shift, q_last + q_shift, mask_kind, window, kKeyTile, lo, hi);
  for (int jt = lo; jt < hi; ++jt) {
    __syncthreads();
    for (int e = threadIdx.x; e < kKeyTile * DP; e += kThreadsF32) {
      const int kr = e / DP, c = e % DP;
      const int key = jt * kKeyTile + kr;
      const bool in = key < Lk && c < d;
      const size_t off = head_kv + static_cast<size_t>(in ? key : 0) * d + (in ? c : 0);
      Ks[e] = in ? k[off] : 0.f;
      Vs[e] = in ? v[off] : 0.f;
    }
    __syncthreads();

    int c_lo, c_hi;
    row_allowed_cols(Lk, row + q_shift, jt, mask_kind, window, kKeyTile, c_lo, c_hi);
    float s[kKeyTile];
    float mt = -INFINITY;
#pragma unroll
    for (int jj = 0; jj < kKeyTile; ++jj) {
      float part_dot = 0.f;
#pragma unroll
      for (int i = 0; i < DPT; ++i) part_dot = fmaf(qv[i], Ks[jj * DP + part + kParts * i], part_dot);
      part_dot += __shfl_xor_sync(0xffffffffu, part_dot, 1);
      part_dot += __shfl_xor_sync(0xffffffffu, part_dot, 2);
      s[jj] = (jj >= c_lo && jj < c_hi) ? part_dot * scale : -INFINITY;
      mt = fmaxf(mt, s[jj]);
    }
    const float m_new = fmaxf(m, mt);
    if (m_new == -INFINITY) continue;  // nothing allowed for this row yet
    const float alpha = expf(m - m_new);  // 0 when m is still -inf
    l *= alpha;
#pragma unroll
    for (int i = 0; i < DPT; ++i) o[i] *= alpha;
#pragma unroll
    for (int jj = 0; jj < kKeyTile; ++jj) {
      const float pj = expf(s[jj] - m_new);
      l += pj;
#pragma unroll
      for (int i = 0; i < DPT; ++i) o[i] = fmaf(pj, Vs[jj * DP + part + kParts * i], o[i]);
    }
    m = m_new;
  }

  if (row < L) {
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int i = 0; i < DPT; ++i) {
      const int c = part + kParts * i;
      if (c < d) out[head + static_cast<size_t>(row) * d + c] = o[i] * inv_l;
    }
    if (part == 0 && lse != nullptr)
      lse[static_cast<size_t>(bh) * L + row] = l > 0.f ? m + logf(l) : -INFINITY;
  }
}

template <int DPT>
int launch_f32_t(const FwdArgs& a, cudaStream_t stream, cudaError_t* err) {
  constexpr int DP = kParts * DPT;
  const int smem = 2 * kKeyTile * DP * static_cast<int>(sizeof(float));
  auto kernel = attn_fwd_f32_kernel<DPT>;
  if (smem > 48 * 1024) {
    int device = 0;
    if ((*err = cudaGetDevice(&device)) != cudaSuccess) return ATTN_ERR_CUDA;
    static std::mutex mu;
    static bool attr_set[64] = {false};
    std::lock_guard<std::mutex> g(mu);
    if (device >= 64) {
      *err = cudaErrorInvalidDevice;
      return ATTN_ERR_CUDA;
    }
    if (!attr_set[device]) {
      *err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (*err != cudaSuccess) return ATTN_ERR_CUDA;
      attr_set[device] = true;
    }
  }
  const long long blocks = static_cast<long long>((a.L + kRows - 1) / kRows) * a.B * a.H;
  if (blocks > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  const dim3 grid(static_cast<unsigned>(blocks));
  kernel<<<grid, kThreadsF32, smem, stream>>>(
      static_cast<const float*>(a.q), static_cast<const float*>(a.k),
      static_cast<const float*>(a.v), static_cast<float*>(a.out), a.lse, a.L, a.d, a.scale,
      a.mask_kind, a.window, a.Lk > 0 ? a.Lk : a.L, a.q_shift);
  *err = cudaGetLastError();
  return *err == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

int launch_fwd_f32(const FwdArgs& a, cudaStream_t stream, cudaError_t* err) {
  *err = cudaSuccess;
  if (a.d <= 64) return launch_f32_t<16>(a, stream, err);
  if (a.d <= 128) return launch_f32_t<32>(a, stream, err);
  if (a.d <= 256) return launch_f32_t<64>(a, stream, err);
  return ATTN_ERR_UNSUPPORTED;
}

}  // namespace ebh
