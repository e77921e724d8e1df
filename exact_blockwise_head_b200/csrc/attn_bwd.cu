// attn_bwd.cu -- backward of the attention forward by recomputation.
//
// "Attention optimisation strategies and practice for long-sequence
// inference" (trdm.cn), section 3.1, and "Mosaic multi-GPU sequence-sharded
// attention" (kwkr.cn), section 2.2: the backward recomputes the attention
// weights from Q, K and the forward's log-sum-exp instead of storing them, so
// memory stays O(L).  With P_ij = exp(scale <q_i, k_j> - lse_i) on the allowed
// pairs:
//   D_i   = <dO_i, O_i>                       (= sum_j P_ij <dO_i, v_j>)
//   dS_ij = P_ij (<dO_i, v_j> - D_i)
//   dV_j  = sum_i P_ij dO_i
//   dK_j  = scale sum_i dS_ij q_i
//   dQ_i  = scale sum_j dS_ij k_j
// Three kernels: D per row; dK and dV per key tile, walking the query rows
// that may attend to it; dQ per query tile, walking its key tiles.  No
// atomics.  fp32 arithmetic on the CUDA cores (inputs bf16 or fp32, gradients
// fp32); four threads share a row and split d.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "attn.h"
#include "kernels.h"
#include "tiles.h"

namespace ebh {
namespace {

constexpr int kParts = 4;           // threads per row
constexpr int kTileRows = 32;       // rows per tile (keys or queries)
constexpr int kBwdThreads = kTileRows * kParts;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__global__ void __launch_bounds__(256)
    bwd_rowdot_kernel(const T* __restrict__ out, const T* __restrict__ dout, float* __restrict__ D,
                      long long rows, int d) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  const T* o = out + row * d;
  const T* g = dout + row * d;
  float acc = 0.f;
  for (int c = lane; c < d; c += 32) acc = fmaf(to_f32(o[c]), to_f32(g[c]), acc);
#pragma unroll
  for (int x = 16; x >= 1; x >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, x);
  if (lane == 0) D[row] = acc;
}

// sum over the four threads of a row
__device__ __forceinline__ float row_sum4(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  return x;
}

// dK, dV for one tile of kTileRows keys of one head.  DPT = columns per thread.
template <typename T, int DPT>
__global__ void __launch_bounds__(kBwdThreads)
    bwd_dkdv_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                    const T* __restrict__ dout, const float* __restrict__ lse,
                    const float* __restrict__ D, float* __restrict__ dk, float* __restrict__ dv,
                    int L, int d, float scale, int mask_kind, int window) {
  constexpr int DP = kParts * DPT;
  __shared__ float Qs[kTileRows][DP];
  __shared__ float Gs[kTileRows][DP];
  __shared__ float lse_s[kTileRows];
  __shared__ float D_s[kTileRows];

  const int ntiles = (L + kTileRows - 1) / kTileRows;
  const int bh = blockIdx.x / ntiles;
  const int k_first = (blockIdx.x % ntiles) * kTileRows;
  const int k_last = min(k_first + kTileRows - 1, L - 1);
  const int r = threadIdx.x / kParts;
  const int part = threadIdx.x % kParts;
  const int j = k_first + r;  // this thread's key
  const size_t head = static_cast<size_t>(bh) * L * d;

  float kr[DPT], vr[DPT], gk[DPT], gv[DPT];
#pragma unroll
  for (int i = 0; i < DPT; ++i) {
    const int c = part + kParts * i;
    const bool in = j < L && c < d;
    kr[i] = in ? to_f32(k[head + static_cast<size_t>(j) * d + c]) : 0.f;
    vr[i] = in ? to_f32(v[head + static_cast<size_t>(j) * d + c]) : 0.f;
    gk[i] = 0.f;
    gv[i] = 0.f;
  }
  int r_lo, r_hi;
  query_rows_for_keys(L, k_first, k_last, mask_kind, window, r_lo, r_hi);
  for (int t0 = (r_lo / kTileRows) * kTileRows; t0 < r_hi; t0 += kTileRows) {
    __syncthreads();
    for (int e = threadIdx.x; e < kTileRows * DP; e += kBwdThreads) {
      const int rr = e / DP, c = e % DP;
      const int i = t0 + rr;
      const bool in = i < L && c < d;
      const size_t off = head + static_cast<size_t>(in ? i : 0) * d + (in ? c : 0);
      Qs[rr][c] = in ? to_f32(q[off]) : 0.f;
      Gs[rr][c] = in ? to_f32(dout[off]) : 0.f;
    }
    if (threadIdx.x < kTileRows) {
      const int i = t0 + threadIdx.x;
      lse_s[threadIdx.x] = i < L ? lse[static_cast<size_t>(bh) * L + i] : 0.f;
      D_s[threadIdx.x] = i < L ? D[static_cast<size_t>(bh) * L + i] : 0.f;
    }
    __syncthreads();
    const int rows = min(kTileRows, L - t0);
    for (int rr = 0; rr < rows; ++rr) {
      const int i = t0 + rr;
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int c = 0; c < DPT; ++c) {
        s = fmaf(Qs[rr][part + kParts * c], kr[c], s);
        dp = fmaf(Gs[rr][part + kParts * c], vr[c], dp);
      }
      s = row_sum4(s);
      dp = row_sum4(dp);
      const bool ok = j < L && pair_allowed(i, j, mask_kind, window);
      const float p = ok ? expf(s * scale - lse_s[rr]) : 0.f;
      const float ds = p * (dp - D_s[rr]) * scale;
#pragma unroll
      for (int c = 0; c < DPT; ++c) {
        gv[c] = fmaf(p, Gs[rr][part + kParts * c], gv[c]);
        gk[c] = fmaf(ds, Qs[rr][part + kParts * c], gk[c]);
      }
    }
  }
  if (j < L) {
#pragma unroll
    for (int i = 0; i < DPT; ++i) {
      const int c = part + kParts * i;
      if (c < d) {
        dk[head + static_cast<size_t>(j) * d + c] = gk[i];
        dv[head + static_cast<size_t>(j) * d + c] = gv[i];
      }
    }
  }
}

// dQ for one tile of kTileRows query rows of one head.
template <typename T, int DPT>
__global__ void __launch_bounds__(kBwdThreads)
    bwd_dq_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  const T* __restrict__ dout, const float* __restrict__ lse,
                  const float* __restrict__ D, float* __restrict__ dq, int L, int d, float scale,
                  int mask_kind, int window) {
  constexpr int DP = kParts * DPT;
  __shared__ float Ks[kTileRows][DP];
  __shared__ float Vs[kTileRows][DP];

  const int ntiles = (L + kTileRows - 1) / kTileRows;
  const int bh = blockIdx.x / ntiles;
  const int q_first = (blockIdx.x % ntiles) * kTileRows;
  const int q_last = min(q_first + kTileRows - 1, L - 1);
  const int r = threadIdx.x / kParts;
  const int part = threadIdx.x % kParts;
  const int i = q_first + r;  // this thread's query row
  const size_t head = static_cast<size_t>(bh) * L * d;

  float qr[DPT], gr[DPT], gq[DPT];
#pragma unroll
  for (int c = 0; c < DPT; ++c) {
    const int col = part + kParts * c;
    const bool in = i < L && col < d;
    qr[c] = in ? to_f32(q[head + static_cast<size_t>(i) * d + col]) : 0.f;
    gr[c] = in ? to_f32(dout[head + static_cast<size_t>(i) * d + col]) : 0.f;
    gq[c] = 0.f;
  }
  const float lse_i = i < L ? lse[static_cast<size_t>(bh) * L + i] : 0.f;
  const float D_i = i < L ? D[static_cast<size_t>(bh) * L + i] : 0.f;
  int lo, hi;
  kv_tile_range(L, q_first, q_last, mask_kind, window, kTileRows, lo, hi);
  for (int jt = lo; jt < hi; ++jt) {
    __syncthreads();
    for (int e = threadIdx.x; e < kTileRows * DP; e += kBwdThreads) {
      const int rr = e / DP, c = e % DP;
      const int j = jt * kTileRows + rr;
      const bool in = j < L && c < d;
      const size_t off = head + static_cast<size_t>(in ? j : 0) * d + (in ? c : 0);
      Ks[rr][c] = in ? to_f32(k[off]) : 0.f;
      Vs[rr][c] = in ? to_f32(v[off]) : 0.f;
    }
    __syncthreads();
    const int keys = min(kTileRows, L - jt * kTileRows);
    for (int rr = 0; rr < keys; ++rr) {
      const int j = jt * kTileRows + rr;
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int c = 0; c < DPT; ++c) {
        s = fmaf(qr[c], Ks[rr][part + kParts * c], s);
        dp = fmaf(gr[c], Vs[rr][part + kParts * c], dp);
      }
      s = row_sum4(s);
      dp = row_sum4(dp);
      const bool ok = i < L && pair_allowed(i, j, mask_kind, window);
      const float p = ok ? expf(s * scale - lse_i) : 0.f;
      const float ds = p * (dp - D_i) * scale;
#pragma unroll
      for (int c = 0; c < DPT; ++c) gq[c] = fmaf(ds, Ks[rr][part + kParts * c], gq[c]);
    }
  }
  if (i < L) {
#pragma unroll
    for (int c = 0; c < DPT; ++c) {
      const int col = part + kParts * c;
      if (col < d) dq[head + static_cast<size_t>(i) * d + col] = gq[c];
    }
  }
}

template <typename T, int DPT>
int launch_bwd_t(const BwdArgs& a, cudaStream_t stream, cudaError_t* err) {
  const long long rows = static_cast<long long>(a.B) * a.H * a.L;
  const long long tiles = static_cast<long long>(a.B) * a.H * ((a.L + kTileRows - 1) / kTileRows);
  if ((rows + 7) / 8 > 0x7fffffffLL || tiles > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  const T* q = static_cast<const T*>(a.q);
  const T* k = static_cast<const T*>(a.k);
  const T* v = static_cast<const T*>(a.v);
  const T* o = static_cast<const T*>(a.out);
  const T* g = static_cast<const T*>(a.dout);
  bwd_rowdot_kernel<T><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(o, g, a.D, rows,
                                                                                a.d);
  if ((*err = cudaGetLastError()) != cudaSuccess) return ATTN_ERR_CUDA;
  bwd_dkdv_kernel<T, DPT><<<static_cast<unsigned>(tiles), kBwdThreads, 0, stream>>>(
      q, k, v, g, a.lse, a.D, a.dk, a.dv, a.L, a.d, a.scale, a.mask_kind, a.window);
  if ((*err = cudaGetLastError()) != cudaSuccess) return ATTN_ERR_CUDA;
  bwd_dq_kernel<T, DPT><<<static_cast<unsigned>(tiles), kBwdThreads, 0, stream>>>(
      q, k, v, g, a.lse, a.D, a.dq, a.L, a.d, a.scale, a.mask_kind, a.window);
  *err = cudaGetLastError();
  return *err == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <typename T>
int launch_bwd_dtype(const BwdArgs& a, cudaStream_t stream, cudaError_t* err) {
  if (a.d <= 32) return launch_bwd_t<T, 8>(a, stream, err);
  if (a.d <= 64) return launch_bwd_t<T, 16>(a, stream, err);
  if (a.d <= 128) return launch_bwd_t<T, 32>(a, stream, err);
  return ATTN_ERR_UNSUPPORTED;
}

}  // namespace

int launch_bwd(const BwdArgs& a, cudaStream_t stream, cudaError_t* err) {
  *err = cudaSuccess;
  if (a.bf16 && (a.d == 64 || a.d == 128)) {
    // D on the CUDA cores (one warp per row), the five products on the
    // tensor cores
    const long long rows = static_cast<long long>(a.B) * a.H * a.L;
    if ((rows + 7) / 8 > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    bwd_rowdot_kernel<__nv_bfloat16><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(a.out), static_cast<const __nv_bfloat16*>(a.dout), a.D,
        rows, a.d);
    if ((*err = cudaGetLastError()) != cudaSuccess) return ATTN_ERR_CUDA;
    return launch_bwd_sm100(a, stream, err);
  }
  return a.bf16 ? launch_bwd_dtype<__nv_bfloat16>(a, stream, err)
                : launch_bwd_dtype<float>(a, stream, err);
}

}  // namespace ebh
