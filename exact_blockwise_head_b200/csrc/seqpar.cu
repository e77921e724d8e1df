// seqpar.cu -- layout step of sequence-sharded attention.
//
// In "Mosaic multi-GPU sequence-sharded attention" (kwkr.cn), section 2.1,
// each GPU holds one contiguous shard of the sequence.  An all-gather of the
// K (or V) shards leaves them rank-major, [S, B, H, Ls, d]; the forward kernel
// reads each head's keys contiguously, [B, H, S Ls, d].  This kernel moves
// the rows into that order: shard g's row c of head (b, h) becomes key g Ls + c.
#include <cuda_runtime.h>

#include <cstdint>

#include "attn.h"
#include "kernels.h"

namespace ebh {
namespace {

constexpr int kUnshardThreads = 256;

// One thread per 16-byte chunk (rows whose byte length is a multiple of 16).
__global__ void __launch_bounds__(kUnshardThreads)
    unshard_vec16_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int S, int BH,
                         int Ls, int row_chunks) {
  const long long total = static_cast<long long>(S) * BH * Ls * row_chunks;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int chunk = static_cast<int>(e % row_chunks);
    const long long row = e / row_chunks;  // row of the source [S, BH, Ls]
    const int c = static_cast<int>(row % Ls);
    const long long gbh = row / Ls;
    const int bh = static_cast<int>(gbh % BH);
    const int g = static_cast<int>(gbh / BH);
    const long long drow = static_cast<long long>(bh) * S * Ls + static_cast<long long>(g) * Ls + c;
    dst[drow * row_chunks + chunk] = src[e];
  }
}

// Element by element (2- or 4-byte elements), for other row lengths.
template <typename T>
__global__ void __launch_bounds__(kUnshardThreads)
    unshard_elem_kernel(const T* __restrict__ src, T* __restrict__ dst, int S, int BH, int Ls,
                        int d) {
  const long long total = static_cast<long long>(S) * BH * Ls * d;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int col = static_cast<int>(e % d);
    const long long row = e / d;
    const int c = static_cast<int>(row % Ls);
    const long long gbh = row / Ls;
    const int bh = static_cast<int>(gbh % BH);
    const int g = static_cast<int>(gbh / BH);
    const long long drow = static_cast<long long>(bh) * S * Ls + static_cast<long long>(g) * Ls + c;
    dst[drow * d + col] = src[e];
  }
}

}  // namespace

int launch_unshard(const void* src, void* dst, int S, int BH, int Ls, int d, int elem_bytes,
                   cudaStream_t stream, cudaError_t* err) {
  *err = cudaSuccess;
  const long long row_bytes = static_cast<long long>(d) * elem_bytes;
  const bool vec = row_bytes % 16 == 0 && reinterpret_cast<uintptr_t>(src) % 16 == 0 &&
                   reinterpret_cast<uintptr_t>(dst) % 16 == 0;
  const long long units = static_cast<long long>(S) * BH * Ls * (vec ? row_bytes / 16 : d);
  long long blocks = (units + kUnshardThreads - 1) / kUnshardThreads;
  if (blocks > 148LL * 64) blocks = 148LL * 64;  // grid-stride beyond that
  if (blocks < 1) blocks = 1;
  const unsigned grid = static_cast<unsigned>(blocks);
  if (vec) {
    unshard_vec16_kernel<<<grid, kUnshardThreads, 0, stream>>>(
        static_cast<const uint4*>(src), static_cast<uint4*>(dst), S, BH, Ls,
        static_cast<int>(row_bytes / 16));
  } else if (elem_bytes == 2) {
    unshard_elem_kernel<uint16_t><<<grid, kUnshardThreads, 0, stream>>>(
        static_cast<const uint16_t*>(src), static_cast<uint16_t*>(dst), S, BH, Ls, d);
  } else if (elem_bytes == 4) {
    unshard_elem_kernel<uint32_t><<<grid, kUnshardThreads, 0, stream>>>(
        static_cast<const uint32_t*>(src), static_cast<uint32_t*>(dst), S, BH, Ls, d);
  } else {
    return ATTN_ERR_UNSUPPORTED;
  }
  *err = cudaGetLastError();
  return *err == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace ebh
