// linear_sm100.cuh -- the projections of the multi-head attention layer,
// Y[M, N] = X[M, K] W[N, K]^T + bias[N] in bf16 with fp32 accumulation, on the
// sm_100a tensor cores (included by attn_sm100.cu, which holds every kernel
// that records time-outs in the per-device status word).
//
// "Transformer multi-head attention, 8-head parallel computation" (lshu.cn),
// section 2.1: the layer's Linear(E, 3E) and Linear(E, E).  W is in nn.Linear
// layout (row n makes output feature n), so both X and W are K-major operands,
// like Q and K in the attention's S = Q K^T.
//
// A persistent kernel, one CTA per SM walking 128 x BN output tiles (BN = 256
// when the problem has at least two such tiles per SM, else 128), n fastest so
// that consecutive tiles reuse the same X rows from L2:
//   - a producer warp streams 64-wide K slices of X and W through a
//     four-stage TMA ring (128-byte swizzle), continuing across tiles;
//   - one elected thread of the MMA warp issues tcgen05 MMAs into one of two
//     128 x BN fp32 accumulators in tensor memory, so that the next tile's
//     products run while the previous tile's epilogue drains;
//   - four epilogue warps (one per tensor-memory sub-partition, one output row
//     per thread) add the bias, round to bf16 and write each 32-row x
//     64-column chunk through a swizzled shared-memory box with a TMA store.
// Ragged edges: loads past M, N or K read zeros, and the stores' tensor map
// clips rows past M and columns past N.
#pragma once

namespace ebh {
namespace {

constexpr int kLinBM = 128;   // output rows per tile (tensor-memory lanes)
constexpr int kLinBK = 64;    // K per stage: one 128-byte swizzle row of bf16
constexpr int kLinThreads = 6 * 32;  // producer, MMA, 4 epilogue warps
constexpr int kLinStages = 4;

template <int BN>
struct LinCfg {
  static_assert(BN == 128 || BN == 256, "tile width");
  static constexpr int kTileX = kLinBM * kLinBK * 2;  // 16 KB
  static constexpr int kTileW = BN * kLinBK * 2;      // 16 or 32 KB
  static constexpr int kStageBytes = kTileX + kTileW;
  static constexpr int kBoxBytes = 32 * 128;          // one epilogue warp's 32 x 64 box
  // ring, epilogue boxes, then barriers, tensor-memory address and abort flag
  static constexpr int kSmemBytes = 1024 + kLinStages * kStageBytes + 4 * kBoxBytes + 256;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static constexpr int kBarFull = 0, kBarEmpty = kLinStages, kBarAccFull = 2 * kLinStages,
                       kBarAccEmpty = 2 * kLinStages + 2, kBarDrain = 2 * kLinStages + 4,
                       kNumBars = 2 * kLinStages + 5;
  static constexpr int kTmemCols = 2 * BN;  // two accumulators
};

struct LinearParams {
  const uint16_t* bias;  // bf16 [N] or null
  int M, N, K;
  int tiles_n, num_tiles;
  uint64_t timeout_ns;
};

template <int BN>
__global__ void __launch_bounds__(kLinThreads, 1)
    linear_sm100_kernel(const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_w,
                        const __grid_constant__ CUtensorMap tm_y, const LinearParams p) {
  using C = LinCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t* ring = smem;  // [stage] x (X tile, W tile)
  uint8_t* boxes = smem + kLinStages * C::kStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(boxes + 4 * C::kBoxBytes);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  auto sX = [&](int s) { return ring + s * C::kStageBytes; };
  auto sW = [&](int s) { return ring + s * C::kStageBytes + C::kTileX; };

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  auto bar = [&](int i) -> uint32_t { return smem_addr(&bars[i]); };
  const int n_k = (p.K + kLinBK - 1) / kLinBK;  // a ragged K tail loads as zeros

  if (threadIdx.x == 0) {
    grid_launch_dependents();
    for (int s = 0; s < kLinStages; ++s) {
      mbar_init(bar(C::kBarFull + s), 1);
      mbar_init(bar(C::kBarEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(C::kBarAccFull + b), 1);
      mbar_init(bar(C::kBarAccEmpty + b), 128);
    }
    mbar_init(bar(C::kBarDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_holder), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint64_t limit = p.timeout_ns;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const bool leader = elect_one_sync();
    if (leader) {
      tma_prefetch_desc(&tm_x);
      tma_prefetch_desc(&tm_w);
    }
    // in a dependent launch, X is read from here on; the MMA and epilogue
    // warps touch global memory only after data these loads brought in
    grid_dependency_wait();
    int it = 0;  // K slices issued so far (ring position)
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
      const int m0 = (tile / p.tiles_n) * kLinBM, n0 = (tile % p.tiles_n) * BN;
      for (int kb = 0; kb < n_k; ++kb, ++it) {
        const int s = it % kLinStages;
        if (!(ok = warp_wait(bar(C::kBarEmpty + s), ((it / kLinStages) & 1) ^ 1, abort_flag,
                             limit)))
          break;
        if (leader) {
          mbar_arrive_expect_tx(bar(C::kBarFull + s), C::kStageBytes);
          tma_load_2d(smem_addr(sX(s)), &tm_x, bar(C::kBarFull + s), kb * kLinBK, m0);
          tma_load_2d(smem_addr(sW(s)), &tm_w, bar(C::kBarFull + s), kb * kLinBK, n0);
        }
        __syncwarp();
      }
    }
    // every copy issued must land before the CTA may exit
    for (int s = 0; s < kLinStages; ++s)
      if (it > s) drain_wait(bar(C::kBarFull + s), ((it - 1 - s) / kLinStages) & 1, limit);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const bool leader = elect_one_sync();
    constexpr uint32_t idesc = idesc_bf16_f32(kLinBM, BN, false);
    int it = 0, local = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x, ++local) {
      const int b = local & 1;  // accumulator of this tile
      // the epilogue has read this accumulator's previous tile
      if (!(ok = warp_wait(bar(C::kBarAccEmpty + b), ((local >> 1) & 1) ^ 1, abort_flag, limit)))
        break;
      tc_fence_after();
      const uint32_t acc = tmem + b * BN;
      for (int kb = 0; kb < n_k; ++kb, ++it) {
        const int s = it % kLinStages;
        if (!(ok = warp_wait(bar(C::kBarFull + s), (it / kLinStages) & 1, abort_flag, limit)))
          break;
        tc_fence_after();
        if (leader) {
          const uint64_t da = sdesc_sw128(smem_addr(sX(s)), 16, 1024);
          const uint64_t db = sdesc_sw128(smem_addr(sW(s)), 16, 1024);
#pragma unroll
          for (int k = 0; k < kLinBK / 16; ++k)  // 32 bytes per 16-element K step
            mma_ss(acc, da + ((k * 32) >> 4), db + ((k * 32) >> 4), idesc,
                   (kb > 0 || k > 0) ? 1u : 0u);
          mma_commit(bar(C::kBarEmpty + s));
        }
        __syncwarp();
      }
      if (ok && leader) mma_commit(bar(C::kBarAccFull + b));
      __syncwarp();
    }
    if (leader) mma_commit(bar(C::kBarDrain));
    __syncwarp();
    drain_wait(bar(C::kBarDrain), 0, limit);
  } else {
    // ------------------------------------------------------------ epilogue
    const int sub = warp % 4;  // tensor-memory sub-partition: rows 32 sub ..
    const uint32_t trow = static_cast<uint32_t>(32 * sub) << 16;
    uint8_t* box = boxes + sub * C::kBoxBytes;
    int local = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++local) {
      const int b = local & 1;
      const int m0 = (tile / p.tiles_n) * kLinBM, n0 = (tile % p.tiles_n) * BN;
      if (!warp_wait(bar(C::kBarAccFull + b), (local >> 1) & 1, abort_flag, limit)) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < BN / 64; ++c) {
        uint32_t r[64];
        tmem_ld32(tmem + trow + b * BN + 64 * c, r);
        tmem_ld32(tmem + trow + b * BN + 64 * c + 32, r + 32);
        tmem_wait_ld();
        reg_fence32(r);
        reg_fence32(r + 32);
        if (c == BN / 64 - 1) {  // the whole accumulator has been read
          tc_fence_before();
          mbar_arrive(bar(C::kBarAccEmpty + b));
        }
        // bias of these 64 columns (0 without one or past N): lane l holds
        // columns 2l and 2l + 1, shared across the warp by shuffles
        float b0 = 0.f, b1 = 0.f;
        const int cb = n0 + 64 * c + 2 * lane;
        if (p.bias != nullptr) {
          if (cb < p.N) b0 = __uint_as_float(static_cast<uint32_t>(p.bias[cb]) << 16);
          if (cb + 1 < p.N) b1 = __uint_as_float(static_cast<uint32_t>(p.bias[cb + 1]) << 16);
        }
        if (lane == 0) bulk_wait_group_read0();  // the box's previous store has read it
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 8; ++u) {  // 16-byte units of the row
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int col = 8 * u + 2 * e;  // within the chunk
            const float c0 = __shfl_sync(0xffffffffu, b0, col / 2);
            const float c1 = __shfl_sync(0xffffffffu, b1, col / 2);
            pk[e] = pack_bf16x2(__uint_as_float(r[col]) + c0, __uint_as_float(r[col + 1]) + c1);
          }
          *reinterpret_cast<uint4*>(box + lane * 128 + ((u ^ (lane & 7)) * 16)) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0 && m0 + 32 * sub < p.M && n0 + 64 * c < p.N) {
          tma_store_2d(&tm_y, smem_addr(box), n0 + 64 * c, m0 + 32 * sub);
          bulk_commit_group();
        }
      }
    }
    // the box must have been read before the CTA's shared memory goes; the
    // global writes complete with the kernel
    if (lane == 0) bulk_wait_group_read0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// 2-D bf16 tensor map over a row-major [rows, cols] array: boxes of
// box_rows x 64 columns, 128-byte swizzle.
bool make_map_2d(CUtensorMap* map, const void* base, int rows, int cols, int box_rows,
                 cudaError_t* err) {
  EncodeTiledFn fn = encode_fn(err);
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    *err = cudaErrorInvalidValue;
    return false;
  }
  return true;
}

template <int BN>
int launch_linear_t(const void* x, const void* w, const void* bias, void* y, int M, int N, int K,
                    int nsm, uint64_t timeout_ns, cudaStream_t stream, cudaError_t* err,
                    bool dependent) {
  using C = LinCfg<BN>;
  int device = 0;
  if ((*err = cudaGetDevice(&device)) != cudaSuccess) return ATTN_ERR_CUDA;
  {
    static std::mutex mu;
    static bool done[64] = {};
    std::lock_guard<std::mutex> g(mu);
    if (device < 0 || device >= 64) {
      *err = cudaErrorInvalidDevice;
      return ATTN_ERR_CUDA;
    }
    if (!done[device]) {
      *err = cudaFuncSetAttribute(linear_sm100_kernel<BN>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
      if (*err != cudaSuccess) return ATTN_ERR_CUDA;
      done[device] = true;
    }
  }
  CUtensorMap tx, tw, ty;
  if (!make_map_2d(&tx, x, M, K, kLinBM, err) || !make_map_2d(&tw, w, N, K, BN, err) ||
      !make_map_2d(&ty, y, M, N, 32, err))
    return ATTN_ERR_CUDA;
  LinearParams p;
  p.bias = static_cast<const uint16_t*>(bias);
  p.M = M;
  p.N = N;
  p.K = K;
  p.tiles_n = (N + BN - 1) / BN;
  const long long tiles = static_cast<long long>((M + kLinBM - 1) / kLinBM) * p.tiles_n;
  if (tiles > 0x7fffffffLL) {
    *err = cudaErrorInvalidValue;
    return ATTN_ERR_UNSUPPORTED;
  }
  p.num_tiles = static_cast<int>(tiles);
  p.timeout_ns = timeout_ns;
  const int grid = p.num_tiles < nsm ? p.num_tiles : nsm;
  *err = launch_kernel(linear_sm100_kernel<BN>, grid, kLinThreads, C::kSmemBytes, stream, dependent,
                       tx, tw, ty, p);
  return *err == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

int launch_linear_bf16(const void* x, const void* w, const void* bias, void* y, int M, int N, int K,
                       uint64_t timeout_ns, cudaStream_t stream, cudaError_t* err, bool dependent) {
  *err = cudaSuccess;
  // rows of 16-byte multiples (the tensor maps' stride rule); ragged tiles
  // load zeros past N and K and their stores are clipped at M and N
  if (M <= 0 || N <= 0 || K <= 0 || N % 8 != 0 || K % 8 != 0) return ATTN_ERR_UNSUPPORTED;
  int device = 0;
  if ((*err = cudaGetDevice(&device)) != cudaSuccess) return ATTN_ERR_CUDA;
  const int nsm = sm_count(device, err);
  if (nsm <= 0) return ATTN_ERR_CUDA;
  // 256-wide tiles halve the re-reads of X, but only pay when every SM gets
  // at least two of them
  const long long tiles256 = static_cast<long long>((M + kLinBM - 1) / kLinBM) * ((N + 255) / 256);
  if (tiles256 >= 2LL * nsm)
    return launch_linear_t<256>(x, w, bias, y, M, N, K, nsm, timeout_ns, stream, err, dependent);
  return launch_linear_t<128>(x, w, bias, y, M, N, K, nsm, timeout_ns, stream, err, dependent);
}

}  // namespace ebh
