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
// One CTA per 128 x BN output tile (BN = 256 when the problem has enough such
// tiles to fill the GPU twice over, else 128), two CTAs per SM so that one's
// epilogue overlaps the other's main loop: a producer warp streams 64-wide K
// slices of X and W through a TMA ring (128-byte swizzle; two stages at BN =
// 256, three at 128, about 100 KB either way), one elected thread of the MMA
// warp issues tcgen05 MMAs into a 128 x BN fp32 accumulator in tensor memory,
// and four epilogue warps (one per
// tensor-memory sub-partition, one output row per thread) add the bias, round
// to bf16 and stage their 32 rows in the ring -- idle once the accumulator is
// final -- for TMA stores.  Ragged edges: loads past M, N or K read zeros, and
// the stores' tensor map clips rows past M and columns past N.
#pragma once

namespace ebh {
namespace {

constexpr int kLinBM = 128;   // output rows per tile (tensor-memory lanes)
constexpr int kLinBK = 64;    // K per stage: one 128-byte swizzle row of bf16
constexpr int kLinThreads = 6 * 32;  // producer, MMA, 4 epilogue warps

template <int BN>
struct LinCfg {
  static_assert(BN == 128 || BN == 256, "tile width");
  static constexpr int kStages = BN == 256 ? 2 : 3;
  static constexpr int kTileX = kLinBM * kLinBK * 2;  // 16 KB
  static constexpr int kTileW = BN * kLinBK * 2;      // 16 or 32 KB
  static constexpr int kStageBytes = kTileX + kTileW;
  // ring, then barriers, tensor-memory address, abort flag and the bias row
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 2048;
  static constexpr int kBarFull = 0, kBarEmpty = kStages, kBarAcc = 2 * kStages,
                       kBarDrain = 2 * kStages + 1, kNumBars = 2 * kStages + 2;
  // the epilogue's staging (4 warps x 32 rows x BN columns of bf16) reuses the ring
  static_assert(4 * 32 * BN * 2 <= kStages * kStageBytes, "epilogue staging");
};

struct LinearParams {
  const uint16_t* bias;  // bf16 [N] or null
  int M, N, K;
  uint64_t timeout_ns;
};

template <int BN>
__global__ void __launch_bounds__(kLinThreads, 2)
    linear_sm100_kernel(const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_w,
                        const __grid_constant__ CUtensorMap tm_y, const LinearParams p) {
  using C = LinCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t* ring = smem;  // [stage] x (X tile, W tile)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  float* sbias = reinterpret_cast<float*>(tmem_holder + 4);  // [BN]
  auto sX = [&](int s) { return ring + s * C::kStageBytes; };
  auto sW = [&](int s) { return ring + s * C::kStageBytes + C::kTileX; };

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  auto bar = [&](int i) -> uint32_t { return smem_addr(&bars[i]); };
  const int n_tiles_n = (p.N + BN - 1) / BN;
  const int n0 = (blockIdx.x % n_tiles_n) * BN;  // neighbouring CTAs share X rows
  const int m0 = (blockIdx.x / n_tiles_n) * kLinBM;
  const int n_k = (p.K + kLinBK - 1) / kLinBK;  // a ragged K tail loads as zeros

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(C::kBarFull + s), 1);
      mbar_init(bar(C::kBarEmpty + s), 1);
    }
    mbar_init(bar(C::kBarAcc), 1);
    mbar_init(bar(C::kBarDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_holder), BN);
    tmem_relinquish();
  }
  if (warp >= 2) {  // the tile's bias, widened (0 without one or past N)
    for (int c = threadIdx.x - 64; c < BN; c += 128)
      sbias[c] = (p.bias && n0 + c < p.N)
                     ? __uint_as_float(static_cast<uint32_t>(p.bias[n0 + c]) << 16)
                     : 0.f;
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
    int issued = 0;
    for (int kb = 0; kb < n_k; ++kb) {
      const int s = kb % C::kStages;
      if (!warp_wait(bar(C::kBarEmpty + s), ((kb / C::kStages) & 1) ^ 1, abort_flag, limit)) break;
      if (leader) {
        mbar_arrive_expect_tx(bar(C::kBarFull + s), C::kStageBytes);
        tma_load_2d(smem_addr(sX(s)), &tm_x, bar(C::kBarFull + s), kb * kLinBK, m0);
        tma_load_2d(smem_addr(sW(s)), &tm_w, bar(C::kBarFull + s), kb * kLinBK, n0);
      }
      __syncwarp();
      ++issued;
    }
    for (int s = 0; s < C::kStages; ++s)
      if (issued > s)
        drain_wait(bar(C::kBarFull + s), ((issued - 1 - s) / C::kStages) & 1, limit);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const bool leader = elect_one_sync();
    constexpr uint32_t idesc = idesc_bf16_f32(kLinBM, BN, false);
    bool ok = true;
    for (int kb = 0; ok && kb < n_k; ++kb) {
      const int s = kb % C::kStages;
      if (!(ok = warp_wait(bar(C::kBarFull + s), (kb / C::kStages) & 1, abort_flag, limit))) break;
      tc_fence_after();
      if (leader) {
        const uint64_t da = sdesc_sw128(smem_addr(sX(s)), 16, 1024);
        const uint64_t db = sdesc_sw128(smem_addr(sW(s)), 16, 1024);
#pragma unroll
        for (int k = 0; k < kLinBK / 16; ++k)  // 32 bytes per 16-element K step
          mma_ss(tmem, da + ((k * 32) >> 4), db + ((k * 32) >> 4), idesc,
                 (kb > 0 || k > 0) ? 1u : 0u);
        mma_commit(bar(C::kBarEmpty + s));
      }
      __syncwarp();
    }
    if (leader) {
      if (ok) mma_commit(bar(C::kBarAcc));
      mma_commit(bar(C::kBarDrain));
    }
    __syncwarp();
    drain_wait(bar(C::kBarDrain), 0, limit);
  } else {
    // ------------------------------------------------------------ epilogue
    const int sub = warp % 4;  // tensor-memory sub-partition: rows 32 sub ..
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * sub) << 16);
    if (warp_wait(bar(C::kBarAcc), 0, abort_flag, limit)) {
      tc_fence_after();
      // staging: this warp's 32 rows x 64 columns per chunk (4 KB, swizzled),
      // in the ring (every load has been consumed once the accumulator is
      // final)
      uint8_t* box = ring + sub * (BN / 64) * 4096;
#pragma unroll 1
      for (int c = 0; c < BN / 64; ++c) {
        uint32_t r[64];
        tmem_ld32(trow + 64 * c, r);
        tmem_ld32(trow + 64 * c + 32, r + 32);
        tmem_wait_ld();
        reg_fence32(r);
        reg_fence32(r + 32);
        uint8_t* b = box + c * 4096;
#pragma unroll
        for (int u = 0; u < 8; ++u) {  // 16-byte units of the row
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(r[8 * u]) + sbias[64 * c + 8 * u],
                            __uint_as_float(r[8 * u + 1]) + sbias[64 * c + 8 * u + 1]);
          v.y = pack_bf16x2(__uint_as_float(r[8 * u + 2]) + sbias[64 * c + 8 * u + 2],
                            __uint_as_float(r[8 * u + 3]) + sbias[64 * c + 8 * u + 3]);
          v.z = pack_bf16x2(__uint_as_float(r[8 * u + 4]) + sbias[64 * c + 8 * u + 4],
                            __uint_as_float(r[8 * u + 5]) + sbias[64 * c + 8 * u + 5]);
          v.w = pack_bf16x2(__uint_as_float(r[8 * u + 6]) + sbias[64 * c + 8 * u + 6],
                            __uint_as_float(r[8 * u + 7]) + sbias[64 * c + 8 * u + 7]);
          *reinterpret_cast<uint4*>(b + lane * 128 + ((u ^ (lane & 7)) * 16)) = v;
        }
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0 && m0 + 32 * sub < p.M && n0 + 64 * c < p.N) {
          tma_store_2d(&tm_y, smem_addr(b), n0 + 64 * c, m0 + 32 * sub);
          bulk_commit_group();
        }
      }
      // the staging must have been read before the CTA's shared memory goes;
      // the global writes complete with the kernel
      if (lane == 0) bulk_wait_group_read0();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
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
                    uint64_t timeout_ns, cudaStream_t stream, cudaError_t* err) {
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
  p.timeout_ns = timeout_ns;
  const long long ctas = static_cast<long long>((M + kLinBM - 1) / kLinBM) * ((N + BN - 1) / BN);
  if (ctas > 0x7fffffffLL) {
    *err = cudaErrorInvalidValue;
    return ATTN_ERR_UNSUPPORTED;
  }
  linear_sm100_kernel<BN><<<static_cast<unsigned>(ctas), kLinThreads, C::kSmemBytes, stream>>>(
      tx, tw, ty, p);
  *err = cudaGetLastError();
  return *err == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

int launch_linear_bf16(const void* x, const void* w, const void* bias, void* y, int M, int N, int K,
                       uint64_t timeout_ns, cudaStream_t stream, cudaError_t* err) {
  *err = cudaSuccess;
  // rows of 16-byte multiples (the tensor maps' stride rule); ragged tiles
  // load zeros past N and K and their stores are clipped at M and N
  if (M <= 0 || N <= 0 || K <= 0 || N % 8 != 0 || K % 8 != 0) return ATTN_ERR_UNSUPPORTED;
  int device = 0;
  if ((*err = cudaGetDevice(&device)) != cudaSuccess) return ATTN_ERR_CUDA;
  const int nsm = sm_count(device, err);
  if (nsm <= 0) return ATTN_ERR_CUDA;
  // 256-wide tiles halve the re-reads of X, but only when there are enough of
  // them for two CTAs on every SM
  const long long tiles256 = static_cast<long long>((M + kLinBM - 1) / kLinBM) * ((N + 255) / 256);
  if (tiles256 >= 2LL * nsm)
    return launch_linear_t<256>(x, w, bias, y, M, N, K, timeout_ns, stream, err);
  return launch_linear_t<128>(x, w, bias, y, M, N, K, timeout_ns, stream, err);
}

}  // namespace ebh
