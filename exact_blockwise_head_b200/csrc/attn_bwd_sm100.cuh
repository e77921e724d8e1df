// attn_bwd_sm100.cuh -- backward of the bf16 attention forward on the sm_100a
// tensor cores (included by attn_sm100.cu, which holds every kernel that
// records time-outs in the per-device status word).
//
// "Attention optimisation strategies and practice for long-sequence
// inference" (trdm.cn), section 3.1, and "Mosaic multi-GPU sequence-sharded
// attention" (kwkr.cn), section 2.2: the weights are recomputed from Q, K and
// the forward's log-sum-exp instead of being stored.  With
//   P_ij = exp(scale <q_i, k_j> - lse_i)    on the allowed pairs (else 0),
//   D_i = <dO_i, O_i>,  dS_ij = P_ij (<dO_i, v_j> - D_i):
//   dV_j = sum_i P_ij dO_i,  dK_j = scale sum_i dS_ij q_i,  dQ_i = scale sum_j dS_ij k_j.
// Every product is a dense 128 x 128 x d contraction per (query tile, key
// tile) pair, so all five run as tcgen05 MMAs with fp32 accumulators in
// tensor memory:
//
// dK/dV kernel -- one CTA per 128-key tile of one head; K and V stay in shared
// memory while the query tiles that may attend to the keys stream through a
// two-stage ring (Q, dO, and the rows' LSE and D):
//   S^T  = K Q^T         SS MMA  -> tensor memory [keys x queries]
//   dP^T = V dO^T        SS MMA  -> tensor memory
//   P^T, dS^T            element-wise, written back as bf16 over S^T / dP^T
//   dV  += P^T dO        TS MMA  (A = P^T from tensor memory)
//   dK  += dS^T Q        TS MMA
// dQ kernel -- one CTA per 128-query tile; Q and dO stay, the key tiles it
// visits stream through the ring:
//   S = Q K^T, dP = dO V^T (SS), dS element-wise over S, dQ += dS K (TS).
// No atomics: each gradient row is owned by one CTA.  The element-wise work
// runs on eight warps, two per tensor-memory sub-partition; each thread owns
// one row (one tensor-memory lane) and one half of the 128 columns.  Its bf16
// results go over the first half of its own fp32 columns, so the two warps of
// a sub-partition never overwrite columns the other has yet to read; the
// MMAs read the A operand from those two 32-column runs.
#pragma once

namespace ebh {
namespace {

constexpr int kBwdRows = 128;     // rows per tile (keys or queries; tensor-memory lanes)
constexpr int kBwdEwWarps = 8;    // element-wise warps
constexpr int kBwdEwThreads = kBwdEwWarps * 32;
constexpr int kBwdThreads = (kBwdEwWarps + 4) * 32;  // + producer, MMA, 2 idle
constexpr int kBwdProducerWarp = kBwdEwWarps;
constexpr int kBwdMmaWarp = kBwdEwWarps + 1;
constexpr int kBwdLaunchRegs = (65536 / kBwdThreads) / 8 * 8;  // 168
constexpr int kBwdEwRegs = 216;
constexpr int kBwdOtherRegs = 56;
static_assert(kBwdEwRegs * kBwdEwThreads + kBwdOtherRegs * 128 <= kBwdLaunchRegs * kBwdThreads,
              "register split exceeds the launch allocation");

template <int D>
struct BwdCfg {
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr int kDChunks = D / 64;
  static constexpr int kTileBytes = kBwdRows * D * 2;  // one 128-row bf16 tile
  static constexpr int kVecBytes = 2 * kBwdRows * 4;    // lse * log2(e) and D of 128 rows
  // resident pair, then two stages of (streamed pair + row vectors)
  static constexpr int kStageBytes = 2 * kTileBytes + kVecBytes;
  static constexpr int kSmemBytes = 1024 + 2 * kTileBytes + 2 * kStageBytes + 256;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  // tensor-memory columns
  static constexpr int kColS = 0;          // S^T or S, then P^T / dS (bf16) over it
  static constexpr int kColDP = 128;       // dP^T or dP, then dS^T (bf16) over it
  static constexpr int kColAcc0 = 256;     // dV (dK/dV kernel) or dQ (dQ kernel)
  static constexpr int kColAcc1 = 256 + D; // dK
};

// barrier indices
enum : int {
  kBwBarRes = 0,     // resident pair landed
  kBwBarFull = 1,    // [2] streamed stage landed
  kBwBarEmpty = 3,   // [2] stage free again
  kBwBarS = 5,       // S product done
  kBwBarDP = 6,      // dP product done
  kBwBarP = 7,       // P^T written (dK/dV kernel)
  kBwBarDS = 8,      // dS written
  kBwBarAcc = 9,     // accumulators final
  kBwBarDrain = 10,
  kBwNumBars = 11
};

struct BwdParams {
  const float* lse;   // [BH, L] natural-log LSE of the forward
  const float* dvec;  // [BH, L] D_i = <dO_i, O_i>
  float* dq;
  float* dk;
  float* dv;
  int BH, L, n_tiles;
  int mask_kind, window;
  float scale, scale_log2;
  uint64_t timeout_ns;
};

// Allowed query columns [c_lo, c_hi) of key k among the queries
// [q_base, q_base + ncols) (clipped to queries < L; empty for k >= L): the
// transpose of row_allowed_cols.
__device__ __forceinline__ void key_allowed_cols(int L, int k, int q_base, int ncols,
                                                 int mask_kind, int window, int& c_lo,
                                                 int& c_hi) {
  long long lo = 0, hi = ncols;
  if (static_cast<long long>(L) - q_base < hi) hi = static_cast<long long>(L) - q_base;
  if (k >= L) hi = 0;
  if (mask_kind == kMaskCausal) {
    lo = max(lo, static_cast<long long>(k) - q_base);
  } else if (mask_kind == kMaskWindow) {
    lo = max(lo, static_cast<long long>(k) - window - q_base);
    hi = min(hi, static_cast<long long>(k) + window + 1 - q_base);
  } else if (mask_kind == kMaskCausalWindow) {
    lo = max(lo, static_cast<long long>(k) - q_base);
    hi = min(hi, static_cast<long long>(k) + window + 1 - q_base);
  }
  if (hi < lo) hi = lo;
  if (lo > ncols) lo = ncols;
  if (hi < 0) hi = 0;
  c_lo = static_cast<int>(lo);
  c_hi = static_cast<int>(hi);
}

// Load 64 fp32 columns of this warp's 32 lanes (one row per thread).
__device__ __forceinline__ void bwd_ld64(uint32_t taddr, uint32_t* r) {
  tmem_ld32(taddr, r);
  tmem_ld32(taddr + 32, r + 32);
  tmem_wait_ld();
  reg_fence32(r);
  reg_fence32(r + 32);
}

// 64 values -> 32 packed bf16 pairs (column c, c + 1 in one word), stored over
// the 32 columns at taddr; waits for the store and orders it before a barrier
// arrive.
__device__ __forceinline__ void bwd_st_packed(uint32_t taddr, const float* x) {
  uint32_t pk[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
  tmem_st32(taddr, pk);
  tmem_wait_st();
  tc_fence_before();
}

// The A operand of a TS MMA over 128 packed columns laid out as two runs of
// 32 (one per column half): K-step k (16 elements) of the 8.
__device__ __forceinline__ uint32_t split_a_col(uint32_t base, int k) {
  return base + (k / 4) * 64 + (k % 4) * 8;
}

// Write the thread's 64 (or 32) accumulator columns of row `row` (< L) as fp32,
// times `mul`.
template <int D>
__device__ __forceinline__ void bwd_store_acc(uint32_t taddr, float* dst, float mul, bool ok) {
  constexpr int kCols = D / 2;
  uint32_t r[64];
  tmem_ld32(taddr, r);
  if constexpr (kCols == 64) tmem_ld32(taddr + 32, r + 32);
  tmem_wait_ld();
  reg_fence32(r);
  if constexpr (kCols == 64) reg_fence32(r + 32);
  if (!ok) return;
  if ((reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
    float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int i = 0; i < kCols / 4; ++i)
      d4[i] = make_float4(__uint_as_float(r[4 * i]) * mul, __uint_as_float(r[4 * i + 1]) * mul,
                          __uint_as_float(r[4 * i + 2]) * mul,
                          __uint_as_float(r[4 * i + 3]) * mul);
  } else {  // gradients only 4-byte aligned (the call allows it)
#pragma unroll
    for (int i = 0; i < kCols; ++i) dst[i] = __uint_as_float(r[i]) * mul;
  }
}

// ------------------------------------------------------------ dK, dV
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkdv_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_do, const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t* sK = smem;
  uint8_t* sV = smem + C::kTileBytes;
  uint8_t* stage0 = smem + 2 * C::kTileBytes;  // [2] x (Q, dO, lse2[128], D[128])
  uint64_t* bars = reinterpret_cast<uint64_t*>(stage0 + 2 * C::kStageBytes);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + kBwNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  auto sQ = [&](int st) { return stage0 + st * C::kStageBytes; };
  auto sDO = [&](int st) { return stage0 + st * C::kStageBytes + C::kTileBytes; };
  auto sVec = [&](int st) {
    return reinterpret_cast<float*>(stage0 + st * C::kStageBytes + 2 * C::kTileBytes);
  };

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  auto bar = [&](int i) -> uint32_t { return smem_addr(&bars[i]); };
  // key tiles in ascending order, all heads of tile 0 first: for causal masks
  // the lowest keys have the most query tiles, so the longest CTAs start first
  const int kt = blockIdx.x / p.BH;
  const int bh = blockIdx.x % p.BH;
  const int k0 = kt * kBwdRows;
  const int k_last = min(k0 + kBwdRows - 1, p.L - 1);
  int r_lo, r_hi;
  query_rows_for_keys(p.L, k0, k_last, p.mask_kind, p.window, r_lo, r_hi);
  const int qt_lo = r_lo / kBwdRows;
  const int n_q = r_hi > r_lo ? (r_hi + kBwdRows - 1) / kBwdRows - qt_lo : 0;

  if (threadIdx.x == 0) {
    mbar_init(bar(kBwBarRes), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBwBarFull + s), 1 + 32);  // expect_tx + every producer lane's row vectors
      mbar_init(bar(kBwBarEmpty + s), 1);
    }
    mbar_init(bar(kBwBarS), 1);
    mbar_init(bar(kBwBarDP), 1);
    mbar_init(bar(kBwBarP), kBwdEwThreads);
    mbar_init(bar(kBwBarDS), kBwdEwThreads);
    mbar_init(bar(kBwBarAcc), 1);
    mbar_init(bar(kBwBarDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kBwdMmaWarp) {
    tmem_alloc(smem_addr(tmem_holder), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint64_t limit = p.timeout_ns;

  if (warp >= kBwdProducerWarp) {
    regs_shrink<kBwdOtherRegs>();
    if (warp == kBwdProducerWarp && n_q > 0) {
      // ------------------------------------------------------------ producer
      const bool leader = elect_one_sync();
      if (leader) {
        mbar_arrive_expect_tx(bar(kBwBarRes), 2 * C::kTileBytes);
#pragma unroll
        for (int c = 0; c < C::kDChunks; ++c) {
          tma_load_3d(smem_addr(sK) + c * kBwdRows * 128, &tm_k, bar(kBwBarRes), c * 64, k0, bh);
          tma_load_3d(smem_addr(sV) + c * kBwdRows * 128, &tm_v, bar(kBwBarRes), c * 64, k0, bh);
        }
      }
      __syncwarp();
      int issued = 0;
      for (int n = 0; n < n_q; ++n) {
        const int st = n & 1;
        if (!warp_wait(bar(kBwBarEmpty + st), ((n >> 1) & 1) ^ 1, abort_flag, limit)) break;
        const int q0 = (qt_lo + n) * kBwdRows;
        if (leader) {
          mbar_arrive_expect_tx(bar(kBwBarFull + st), 2 * C::kTileBytes);
#pragma unroll
          for (int c = 0; c < C::kDChunks; ++c) {
            tma_load_3d(smem_addr(sQ(st)) + c * kBwdRows * 128, &tm_q, bar(kBwBarFull + st),
                        c * 64, q0, bh);
            tma_load_3d(smem_addr(sDO(st)) + c * kBwdRows * 128, &tm_do, bar(kBwBarFull + st),
                        c * 64, q0, bh);
          }
        }
        // lse2 = LSE log2(e) and D of the tile's rows; rows past L get
        // lse2 = +inf (P = 0) and D = 0
        float* vec = sVec(st);
#pragma unroll
        for (int r = lane; r < kBwdRows; r += 32) {
          const int q = q0 + r;
          const size_t g = static_cast<size_t>(bh) * p.L + q;
          vec[r] = q < p.L ? p.lse[g] * 1.4426950408889634f : INFINITY;
          vec[kBwdRows + r] = q < p.L ? p.dvec[g] : 0.f;
        }
        mbar_arrive(bar(kBwBarFull + st));
        ++issued;
      }
      // every copy this warp issued must land before the CTA may exit
      drain_wait(bar(kBwBarRes), 0, limit);
      for (int st = 0; st < 2; ++st)
        if (issued > st) drain_wait(bar(kBwBarFull + st), (((issued - 1 - st) >> 1)) & 1, limit);
    } else if (warp == kBwdMmaWarp && n_q > 0) {
      // ------------------------------------------------------------ MMA issuer
      const bool leader = elect_one_sync();
      constexpr uint32_t idesc_s = idesc_bf16_f32(kBwdRows, kBwdRows, false);
      constexpr uint32_t idesc_g = idesc_bf16_f32(kBwdRows, D, true);
      const uint32_t desc_hi = static_cast<uint32_t>(sdesc_sw128(0, 16, 1024) >> 32);
      auto desc = [&](uint32_t lo) -> uint64_t {
        return (static_cast<uint64_t>(desc_hi) << 32) | lo;
      };
      auto kmaj = [&](const uint8_t* t) {
        return static_cast<uint32_t>(sdesc_sw128(smem_addr(t), 16, 1024));
      };
      auto mnmaj = [&](const uint8_t* t) {
        return static_cast<uint32_t>(sdesc_sw128(smem_addr(t), kBwdRows * 128, 1024));
      };
      // K-major operands: K-step k of 16 columns inside 64-column chunks
      auto koff = [](int k) -> uint32_t {
        return static_cast<uint32_t>(((k / 4) * kBwdRows * 128 + (k % 4) * 32) >> 4);
      };
      bool ok = warp_wait(bar(kBwBarRes), 0, abort_flag, limit);
      for (int n = 0; ok && n < n_q; ++n) {
        const int st = n & 1;
        if (!(ok = warp_wait(bar(kBwBarFull + st), (n >> 1) & 1, abort_flag, limit))) break;
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            mma_ss(tmem + C::kColS, desc(kmaj(sK) + koff(k)), desc(kmaj(sQ(st)) + koff(k)),
                   idesc_s, k > 0 ? 1u : 0u);
          mma_commit(bar(kBwBarS));
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            mma_ss(tmem + C::kColDP, desc(kmaj(sV) + koff(k)), desc(kmaj(sDO(st)) + koff(k)),
                   idesc_s, k > 0 ? 1u : 0u);
          mma_commit(bar(kBwBarDP));
        }
        __syncwarp();
        if (!(ok = warp_wait(bar(kBwBarP), n & 1, abort_flag, limit))) break;
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int k = 0; k < kBwdRows / 16; ++k)
            mma_ts(tmem + C::kColAcc0, split_a_col(tmem + C::kColS, k),
                   desc(mnmaj(sDO(st)) + ((k * 16 * 128) >> 4)), idesc_g,
                   (n > 0 || k > 0) ? 1u : 0u);
        }
        __syncwarp();
        if (!(ok = warp_wait(bar(kBwBarDS), n & 1, abort_flag, limit))) break;
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int k = 0; k < kBwdRows / 16; ++k)
            mma_ts(tmem + C::kColAcc1, split_a_col(tmem + C::kColDP, k),
                   desc(mnmaj(sQ(st)) + ((k * 16 * 128) >> 4)), idesc_g,
                   (n > 0 || k > 0) ? 1u : 0u);
          mma_commit(bar(kBwBarEmpty + st));
        }
        __syncwarp();
      }
      if (leader) {
        if (ok) mma_commit(bar(kBwBarAcc));
        mma_commit(bar(kBwBarDrain));
      }
      __syncwarp();
      drain_wait(bar(kBwBarDrain), 0, limit);
    }
  } else {
    // ------------------------------------------------------------ element-wise
    regs_grow<kBwdEwRegs>();
    const int sub = warp % 4, h = warp / 4;  // sub-partition; column half
    const int krow = 32 * sub + lane;        // key row in the tile (= tensor-memory lane)
    const int kglob = k0 + krow;
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * sub) << 16);
    const float cl2 = p.scale_log2;
    bool ok = true;
    for (int n = 0; ok && n < n_q; ++n) {
      const int st = n & 1;
      const int q0 = (qt_lo + n) * kBwdRows;
      const int q_last = min(q0 + kBwdRows - 1, p.L - 1);
      const bool full =
          kv_tile_class(p.L, q0, q_last, kt, p.mask_kind, p.window, kBwdRows) == kTileFull;
      // the stage's row vectors (written by the producer's lanes), then S^T;
      // the stage cannot move on before this thread's dS arrive below
      if (!(ok = warp_wait(bar(kBwBarFull + st), (n >> 1) & 1, abort_flag, limit))) break;
      if (!(ok = warp_wait(bar(kBwBarS), n & 1, abort_flag, limit))) break;
      tc_fence_after();
      uint32_t sr[64];
      bwd_ld64(trow + C::kColS + 64 * h, sr);
      float* s = reinterpret_cast<float*>(sr);
      if (!full) {
        int c_lo, c_hi;
        key_allowed_cols(p.L, kglob, q0 + 64 * h, 64, p.mask_kind, p.window, c_lo, c_hi);
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c < c_lo || c >= c_hi) s[c] = -INFINITY;
      }
      const float* lse2 = sVec(st) + 64 * h;
      const float* dv = sVec(st) + kBwdRows + 64 * h;
      // P^T (fp32, kept for dS) -> bf16 over the first 32 of this warp's columns
#pragma unroll
      for (int c = 0; c < 64; ++c) s[c] = ex2_approx(fmaf(s[c], cl2, -lse2[c]));
      bwd_st_packed(trow + C::kColS + 64 * h, s);
      mbar_arrive(bar(kBwBarP));
      if (!(ok = warp_wait(bar(kBwBarDP), n & 1, abort_flag, limit))) break;
      tc_fence_after();
      uint32_t dr[64];
      bwd_ld64(trow + C::kColDP + 64 * h, dr);
      float* dp = reinterpret_cast<float*>(dr);
#pragma unroll
      for (int c = 0; c < 64; ++c) dp[c] = s[c] * (dp[c] - dv[c]);
      bwd_st_packed(trow + C::kColDP + 64 * h, dp);
      mbar_arrive(bar(kBwBarDS));
    }
    if (ok && n_q > 0) ok = warp_wait(bar(kBwBarAcc), 0, abort_flag, limit);
    if (ok) {
      tc_fence_after();
      const bool row_ok = kglob < p.L;
      const size_t off = (static_cast<size_t>(bh) * p.L + (row_ok ? kglob : 0)) * D + (D / 2) * h;
      if (n_q > 0) {
        bwd_store_acc<D>(trow + C::kColAcc0 + (D / 2) * h, p.dv + off, 1.f, row_ok);
        bwd_store_acc<D>(trow + C::kColAcc1 + (D / 2) * h, p.dk + off, p.scale, row_ok);
      } else if (row_ok) {  // no query attends to these keys: zero gradients
        for (int c = 0; c < D / 2; ++c) p.dv[off + c] = p.dk[off + c] = 0.f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------ dQ
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dq_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_do, const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = smem;
  uint8_t* sDO = smem + C::kTileBytes;
  uint8_t* stage0 = smem + 2 * C::kTileBytes;  // [2] x (K, V)
  uint64_t* bars = reinterpret_cast<uint64_t*>(stage0 + 2 * C::kStageBytes);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + kBwNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  auto sK = [&](int st) { return stage0 + st * C::kStageBytes; };
  auto sV = [&](int st) { return stage0 + st * C::kStageBytes + C::kTileBytes; };

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  auto bar = [&](int i) -> uint32_t { return smem_addr(&bars[i]); };
  // query tiles in descending order: for causal masks the last queries visit
  // the most key tiles, so the longest CTAs start first
  const int qt = p.n_tiles - 1 - static_cast<int>(blockIdx.x / p.BH);
  const int bh = blockIdx.x % p.BH;
  const int q0 = qt * kBwdRows;
  const int q_last = min(q0 + kBwdRows - 1, p.L - 1);
  int lo, hi, full_lo, full_hi;
  kv_tile_range(p.L, q0, q_last, p.mask_kind, p.window, kBwdRows, lo, hi);
  kv_full_range(p.L, q0, q_last, p.mask_kind, p.window, kBwdRows, full_lo, full_hi);
  const int n_k = hi - lo;

  if (threadIdx.x == 0) {
    mbar_init(bar(kBwBarRes), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBwBarFull + s), 1);
      mbar_init(bar(kBwBarEmpty + s), 1);
    }
    mbar_init(bar(kBwBarS), 1);
    mbar_init(bar(kBwBarDP), 1);
    mbar_init(bar(kBwBarP), kBwdEwThreads);
    mbar_init(bar(kBwBarDS), kBwdEwThreads);
    mbar_init(bar(kBwBarAcc), 1);
    mbar_init(bar(kBwBarDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kBwdMmaWarp) {
    tmem_alloc(smem_addr(tmem_holder), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint64_t limit = p.timeout_ns;

  if (warp >= kBwdProducerWarp) {
    regs_shrink<kBwdOtherRegs>();
    if (warp == kBwdProducerWarp && n_k > 0) {
      // ------------------------------------------------------------ producer
      const bool leader = elect_one_sync();
      if (leader) {
        mbar_arrive_expect_tx(bar(kBwBarRes), 2 * C::kTileBytes);
#pragma unroll
        for (int c = 0; c < C::kDChunks; ++c) {
          tma_load_3d(smem_addr(sQ) + c * kBwdRows * 128, &tm_q, bar(kBwBarRes), c * 64, q0, bh);
          tma_load_3d(smem_addr(sDO) + c * kBwdRows * 128, &tm_do, bar(kBwBarRes), c * 64, q0,
                      bh);
        }
      }
      __syncwarp();
      int issued = 0;
      for (int n = 0; n < n_k; ++n) {
        const int st = n & 1;
        if (!warp_wait(bar(kBwBarEmpty + st), ((n >> 1) & 1) ^ 1, abort_flag, limit)) break;
        const int kk0 = (lo + n) * kBwdRows;
        if (leader) {
          mbar_arrive_expect_tx(bar(kBwBarFull + st), 2 * C::kTileBytes);
#pragma unroll
          for (int c = 0; c < C::kDChunks; ++c) {
            tma_load_3d(smem_addr(sK(st)) + c * kBwdRows * 128, &tm_k, bar(kBwBarFull + st),
                        c * 64, kk0, bh);
            tma_load_3d(smem_addr(sV(st)) + c * kBwdRows * 128, &tm_v, bar(kBwBarFull + st),
                        c * 64, kk0, bh);
          }
        }
        __syncwarp();
        ++issued;
      }
      drain_wait(bar(kBwBarRes), 0, limit);
      for (int st = 0; st < 2; ++st)
        if (issued > st) drain_wait(bar(kBwBarFull + st), (((issued - 1 - st) >> 1)) & 1, limit);
    } else if (warp == kBwdMmaWarp && n_k > 0) {
      // ------------------------------------------------------------ MMA issuer
      const bool leader = elect_one_sync();
      constexpr uint32_t idesc_s = idesc_bf16_f32(kBwdRows, kBwdRows, false);
      constexpr uint32_t idesc_g = idesc_bf16_f32(kBwdRows, D, true);
      const uint32_t desc_hi = static_cast<uint32_t>(sdesc_sw128(0, 16, 1024) >> 32);
      auto desc = [&](uint32_t lo_) -> uint64_t {
        return (static_cast<uint64_t>(desc_hi) << 32) | lo_;
      };
      auto kmaj = [&](const uint8_t* t) {
        return static_cast<uint32_t>(sdesc_sw128(smem_addr(t), 16, 1024));
      };
      auto mnmaj = [&](const uint8_t* t) {
        return static_cast<uint32_t>(sdesc_sw128(smem_addr(t), kBwdRows * 128, 1024));
      };
      auto koff = [](int k) -> uint32_t {
        return static_cast<uint32_t>(((k / 4) * kBwdRows * 128 + (k % 4) * 32) >> 4);
      };
      bool ok = warp_wait(bar(kBwBarRes), 0, abort_flag, limit);
      for (int n = 0; ok && n < n_k; ++n) {
        const int st = n & 1;
        if (!(ok = warp_wait(bar(kBwBarFull + st), (n >> 1) & 1, abort_flag, limit))) break;
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            mma_ss(tmem + C::kColS, desc(kmaj(sQ) + koff(k)), desc(kmaj(sK(st)) + koff(k)),
                   idesc_s, k > 0 ? 1u : 0u);
          mma_commit(bar(kBwBarS));
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            mma_ss(tmem + C::kColDP, desc(kmaj(sDO) + koff(k)), desc(kmaj(sV(st)) + koff(k)),
                   idesc_s, k > 0 ? 1u : 0u);
          mma_commit(bar(kBwBarDP));
        }
        __syncwarp();
        if (!(ok = warp_wait(bar(kBwBarDS), n & 1, abort_flag, limit))) break;
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int k = 0; k < kBwdRows / 16; ++k)
            mma_ts(tmem + C::kColAcc0, split_a_col(tmem + C::kColS, k),
                   desc(mnmaj(sK(st)) + ((k * 16 * 128) >> 4)), idesc_g,
                   (n > 0 || k > 0) ? 1u : 0u);
          mma_commit(bar(kBwBarEmpty + st));
        }
        __syncwarp();
      }
      if (leader) {
        if (ok) mma_commit(bar(kBwBarAcc));
        mma_commit(bar(kBwBarDrain));
      }
      __syncwarp();
      drain_wait(bar(kBwBarDrain), 0, limit);
    }
  } else {
    // ------------------------------------------------------------ element-wise
    regs_grow<kBwdEwRegs>();
    const int sub = warp % 4, h = warp / 4;
    const int qrow = 32 * sub + lane;  // query row in the tile (= tensor-memory lane)
    const int qglob = q0 + qrow;
    const bool row_ok = qglob < p.L;
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * sub) << 16);
    const float cl2 = p.scale_log2;
    const size_t g = static_cast<size_t>(bh) * p.L + (row_ok ? qglob : 0);
    // rows past L: P = 0 (lse2 = +inf) and D = 0; they are never stored
    const float lse2 = row_ok ? p.lse[g] * 1.4426950408889634f : INFINITY;
    const float dval = row_ok ? p.dvec[g] : 0.f;
    bool ok = true;
    for (int n = 0; ok && n < n_k; ++n) {
      const int j = lo + n;
      if (!(ok = warp_wait(bar(kBwBarS), n & 1, abort_flag, limit))) break;
      tc_fence_after();
      uint32_t sr[64];
      bwd_ld64(trow + C::kColS + 64 * h, sr);
      float* s = reinterpret_cast<float*>(sr);
      if (!(j >= full_lo && j < full_hi)) {
        int c_lo = 0, c_hi = 0;
        if (row_ok) row_allowed_cols(p.L, qglob, j, p.mask_kind, p.window, kBwdRows, c_lo, c_hi);
        c_lo -= 64 * h;
        c_hi -= 64 * h;
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c < c_lo || c >= c_hi) s[c] = -INFINITY;
      }
#pragma unroll
      for (int c = 0; c < 64; ++c) s[c] = ex2_approx(fmaf(s[c], cl2, -lse2));
      if (!(ok = warp_wait(bar(kBwBarDP), n & 1, abort_flag, limit))) break;
      tc_fence_after();
      uint32_t dr[64];
      bwd_ld64(trow + C::kColDP + 64 * h, dr);
      float* dp = reinterpret_cast<float*>(dr);
#pragma unroll
      for (int c = 0; c < 64; ++c) dp[c] = s[c] * (dp[c] - dval);
      // dS (bf16) over the first 32 of this warp's S columns
      bwd_st_packed(trow + C::kColS + 64 * h, dp);
      mbar_arrive(bar(kBwBarDS));
    }
    if (ok && n_k > 0) ok = warp_wait(bar(kBwBarAcc), 0, abort_flag, limit);
    if (ok) {
      tc_fence_after();
      const size_t off = g * D + (D / 2) * h;
      if (n_k > 0) {
        bwd_store_acc<D>(trow + C::kColAcc0 + (D / 2) * h, p.dq + off, p.scale, row_ok);
      } else if (row_ok) {
        for (int c = 0; c < D / 2; ++c) p.dq[off + c] = 0.f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// One-time set-up per (kernel, device): the shared-memory limit and the
// register check.  kWhich tells the two kernels apart (their function types
// are the same, so the kernel's type alone would share one flag between them).
template <int D, int kWhich, typename Kernel>
int bwd_prepare(Kernel kernel, cudaError_t* err) {
  int device = 0;
  if ((*err = cudaGetDevice(&device)) != cudaSuccess) return ATTN_ERR_CUDA;
  static std::mutex mu;
  static bool done[64] = {};
  std::lock_guard<std::mutex> g(mu);
  if (device < 0 || device >= 64) {
    *err = cudaErrorInvalidDevice;
    return ATTN_ERR_CUDA;
  }
  if (!done[device]) {
    *err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                BwdCfg<D>::kSmemBytes);
    if (*err != cudaSuccess) return ATTN_ERR_CUDA;
    cudaFuncAttributes fa;
    if ((*err = cudaFuncGetAttributes(&fa, kernel)) != cudaSuccess) return ATTN_ERR_CUDA;
    if (fa.numRegs != kBwdLaunchRegs) {  // the register split assumes it
      *err = cudaErrorInvalidConfiguration;
      return ATTN_ERR_CUDA;
    }
    done[device] = true;
  }
  return ATTN_OK;
}

template <int D>
int launch_bwd_sm100_t(const BwdArgs& a, cudaStream_t stream, cudaError_t* err) {
  int st = bwd_prepare<D, 0>(bwd_dkdv_sm100_kernel<D>, err);
  if (st != ATTN_OK) return st;
  if ((st = bwd_prepare<D, 1>(bwd_dq_sm100_kernel<D>, err)) != ATTN_OK) return st;
  const int BH = a.B * a.H;
  const long long dense[3] = {D, static_cast<long long>(a.L) * D,
                              static_cast<long long>(a.H) * a.L * D};
  CUtensorMap tq, tk, tv, tdo;
  if (!make_map(&tq, a.q, a.B, a.H, a.L, D, dense, kBwdRows, false, err) ||
      !make_map(&tk, a.k, a.B, a.H, a.L, D, dense, kBwdRows, false, err) ||
      !make_map(&tv, a.v, a.B, a.H, a.L, D, dense, kBwdRows, false, err) ||
      !make_map(&tdo, a.dout, a.B, a.H, a.L, D, dense, kBwdRows, false, err))
    return ATTN_ERR_CUDA;
  BwdParams p;
  p.lse = a.lse;
  p.dvec = a.D;
  p.dq = a.dq;
  p.dk = a.dk;
  p.dv = a.dv;
  p.BH = BH;
  p.L = a.L;
  p.n_tiles = (a.L + kBwdRows - 1) / kBwdRows;
  p.mask_kind = a.mask_kind;
  p.window = a.window;
  p.scale = a.scale;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.timeout_ns = a.timeout_ns;
  const long long ctas = static_cast<long long>(p.n_tiles) * BH;
  if (ctas > 0x7fffffffLL) {
    *err = cudaErrorInvalidValue;
    return ATTN_ERR_UNSUPPORTED;
  }
  bwd_dkdv_sm100_kernel<D><<<static_cast<unsigned>(ctas), kBwdThreads, BwdCfg<D>::kSmemBytes,
                             stream>>>(tq, tk, tv, tdo, p);
  if ((*err = cudaGetLastError()) != cudaSuccess) return ATTN_ERR_CUDA;
  bwd_dq_sm100_kernel<D><<<static_cast<unsigned>(ctas), kBwdThreads, BwdCfg<D>::kSmemBytes,
                           stream>>>(tq, tk, tv, tdo, p);
  *err = cudaGetLastError();
  return *err == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

int launch_bwd_sm100(const BwdArgs& a, cudaStream_t stream, cudaError_t* err) {
  *err = cudaSuccess;
  if (!a.bf16) return ATTN_ERR_UNSUPPORTED;
  if (a.d == 128) return launch_bwd_sm100_t<128>(a, stream, err);
  if (a.d == 64) return launch_bwd_sm100_t<64>(a, stream, err);
  return ATTN_ERR_UNSUPPORTED;
}

}  // namespace ebh
