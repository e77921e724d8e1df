// attn_sm100.cu -- exact blockwise attention forward, bf16 in, fp32
// accumulate, on the sm_100a tensor cores.
//
// The method is the fused kernel of "Mosaic multi-GPU sequence-sharded
// attention" (kwkr.cn), section 3.2: keep K/V tiles in shared memory, fuse the
// softmax with the two products, carry a running max and sum across key tiles
// and divide by the sum at the end.  That sketch never updates its max and
// never rescales the partial output; here the max is carried in log2 units and
// the output is rescaled whenever the max grows past a threshold, which makes
// the result exact (both the partial output and the sum are taken against the
// same max, so the final division cancels it).  Masked scores are set to -inf
// before the softmax, as in "Transformer multi-head attention, 8-head parallel
// computation" (lshu.cn), section 2.2; key tiles with no allowed pair are
// skipped outright (O(L w) work for the band mask of "Attention optimisation
// strategies and practice for long-sequence inference", section 2.1).
//
// Mapping onto Blackwell.  One persistent CTA per SM walks a static list of
// work units; a unit is 256 query rows of one (batch, head), split into two
// 128-row Q tiles that share the stream of K/V tiles.  Warp roles:
//   warps 0-3   softmax for Q tile 0 (one thread per query row)
//   warps 4-7   softmax for Q tile 1
//   warp  8     TMA producer: Q tiles once per unit, then K_j, V_j into a ring
//   warp  9     MMA issuer: S_t = Q_t K_j^T and O_t += P_t V_j (tcgen05, fp32
//               accumulators in tensor memory); owns the tensor-memory block
//   warps 10-11 idle
// Tensor memory (columns): S_0 | S_1 | O_0 | O_1.  P_t (bf16, two per column)
// is written over the first half of S_t and fed to the P.V product straight
// from tensor memory.  The MMA warp interleaves the two Q tiles,
//   S_0(j), P_1(j-1).V_(j-1), S_1(j), P_0(j).V_j, S_0(j+1), ...
// so each softmax group works while the tensor core runs the other tile's
// products.  Because tcgen05 MMAs complete in issue order, "S_t(j) done"
// also means "P_t(j-1).V done", which lets the softmax thread rescale its
// own row of O_t without any further barrier.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "attn.h"
#include "kernels.h"
#include "sm100_ptx.cuh"
#include "tiles.h"

namespace ebh {
namespace {

constexpr int kBM = 128;          // query rows per Q tile (= tensor-memory lanes)
constexpr int kNQ = 2;            // Q tiles per work unit
constexpr int kUnitRows = kBM * kNQ;
constexpr int kThreads = 384;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kLaunchRegs = 168;   // 65536 / 384 rounded down to a multiple of 8
constexpr int kSoftmaxRegs = 208;
constexpr int kOtherRegs = 80;
static_assert(kSoftmaxRegs * 256 + kOtherRegs * 128 <= kLaunchRegs * kThreads,
              "register split exceeds the launch allocation");
// Share of the exponentials computed on the FMA pipe (polynomial) instead of
// the MUFU pipe, on tiles without masked elements: one pair in kPolyEvery
// (0 = none).
#ifndef EBH_POLY_EVERY
#define EBH_POLY_EVERY 0
#endif
constexpr int kPolyEvery = EBH_POLY_EVERY;
// Lazy rescale: keep the stale max until the row max exceeds it by more than
// 2^8 (probabilities then stay <= 256, far inside fp32/bf16 range).
constexpr float kRescaleThreshold = 8.0f;
// Compute a tile's exponentials against the stale max before its row max is
// known (redo the tile when the max outgrew the threshold).  Needs the whole
// score row live during the exponentials.
#ifndef EBH_SPECULATE
#define EBH_SPECULATE 0
#endif
constexpr bool kSpeculate = EBH_SPECULATE;
// Row-max reduction: independent chains of three-input maxima (0 = a tree).
#ifndef EBH_MAX_CHAINS
#define EBH_MAX_CHAINS 4
#endif
constexpr int kMaxChains = EBH_MAX_CHAINS;

// Pipeline trace for profiling builds (-DEBH_PIPELINE_TRACE): lane 0 of each
// warp of CTA 0 appends (event << 56 | key block << 40 | clock64) records to
// g_pipeline_trace[warp]; attn_pipeline_trace_read() copies them out.
enum : int {
  kEvSWait = 1, kEvSReady = 2, kEvSLoaded = 3, kEvMaxDone = 4, kEvPWritten = 5, kEvMasked = 8,
  kEvEpilogue = 6, kEvEpilogueDone = 7,
  kEvKWait = 10, kEvKReady = 11, kEvVWait = 16, kEvVReady = 17,
  kEvPWait = 13, kEvPReady = 14  // + 10 * Q tile
};
#ifdef EBH_PIPELINE_TRACE
constexpr int kTraceLen = 8192;
__device__ unsigned long long g_pipeline_trace[16][kTraceLen];
#define EBH_TRACE_COUNTER int tr_n = 0
#define EBH_TRACE(ev, jj)                                                               \
  do {                                                                                  \
    if (blockIdx.x == 0 && (threadIdx.x % 32) == 0 && tr_n < kTraceLen)                 \
      g_pipeline_trace[threadIdx.x / 32][tr_n++] =                                      \
          ((unsigned long long)(ev) << 56) | ((unsigned long long)((jj)&0xFFFF) << 40) | \
          (clock64() & 0xFFFFFFFFFFull);                                                \
  } while (0)
#else
#define EBH_TRACE_COUNTER \
  do {                    \
  } while (0)
#define EBH_TRACE(ev, jj) \
  do {                    \
  } while (0)
#endif

template <int D, int BN>
struct Cfg {
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(BN == 64 || BN == 128, "key block");
  static constexpr int kDChunks = D / 64;            // 128-byte (64 x bf16) column chunks
  static constexpr int kQTileBytes = kBM * D * 2;
  static constexpr int kKVTileBytes = BN * D * 2;
  static constexpr int kStages = kKVTileBytes >= 32768 ? 4 : 8;
  static constexpr int kSmemQ = kNQ * kQTileBytes;
  static constexpr int kSmemKV = kStages * kKVTileBytes;
  // barrier indices
  static constexpr int kBarQFull = 0;                  // [kNQ]
  static constexpr int kBarQEmpty = kBarQFull + kNQ;   // [kNQ]
  static constexpr int kBarKVFull = kBarQEmpty + kNQ;  // [kStages]
  static constexpr int kBarKVEmpty = kBarKVFull + kStages;
  static constexpr int kBarSFull = kBarKVEmpty + kStages;  // [kNQ]
  static constexpr int kBarPFull = kBarSFull + kNQ;        // [kNQ]
  static constexpr int kBarOFull = kBarPFull + kNQ;        // [kNQ]
  static constexpr int kBarOEmpty = kBarOFull + kNQ;       // [kNQ]
  static constexpr int kBarDrain = kBarOEmpty + kNQ;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kSmemBytes = 1024 + kSmemQ + kSmemKV + 8 * kNumBars + 16;
  static constexpr int kTmemNeed = 2 * BN + 2 * D;
  static constexpr int kTmemCols = kTmemNeed <= 256 ? 256 : 512;
  static constexpr int kColS = 0;            // + t * BN
  static constexpr int kColO = 2 * BN;       // + t * D
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

struct Params {
  void* out;
  float* lse;
  int BH, L;
  int mask_kind, window;
  float scale_log2;  // scale * log2(e)
  int num_units, nqp;
  uint64_t timeout_ns;
};

struct Unit {
  int bh, qp;
  bool valid[kNQ];
  int q_first[kNQ], q_last[kNQ], lo[kNQ], hi[kNQ];
  int ulo, uhi;  // union of the two key-block ranges
};

template <int BN>
__device__ __forceinline__ Unit decode_unit(int u, const Params& p) {
  Unit w;
  if (p.mask_kind == kMaskCausal) {
    // longest units first: causal work grows with the query position
    w.qp = p.nqp - 1 - u / p.BH;
    w.bh = u % p.BH;
  } else {
    w.bh = u / p.nqp;
    w.qp = u % p.nqp;
  }
  w.ulo = 0x7fffffff;
  w.uhi = 0;
#pragma unroll
  for (int t = 0; t < kNQ; ++t) {
    w.q_first[t] = w.qp * kUnitRows + t * kBM;
    w.valid[t] = w.q_first[t] < p.L;
    w.q_last[t] = min(w.q_first[t] + kBM - 1, p.L - 1);
    w.lo[t] = w.hi[t] = 0;
    if (w.valid[t]) {
      kv_tile_range(p.L, w.q_first[t], w.q_last[t], p.mask_kind, p.window, BN, w.lo[t], w.hi[t]);
      w.ulo = min(w.ulo, w.lo[t]);
      w.uhi = max(w.uhi, w.hi[t]);
    }
  }
  if (w.uhi <= w.ulo) w.ulo = w.uhi = 0;
  return w;
}

// One Q tile of unit u, decoded on its own (no per-tile arrays, so the
// softmax threads, whose tile index is a run-time value, keep it in registers).
struct TileWork {
  int bh;
  bool valid;
  int q_first, q_last, lo, hi;
};

template <int BN>
__device__ __forceinline__ TileWork decode_tile(int u, int t, const Params& p) {
  TileWork w;
  int qp;
  if (p.mask_kind == kMaskCausal) {
    qp = p.nqp - 1 - u / p.BH;
    w.bh = u % p.BH;
  } else {
    w.bh = u / p.nqp;
    qp = u % p.nqp;
  }
  w.q_first = qp * kUnitRows + t * kBM;
  w.valid = w.q_first < p.L;
  w.q_last = min(w.q_first + kBM - 1, p.L - 1);
  w.lo = w.hi = 0;
  if (w.valid) kv_tile_range(p.L, w.q_first, w.q_last, p.mask_kind, p.window, BN, w.lo, w.hi);
  return w;
}

__device__ __forceinline__ bool in_range(const Unit& w, int t, int j) {
  return w.valid[t] && j >= w.lo[t] && j < w.hi[t];
}

// Wait for all lanes of a warp; the outcome is made warp-uniform so that the
// warp-collective tensor-memory instructions that follow run on all lanes or
// none.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          uint64_t limit) {
  bool ok = wait_bounded(bar, parity, abort, limit);
  return __all_sync(0xffffffffu, ok);
}

// Wait used only while tearing down: ignores the abort flag, never raises it.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t limit) {
  const uint64_t t0 = globaltimer_ns();
#pragma unroll 1
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit) {
      atomicOr(&g_attn_status_word, kStatusTimeout);
      return;
    }
  }
}

// O_t row *= alpha for this warp's 32 rows (tensor memory round trip).  The
// caller guarantees no MMA is writing O_t (its previous P.V product was issued
// before the S_t product the caller has waited for, and they complete in order).
template <int D>
__device__ __forceinline__ void rescale_o_row(uint32_t tO, float alpha) {
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    uint32_t o[32];
    tmem_ld32(tO + 32 * c, o);
    tmem_wait_ld();
    reg_fence32(o);
#pragma unroll
    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
    tmem_st32(tO + 32 * c, o);
  }
}

// Max of n values by a tree of three-input maxima (depth log3 n).
template <int N>
struct TreeMax {
  static __device__ __forceinline__ float run(float* v) {
    constexpr int M = (N + 2) / 3;
#pragma unroll
    for (int i = 0; i < M; ++i) {
      if (3 * i + 2 < N) v[i] = max3(v[3 * i], v[3 * i + 1], v[3 * i + 2]);
      else if (3 * i + 1 < N) v[i] = fmaxf(v[3 * i], v[3 * i + 1]);
      else v[i] = v[3 * i];
    }
    return TreeMax<M>::run(v);
  }
};
template <>
struct TreeMax<1> {
  static __device__ __forceinline__ float run(float* v) { return v[0]; }
};

// Max of one row of a score tile: kMaxChains independent chains of
// three-input maxima, or (kMaxChains == 0) a tree.
template <int BN>
__device__ __forceinline__ float row_max(const float* s) {
  if constexpr (kMaxChains == 0) {
    constexpr int M = (BN + 2) / 3;
    float v[M];
#pragma unroll
    for (int i = 0; i < M; ++i) {
      if (3 * i + 2 < BN) v[i] = max3(s[3 * i], s[3 * i + 1], s[3 * i + 2]);
      else if (3 * i + 1 < BN) v[i] = fmaxf(s[3 * i], s[3 * i + 1]);
      else v[i] = s[3 * i];
    }
    return TreeMax<M>::run(v);
  } else {
    constexpr int K = kMaxChains;
    float m[K];
#pragma unroll
    for (int i = 0; i < K; ++i) m[i] = fmaxf(s[i], s[i + K]);
#pragma unroll
    for (int c = 2 * K; c < BN; c += 2 * K) {
#pragma unroll
      for (int i = 0; i < K; ++i) m[i] = max3(m[i], s[c + i], s[c + K + i]);
    }
    return TreeMax<K>::run(m);
  }
}

// p_c = 2^(s_c * cl2 - msub) for one row of a score tile, written to tensor
// memory as packed bf16 over the first half of the tile's S columns (those
// scores are already in registers), 32 keys at a time.  l accumulates the
// probabilities, lr the bf16-rounded probabilities the P.V product will use.
// kPoly: compute one pair in kPolyEvery on the FMA pipe (tiles without masked
// elements only: the polynomial has no -inf handling).
template <int BN, bool kPoly>
__device__ __forceinline__ void write_probabilities(const float* s, float cl2, float msub,
                                                    uint32_t tS, float& l, float& lr) {
  float la = 0.f, lb = 0.f, lc = 0.f, ld = 0.f;
  float ra = 0.f, rb = 0.f, rc = 0.f, rd = 0.f;
#pragma unroll
  for (int cc = 0; cc < BN / 32; ++cc) {
    uint32_t pk[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int e = 32 * cc + 2 * c;
      float x0, x1, p0, p1;
      fma2(x0, x1, s[e], s[e + 1], cl2, cl2, -msub, -msub);
      bool poly = false;
      if constexpr (kPoly) poly = (c % (kPolyEvery > 0 ? kPolyEvery : 1)) == kPolyEvery - 1;
      if (poly) {
        exp2_poly2(x0, x1, p0, p1);
      } else {
        p0 = ex2_approx(x0);
        p1 = ex2_approx(x1);
      }
      pk[c] = pack_bf16x2(p0, p1);
      if (c & 1) {
        add2(lc, ld, lc, ld, p0, p1);
        acc_bf16x2(rc, rd, pk[c]);
      } else {
        add2(la, lb, la, lb, p0, p1);
        acc_bf16x2(ra, rb, pk[c]);
      }
    }
    tmem_st16(tS + 16 * cc, pk);
  }
  l += (la + lb) + (lc + ld);
  lr += (ra + rb) + (rc + rd);
}

template <int D, int BN>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using C = Cfg<D, BN>;
  extern __shared__ uint8_t smem_raw[];
  // 128-byte-swizzled tiles need 1024-byte-aligned shared-memory addresses
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::kSmemQ;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kSmemQ + C::kSmemKV);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  auto bar = [&](int i) -> uint32_t { return smem_addr(&bars[i]); };

  if (threadIdx.x == 0) {
    for (int t = 0; t < kNQ; ++t) {
      mbar_init(bar(C::kBarQFull + t), 1);
      mbar_init(bar(C::kBarQEmpty + t), 1);
      mbar_init(bar(C::kBarSFull + t), 1);
      mbar_init(bar(C::kBarPFull + t), kBM);
      mbar_init(bar(C::kBarOFull + t), 1);
      mbar_init(bar(C::kBarOEmpty + t), kBM);
    }
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(C::kBarKVFull + s), 1);
      mbar_init(bar(C::kBarKVEmpty + s), 1);
    }
    mbar_init(bar(C::kBarDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_addr(tmem_holder), C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint64_t limit = p.timeout_ns;

  // Registers: the softmax warpgroups hold a 128-wide score row per thread;
  // the producer / MMA warpgroup needs few.  kSoftmaxRegs * 256 +
  // kOtherRegs * 128 must not exceed the launch's kLaunchRegs * 384 (checked
  // on the host before launch), or the grow would wait forever.  Each role
  // runs inside the branch that set its register count, so the compiler
  // allocates each role's code under its own limit.
  if (warp >= 8) {
    regs_shrink<kOtherRegs>();
    if (warp == kProducerWarp) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        int kv_it = 0;
        int q_cnt[kNQ] = {0, 0};
        bool ok = true;
        for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x) {
          const Unit w = decode_unit<BN>(u, p);
          auto load_q = [&](int t) -> bool {
            if (!w.valid[t]) return true;
            if (!wait_bounded(bar(C::kBarQEmpty + t), (q_cnt[t] & 1) ^ 1, abort_flag, limit))
              return false;
            mbar_arrive_expect_tx(bar(C::kBarQFull + t), C::kQTileBytes);
            const uint32_t dst = smem_addr(sQ + t * C::kQTileBytes);
  #pragma unroll
            for (int c = 0; c < C::kDChunks; ++c)
              tma_load_3d(dst + c * kBM * 128, &tm_q, bar(C::kBarQFull + t), c * 64, w.q_first[t],
                          w.bh);
            ++q_cnt[t];
            return true;
          };
          ok = load_q(0) && load_q(1);
          for (int j = w.ulo; ok && j < w.uhi; ++j) {
  #pragma unroll 1
            for (int which = 0; which < 2; ++which) {
              const int s = kv_it % C::kStages;
              ok = wait_bounded(bar(C::kBarKVEmpty + s), ((kv_it / C::kStages) & 1) ^ 1, abort_flag,
                                limit);
              if (!ok) break;
              mbar_arrive_expect_tx(bar(C::kBarKVFull + s), C::kKVTileBytes);
              const uint32_t dst = smem_addr(sKV + s * C::kKVTileBytes);
              const CUtensorMap* map = which == 0 ? &tm_k : &tm_v;
  #pragma unroll
              for (int c = 0; c < C::kDChunks; ++c)
                tma_load_3d(dst + c * BN * 128, map, bar(C::kBarKVFull + s), c * 64, j * BN, w.bh);
              ++kv_it;
            }
          }
        }
        // Every load this thread issued must land before the CTA may exit.
        for (int s = 0; s < C::kStages; ++s) {
          if (kv_it > s) {
            const int last = s + C::kStages * ((kv_it - 1 - s) / C::kStages);
            drain_wait(bar(C::kBarKVFull + s), (last / C::kStages) & 1, limit);
          }
        }
        for (int t = 0; t < kNQ; ++t)
          if (q_cnt[t] > 0) drain_wait(bar(C::kBarQFull + t), (q_cnt[t] - 1) & 1, limit);
      }
    } else if (warp == kMmaWarp) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        constexpr uint32_t idesc_s = idesc_bf16_f32(kBM, BN, false);
        constexpr uint32_t idesc_o = idesc_bf16_f32(kBM, D, true);
        int kv_it = 0;
        int q_cnt[kNQ] = {0, 0}, p_cnt[kNQ] = {0, 0}, o_cnt[kNQ] = {0, 0};
        bool ok = true;
        EBH_TRACE_COUNTER;

        auto issue_s = [&](int t, int kst) {
          const uint32_t qa = smem_addr(sQ + t * C::kQTileBytes);
          const uint32_t kb = smem_addr(sKV + kst * C::kKVTileBytes);
  #pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint64_t a = sdesc_sw128(qa + (k / 4) * kBM * 128 + (k % 4) * 32, 16, 1024);
            const uint64_t b = sdesc_sw128(kb + (k / 4) * BN * 128 + (k % 4) * 32, 16, 1024);
            mma_ss(tmem + C::kColS + t * BN, a, b, idesc_s, k > 0 ? 1u : 0u);
          }
        };
        auto issue_pv = [&](int t, int vst, bool first) -> bool {
          EBH_TRACE(kEvPWait + 10 * t, 0);
          if (!wait_bounded(bar(C::kBarPFull + t), p_cnt[t] & 1, abort_flag, limit)) return false;
          EBH_TRACE(kEvPReady + 10 * t, 0);
          ++p_cnt[t];
          if (first &&
              !wait_bounded(bar(C::kBarOEmpty + t), (o_cnt[t] & 1) ^ 1, abort_flag, limit))
            return false;
          tc_fence_after();
          const uint32_t vb = smem_addr(sKV + vst * C::kKVTileBytes);
  #pragma unroll
          for (int k = 0; k < BN / 16; ++k) {
            const uint64_t b = sdesc_sw128(vb + k * 16 * 128, BN * 128, 1024);
            mma_ts(tmem + C::kColO + t * D, tmem + C::kColS + t * BN + k * 8, b, idesc_o,
                   (first && k == 0) ? 0u : 1u);
          }
          return true;
        };

        for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x) {
          const Unit w = decode_unit<BN>(u, p);
          int pend_v = -1;  // ring stage of V_(j-1) still owed a P_1 . V product
          for (int j = w.ulo; ok && j < w.uhi; ++j) {
            const int kst = kv_it % C::kStages;
            const uint32_t kph = (kv_it / C::kStages) & 1;
            ++kv_it;
            const int vst = kv_it % C::kStages;
            const uint32_t vph = (kv_it / C::kStages) & 1;
            ++kv_it;
            EBH_TRACE(kEvKWait, j);
            if (!(ok = wait_bounded(bar(C::kBarKVFull + kst), kph, abort_flag, limit))) break;
            EBH_TRACE(kEvKReady, j);
            const bool in0 = in_range(w, 0, j), in1 = in_range(w, 1, j);
            if (in0) {
              if (j == w.lo[0] &&
                  !(ok = wait_bounded(bar(C::kBarQFull + 0), q_cnt[0] & 1, abort_flag, limit)))
                break;
              tc_fence_after();
              issue_s(0, kst);
              mma_commit(bar(C::kBarSFull + 0));
              if (j == w.hi[0] - 1) mma_commit(bar(C::kBarQEmpty + 0));
            }
            if (pend_v >= 0) {
              if (!(ok = issue_pv(1, pend_v, j - 1 == w.lo[1]))) break;
              mma_commit(bar(C::kBarKVEmpty + pend_v));
              if (j - 1 == w.hi[1] - 1) mma_commit(bar(C::kBarOFull + 1));
              pend_v = -1;
            }
            if (in1) {
              if (j == w.lo[1] &&
                  !(ok = wait_bounded(bar(C::kBarQFull + 1), q_cnt[1] & 1, abort_flag, limit)))
                break;
              tc_fence_after();
              issue_s(1, kst);
              mma_commit(bar(C::kBarSFull + 1));
              if (j == w.hi[1] - 1) mma_commit(bar(C::kBarQEmpty + 1));
            }
            mma_commit(bar(C::kBarKVEmpty + kst));  // K_j no longer needed
            EBH_TRACE(kEvVWait, j);
            if (!(ok = wait_bounded(bar(C::kBarKVFull + vst), vph, abort_flag, limit))) break;
            EBH_TRACE(kEvVReady, j);
            if (in0) {
              if (!(ok = issue_pv(0, vst, j == w.lo[0]))) break;
              if (j == w.hi[0] - 1) mma_commit(bar(C::kBarOFull + 0));
            }
            if (in1) {
              pend_v = vst;
            } else {
              mma_commit(bar(C::kBarKVEmpty + vst));
            }
          }
          if (ok && pend_v >= 0) {
            const int j = w.uhi;
            if ((ok = issue_pv(1, pend_v, j - 1 == w.lo[1]))) {
              mma_commit(bar(C::kBarKVEmpty + pend_v));
              if (j - 1 == w.hi[1] - 1) mma_commit(bar(C::kBarOFull + 1));
            }
          }
          if (w.valid[0]) {
            ++q_cnt[0];
            ++o_cnt[0];
          }
          if (w.valid[1]) {
            ++q_cnt[1];
            ++o_cnt[1];
          }
        }
        // No MMA may still be writing tensor memory when it is freed.
        mma_commit(bar(C::kBarDrain));
        drain_wait(bar(C::kBarDrain), 0, limit);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    regs_grow<kSoftmaxRegs>();
    const int t = warp / 4;
    const int wq = warp % 4;                 // this warp's 32-lane slice of tensor memory
    const int r = threadIdx.x % kBM;         // query row within the Q tile
    const uint32_t lane_base = static_cast<uint32_t>(32 * wq) << 16;
    const uint32_t tS = tmem + lane_base + C::kColS + t * BN;
    const uint32_t tO = tmem + lane_base + C::kColO + t * D;
    const float cl2 = p.scale_log2;
    int s_cnt = 0, o_cnt = 0;
    bool ok = true;
    EBH_TRACE_COUNTER;

    for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x) {
      const TileWork w = decode_tile<BN>(u, t, p);
      if (!w.valid) continue;
      const int row = w.q_first + r;
      float m_used = -INFINITY;  // running max, log2 units
      float l = 0.f;             // running sum of the probabilities against m_used
      float lr = 0.f;            // the same sum over the bf16-rounded probabilities

      for (int j = w.lo; j < w.hi; ++j) {
        EBH_TRACE(kEvSWait, j);
        if (!(ok = warp_wait(bar(C::kBarSFull + t), s_cnt & 1, abort_flag, limit))) break;
        EBH_TRACE(kEvSReady, j);
        ++s_cnt;
        tc_fence_after();
        uint32_t sr[BN];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) tmem_ld32(tS + 32 * c, sr + 32 * c);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) reg_fence32(sr + 32 * c);
        float* s = reinterpret_cast<float*>(sr);
        EBH_TRACE(kEvSLoaded, j);

        const bool full =
            kv_tile_class(p.L, w.q_first, w.q_last, j, p.mask_kind, p.window, BN) == kTileFull;
        if (!full) {
          int c_lo, c_hi;
          row_allowed_cols(p.L, row, j, p.mask_kind, p.window, BN, c_lo, c_hi);
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c < c_lo || c >= c_hi) s[c] = -INFINITY;
        }
        EBH_TRACE(kEvMasked, j);
        const float m_tile = row_max<BN>(s) * cl2;
        if (!kSpeculate || m_used == -INFINITY) {
          float alpha = 1.f;
          bool rescale = false;
          if (m_used == -INFINITY) {
            // nothing accumulated for this row yet (l == 0 and its O row is 0)
            m_used = m_tile;
          } else if (m_tile > m_used + kRescaleThreshold) {
            alpha = ex2_approx(m_used - m_tile);
            l *= alpha;
            lr *= alpha;
            m_used = m_tile;
            rescale = true;
          }
          if (__any_sync(0xffffffffu, rescale)) rescale_o_row<D>(tO, alpha);
          const float msub = m_used == -INFINITY ? 0.f : m_used;
          EBH_TRACE(kEvMaxDone, j);
          if (full) {
            write_probabilities<BN, (kPolyEvery > 0)>(s, cl2, msub, tS, l, lr);
          } else {
            write_probabilities<BN, false>(s, cl2, msub, tS, l, lr);
          }
        } else {
          // Speculate that the stale reference m_used still holds (the tile
          // max exceeds it by at most the threshold), so the exponentials do
          // not wait for the max; if it does not hold for some row, redo the
          // tile against the new max and rescale that row of O.
          const float l0 = l, lr0 = lr;
          EBH_TRACE(kEvMaxDone, j);
          if (full) {
            write_probabilities<BN, (kPolyEvery > 0)>(s, cl2, m_used, tS, l, lr);
          } else {
            write_probabilities<BN, false>(s, cl2, m_used, tS, l, lr);
          }
          const bool redo = m_tile > m_used + kRescaleThreshold;
          if (__any_sync(0xffffffffu, redo)) {
            float alpha = 1.f;
            if (redo) {
              alpha = ex2_approx(m_used - m_tile);
              m_used = m_tile;
            }
            l = l0 * alpha;
            lr = lr0 * alpha;
            rescale_o_row<D>(tO, alpha);
            write_probabilities<BN, false>(s, cl2, m_used, tS, l, lr);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        EBH_TRACE(kEvPWritten, j);
        mbar_arrive(bar(C::kBarPFull + t));
      }
      if (!ok) break;

      // ---- epilogue: O / l -> bf16, LSE = ln 2 * (m + log2 l)
      EBH_TRACE(kEvEpilogue, 0);
      if (!(ok = warp_wait(bar(C::kBarOFull + t), o_cnt & 1, abort_flag, limit))) break;
      ++o_cnt;
      tc_fence_after();
      // O is divided by the sum of exactly the (bf16) weights that multiplied
      // V, so the weights sum to one; LSE uses the unrounded sum.
      const float inv_l = lr > 0.f ? 1.f / lr : 0.f;
      const bool row_ok = row < p.L;
      const size_t row_off = (static_cast<size_t>(w.bh) * p.L + (row_ok ? row : 0)) * D;
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + row_off);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c, o);
        tmem_wait_ld();
        reg_fence32(o);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l,
                              __uint_as_float(o[2 * i + 1]) * inv_l);
        if (row_ok) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[c * 4 + i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      if (row_ok && p.lse != nullptr) {
        const float lse = l > 0.f ? (m_used + log2f(l)) * 0.69314718055994531f : -INFINITY;
        p.lse[static_cast<size_t>(w.bh) * p.L + row] = lse;
      }
      tc_fence_before();
      EBH_TRACE(kEvEpilogueDone, 0);
      mbar_arrive(bar(C::kBarOEmpty + t));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Self test of the bounded wait: one thread waits on a barrier nobody arrives on.
__global__ void selftest_wait_timeout_kernel(uint64_t limit_ns) {
  __shared__ uint64_t b;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&b), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) wait_bounded(smem_addr(&b), 0, &abort_flag, limit_ns);
  __syncthreads();
}

// ---------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn(cudaError_t* err) {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  static cudaError_t status = cudaSuccess;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    status = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q);
    if (status == cudaSuccess && q != cudaDriverEntryPointSuccess) status = cudaErrorNotSupported;
    fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  *err = status;
  return status == cudaSuccess ? fn : nullptr;
}

// [BH, L, D] bf16 tensor, boxes of `rows` x 64 columns, 128-byte swizzle;
// rows past L read as zero.
bool make_map(CUtensorMap* map, const void* base, int BH, int L, int D, int rows,
              cudaError_t* err) {
  EncodeTiledFn fn = encode_fn(err);
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)L, (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)L * D * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    *err = cudaErrorInvalidValue;
    return false;
  }
  return true;
}

int sm_count(int device, cudaError_t* err) {
  static std::mutex mu;
  static int cache[64] = {0};
  std::lock_guard<std::mutex> g(mu);
  if (device < 0 || device >= 64) {
    *err = cudaErrorInvalidDevice;
    return 0;
  }
  if (cache[device] == 0) {
    int n = 0;
    *err = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device);
    if (*err != cudaSuccess) return 0;
    cache[device] = n;
  }
  return cache[device];
}

template <int D, int BN>
int launch_t(const FwdArgs& a, cudaStream_t stream, cudaError_t* err) {
  using C = Cfg<D, BN>;
  auto kernel = attn_fwd_sm100_kernel<D, BN>;
  int device = 0;
  if ((*err = cudaGetDevice(&device)) != cudaSuccess) return ATTN_ERR_CUDA;
  {
    static std::mutex mu;
    static bool attr_set[64] = {false};
    std::lock_guard<std::mutex> g(mu);
    if (device >= 64) {
      *err = cudaErrorInvalidDevice;
      return ATTN_ERR_CUDA;
    }
    if (!attr_set[device]) {
      *err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  C::kSmemBytes);
      if (*err != cudaSuccess) return ATTN_ERR_CUDA;
      // The in-kernel register split assumes exactly kLaunchRegs per thread
      // at launch; refuse to launch a build where that does not hold.
      cudaFuncAttributes fa;
      if ((*err = cudaFuncGetAttributes(&fa, kernel)) != cudaSuccess) return ATTN_ERR_CUDA;
      if (fa.numRegs != kLaunchRegs) {
        *err = cudaErrorInvalidConfiguration;
        return ATTN_ERR_CUDA;
      }
      attr_set[device] = true;
    }
  }
  const int nsm = sm_count(device, err);
  if (nsm <= 0) return ATTN_ERR_CUDA;

  const int BH = a.B * a.H;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, a.q, BH, a.L, D, kBM, err)) return ATTN_ERR_CUDA;
  if (!make_map(&tk, a.k, BH, a.L, D, BN, err)) return ATTN_ERR_CUDA;
  if (!make_map(&tv, a.v, BH, a.L, D, BN, err)) return ATTN_ERR_CUDA;

  Params p;
  p.out = a.out;
  p.lse = a.lse;
  p.BH = BH;
  p.L = a.L;
  p.mask_kind = a.mask_kind;
  p.window = a.window;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.nqp = (a.L + kUnitRows - 1) / kUnitRows;
  const long long units = static_cast<long long>(BH) * p.nqp;
  if (units > 0x7fffffffLL) {
    *err = cudaErrorInvalidValue;
    return ATTN_ERR_UNSUPPORTED;
  }
  p.num_units = static_cast<int>(units);
  p.timeout_ns = a.timeout_ns;
  const int grid = p.num_units < nsm ? p.num_units : nsm;
  kernel<<<grid, kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, p);
  *err = cudaGetLastError();
  return *err == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

int launch_fwd_bf16_sm100(const FwdArgs& a, cudaStream_t stream, cudaError_t* err) {
  *err = cudaSuccess;
  if (a.d == 128 && a.block_n == 128) return launch_t<128, 128>(a, stream, err);
  if (a.d == 128 && a.block_n == 64) return launch_t<128, 64>(a, stream, err);
  if (a.d == 64 && a.block_n == 128) return launch_t<64, 128>(a, stream, err);
  if (a.d == 64 && a.block_n == 64) return launch_t<64, 64>(a, stream, err);
  return ATTN_ERR_UNSUPPORTED;
}

int launch_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t stream, cudaError_t* err) {
  selftest_wait_timeout_kernel<<<1, 32, 0, stream>>>(limit_ns);
  *err = cudaGetLastError();
  return *err == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int read_device_status(int device, int reset, cudaError_t* err) {
  int prev = 0;
  if ((*err = cudaGetDevice(&prev)) != cudaSuccess) return ATTN_ERR_CUDA;
  if ((*err = cudaSetDevice(device)) != cudaSuccess) return ATTN_ERR_CUDA;
  unsigned int word = 0;
  *err = cudaMemcpyFromSymbol(&word, g_attn_status_word, sizeof(word));
  if (*err == cudaSuccess && reset) {
    const unsigned int zero = 0;
    *err = cudaMemcpyToSymbol(g_attn_status_word, &zero, sizeof(zero));
  }
  cudaError_t e2 = cudaSetDevice(prev);
  if (*err != cudaSuccess) return ATTN_ERR_CUDA;
  if ((*err = e2) != cudaSuccess) return ATTN_ERR_CUDA;
  return (word & kStatusTimeout) ? ATTN_ERR_TIMEOUT : ATTN_OK;
}

}  // namespace ebh

#ifdef EBH_PIPELINE_TRACE
// Profiling builds only: copy out / clear the pipeline trace of CTA 0.
extern "C" __attribute__((visibility("default"))) int attn_pipeline_trace_read(
    unsigned long long* host) {
  return static_cast<int>(
      cudaMemcpyFromSymbol(host, ebh::g_pipeline_trace, sizeof(ebh::g_pipeline_trace)));
}
extern "C" __attribute__((visibility("default"))) int attn_pipeline_trace_clear() {
  static unsigned long long zero[16][ebh::kTraceLen];
  return static_cast<int>(cudaMemcpyToSymbol(ebh::g_pipeline_trace, zero, sizeof(zero)));
}
#endif
