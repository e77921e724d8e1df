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
//   warps 0-7   softmax for Q tile 0 (four threads per query row)
//   warps 8-15  softmax for Q tile 1
//   warp  16    TMA producer: Q tiles once per unit, then K_j, V_j into a ring
//   warp  17    MMA issuer: S_t = Q_t K_j^T and O_t += P_t V_j (tcgen05, fp32
//               accumulators in tensor memory); owns the tensor-memory block
//   warps 18-19 idle (they complete the producer / MMA warpgroup)
// Tensor memory (columns): S_0 | S_1 | O_0 | O_1.  P_t (bf16, two per column)
// is written over the first half of S_t and fed to the P.V product straight
// from tensor memory.  The MMA warp interleaves the two Q tiles,
//   S_0(j), P_1(j-1).V_(j-1), S_1(j), P_0(j).V_j, S_0(j+1), ...
// and the two softmax groups take turns at the exponentials, so that each
// works while the tensor core runs the other tile's products.  Because
// tcgen05 MMAs complete in issue order, "S_t(j) done" also means
// "P_t(j-1).V done", which lets a softmax thread rescale its own rows of O_t
// without any further barrier.
// At d = 64 the columns leave room for P in its own block (S_0 | S_1 | P_0 |
// P_1 | O_0 | O_1): S_t(j+1) is then issued as soon as the softmax group has
// loaded S_t(j), one block ahead of P_t(j).V, the groups run without turns,
// and a softmax thread waits for the previous P_t.V product before it writes
// P_t or rescales O_t.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <utility>

#include "attn.h"
#include "kernels.h"
#include "sm100_ptx.cuh"
#include "tiles.h"

namespace ebh {
namespace {

constexpr int kBM = 128;          // query rows per Q tile (= tensor-memory lanes)

// Work-unit shape per key-block size.  With 64- and 128-key blocks a unit is
// two 128-row Q tiles that share the K/V stream (S_0 | S_1 | O_0 | O_1 fill
// the 512 tensor-memory columns at d = 128); with 256-key blocks one Q tile's
// S (256 columns) and O (d columns) already take 384, so a unit is one Q tile.
template <int BN>
struct Layout {
  static constexpr int kNQ = BN == 256 ? 1 : 2;  // Q tiles per work unit
  // softmax warps per Q tile: two per tensor-memory sub-partition, four
  // threads per row (16-lane shapes)
  static constexpr int kSoftmaxWarps = 8;
  static constexpr int kSoftmaxThreads = kSoftmaxWarps * 32;
  static constexpr int kUnitRows = kBM * kNQ;
  static constexpr int kThreads = (kNQ * kSoftmaxWarps + 4) * 32;  // + producer, MMA, 2 idle
  static constexpr int kProducerWarp = kNQ * kSoftmaxWarps;
  static constexpr int kMmaWarp = kProducerWarp + 1;
  // 65536 / kThreads rounded down to a multiple of 8
  static constexpr int kLaunchRegs = (65536 / kThreads) / 8 * 8;
  // softmax: a BN/2-wide half row block per thread plus its packed bf16 copy
  static constexpr int kSoftmaxRegs = kNQ == 2 ? 104 : 208;
  static constexpr int kOtherRegs = 64;
  // epilogue staging rows per softmax warp (its rows of the Q tile)
  static constexpr int kOBoxRows = 16;
  static_assert(kSoftmaxRegs * kNQ * kSoftmaxThreads + kOtherRegs * 128 <=
                    kLaunchRegs * kThreads,
                "register split exceeds the launch allocation");
};
// Tuning knobs of the softmax arithmetic.  kPolyEvery: one column group of
// eight in kPolyEvery takes its exponentials from a polynomial on the FMA pipe
// instead of the MUFU pipe (tiles without masked elements only; 0 = none).
// kScalarMath: scalar fp32 FMA/add (default) instead of the paired f32x2
// forms; the paired forms need register-pair moves on the half-rate ALU pipe
// that cost more than the FMA-pipe slots they save.
#ifndef EBH_POLY_EVERY
#define EBH_POLY_EVERY 0
#endif
#ifndef EBH_SCALAR_MATH
#define EBH_SCALAR_MATH 1
#endif
constexpr int kPolyEvery = EBH_POLY_EVERY > 0 ? EBH_POLY_EVERY : 1;
constexpr bool kPolyOn = EBH_POLY_EVERY > 0;
constexpr bool kScalarMath = EBH_SCALAR_MATH != 0;
// Lazy rescale: keep the stale max until the row max exceeds it by more than
// 32 (log2 units).  Probabilities then stay <= 2^32: bf16 and fp32 keep the
// same relative precision at any magnitude, and 2^32 times 2^30 keys times a
// value's magnitude stays far below fp32 overflow (3.4e38).  Rows whose max
// keeps growing (peaked scores) then almost never redo a block; a larger
// jump still takes the exact redo path.
constexpr float kRescaleThreshold = 32.0f;

// Pipeline trace for profiling builds (-DEBH_PIPELINE_TRACE): lane 0 of each
// warp of CTA 0 appends (event << 56 | key block << 40 | clock64) records to
// g_pipeline_trace[warp]; attn_pipeline_trace_read() copies them out.
enum : int {
  kEvSWait = 1, kEvSReady = 2, kEvSLoaded = 3, kEvMaxDone = 4, kEvPWritten = 5, kEvMasked = 8,
  kEvEpilogue = 6, kEvEpilogueDone = 7,
  kEvKWait = 10, kEvKReady = 11, kEvVWait = 16, kEvVReady = 17,
  kEvPWait = 13, kEvPReady = 14,  // + 10 * Q tile
  kEvSIssued = 30, kEvPVIssued = 32,  // + Q tile
  kEvHalf1 = 40, kEvHalf2Loaded = 41, kEvHalf2 = 42, kEvRowMax = 43
};
#ifdef EBH_PIPELINE_TRACE
constexpr int kTraceLen = 8192;
__device__ unsigned long long g_pipeline_trace[20][kTraceLen];
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

// Bounds-checking builds (-DEBH_BOUNDS_CHECK, the debug library): every
// global store of the kernel checks its element index against the array's
// extent; an index outside is counted in g_bounds_violations and the store is
// skipped (no trap).  Release builds compile the check away.
#ifdef EBH_BOUNDS_CHECK
__device__ unsigned long long g_bounds_violations;
__device__ __forceinline__ bool in_bounds(size_t idx, size_t n) {
  if (idx < n) return true;
  atomicAdd(&g_bounds_violations, 1ull);
  return false;
}
#else
__device__ __forceinline__ bool in_bounds(size_t, size_t) { return true; }
#endif

template <int D, int BN>
struct Cfg {
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(BN == 64 || BN == 128 || BN == 256, "key block");
  static constexpr int kNQ = Layout<BN>::kNQ;
  static constexpr int kDChunks = D / 64;            // 128-byte (64 x bf16) column chunks
  static constexpr int kQTileBytes = kBM * D * 2;
  static constexpr int kKVTileBytes = BN * D * 2;
  static constexpr int kStages = kKVTileBytes >= 65536 ? 2 : (kKVTileBytes >= 32768 ? 4 : 8);
  static constexpr int kSmemQ = kNQ * kQTileBytes;
  static constexpr int kSmemKV = kStages * kKVTileBytes;
  // epilogue staging: one 16-row x 64-column bf16 box (128-byte swizzle) per
  // softmax warp, written by the warp and stored by TMA
  static constexpr int kOBoxBytes = Layout<BN>::kOBoxRows * 128;
  static constexpr int kSmemO = kNQ * Layout<BN>::kSoftmaxWarps * kOBoxBytes;
  // barrier indices
  static constexpr int kBarQFull = 0;                  // [kNQ]
  static constexpr int kBarQEmpty = kBarQFull + kNQ;   // [kNQ]
  static constexpr int kBarKVFull = kBarQEmpty + kNQ;  // [kStages]
  static constexpr int kBarKVEmpty = kBarKVFull + kStages;
  static constexpr int kBarSFull = kBarKVEmpty + kStages;  // [kNQ]
  static constexpr int kBarPFull = kBarSFull + kNQ;        // [kNQ][2]: halves of P_t
  static constexpr int kBarOFull = kBarPFull + 2 * kNQ;    // [kNQ]
  static constexpr int kBarOEmpty = kBarOFull + kNQ;       // [kNQ]
  static constexpr int kBarTok = kBarOEmpty + kNQ;        // [kNQ]
  static constexpr int kBarDrain = kBarTok + kNQ;
  // P in its own tensor-memory columns (d = 64, two-tile units): S_t(j+1)
  // is issued as soon as the softmax has loaded S_t(j), one block ahead of
  // P_t(j) V_j, and the two softmax groups run without turns
  static constexpr bool kDecouple = D == 64 && kNQ == 2;
  static constexpr int kBarSCons = kBarDrain + 1;     // [kNQ]: S_t loaded into registers
  static constexpr int kBarPEmpty = kBarSCons + kNQ;  // [kNQ]: P_t's columns read by P.V
  static constexpr int kNumBars = kBarPEmpty + kNQ;
  static constexpr int kSmemBytes = 1024 + kSmemQ + kSmemKV + kSmemO + 8 * kNumBars + 16;
  static constexpr int kTmemNeed = kNQ * BN + (kDecouple ? kNQ * BN / 2 : 0) + kNQ * D;
  static constexpr int kTmemCols = kTmemNeed <= 256 ? 256 : 512;
  static constexpr int kColS = 0;                                       // + t * BN
  static constexpr int kColP = kDecouple ? kNQ * BN : 0;                // + t * BN / 2
  static constexpr int kColO = kNQ * BN + (kDecouple ? kNQ * BN / 2 : 0);  // + t * D
  static_assert(kTmemNeed <= 512, "tensor memory budget");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

struct Params {
  void* out;
  float* lse;
  long long o_row, o_head, o_batch;  // element strides of out
  size_t o_extent;                   // elements from out to one past its last
  int H;
  int BH, L;      // L query rows per head (q, out, lse)
  int Lk;         // key rows per head (k, v)
  int q_shift;    // query row i sits at key position q_shift + i
  int mask_kind, window;
  float scale_log2;  // scale * log2(e)
  int num_units, nqp;
  uint64_t timeout_ns;
  // Split-KV mode (o_part != nullptr): the key blocks are cut into runs of
  // split_blocks; unit u covers split u % num_splits, and writes its fp32
  // partial O (normalised within the split) and partial LSE to
  // o_part[s][bh][row][:] and lse_part[s][bh][row] instead of out / lse.
  int num_splits, split_blocks;
  float* o_part;
  float* lse_part;
};

// One Q tile of unit u: its head, first/last query row and the key blocks
// [lo, hi) it must visit (empty -> the tile does no work in this unit).
struct TileWork {
  int bh, split;
  bool valid;
  int q_first, q_last, lo, hi;
};

template <int BN>
__device__ __forceinline__ TileWork decode_tile(int u, int t, const Params& p) {
  TileWork w;
  w.split = 0;
  if (p.num_splits > 1) {
    w.split = u % p.num_splits;
    u /= p.num_splits;
  }
  int qp;
  if (p.mask_kind == kMaskCausal) {
    // longest units first: causal work grows with the query position
    qp = p.nqp - 1 - u / p.BH;
    w.bh = u % p.BH;
  } else {
    w.bh = u / p.nqp;
    qp = u % p.nqp;
  }
  w.q_first = qp * Layout<BN>::kUnitRows + t * kBM;
  w.valid = t < Layout<BN>::kNQ && w.q_first < p.L &&
            in_bounds(static_cast<size_t>(w.bh), static_cast<size_t>(p.BH));
  w.q_last = min(w.q_first + kBM - 1, p.L - 1);
  w.lo = w.hi = 0;
  if (w.valid) {
    kv_tile_range(p.Lk, w.q_first + p.q_shift, w.q_last + p.q_shift, p.mask_kind, p.window, BN,
                  w.lo, w.hi);
    if (w.hi <= w.lo) {
      // no key block to visit (query rows placed outside a key shard's
      // reach): the tile does no work and writes nothing
      w.valid = false;
      w.lo = w.hi = 0;
    }
    if (w.valid && p.num_splits > 1) {
      w.lo = max(w.lo, w.split * p.split_blocks);
      w.hi = min(w.hi, (w.split + 1) * p.split_blocks);
      if (w.hi <= w.lo) {
        w.valid = false;
        w.lo = w.hi = 0;
      }
    }
  }
  return w;
}

struct Unit {
  int bh;
  bool valid[2];  // per Q tile of the unit (a one-tile unit leaves [1] invalid)
  int q_first[2], lo[2], hi[2];
  int ulo, uhi;  // union of the two key-block ranges
};

template <int BN>
__device__ __forceinline__ Unit decode_unit(int u, const Params& p) {
  Unit w;
  w.ulo = 0x7fffffff;
  w.uhi = 0;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const TileWork tw = decode_tile<BN>(u, t, p);
    w.bh = tw.bh;
    w.valid[t] = tw.valid;
    w.q_first[t] = tw.q_first;
    w.lo[t] = tw.lo;
    w.hi[t] = tw.hi;
    if (tw.valid) {
      w.ulo = min(w.ulo, tw.lo);
      w.uhi = max(w.uhi, tw.hi);
    }
  }
  if (w.uhi <= w.ulo) w.ulo = w.uhi = 0;
  return w;
}

// The k-th unit of this CTA.  Units are dealt out in rounds of gridDim.x,
// every other round in reverse CTA order: with causal units sorted longest
// first, this evens the per-CTA totals (plain round-robin gives CTA 0 the
// longest unit of every round).  Returns num_units once the CTA is done.
__device__ __forceinline__ int unit_of(int k, const Params& p) {
  const long long base = static_cast<long long>(k) * gridDim.x;
  const long long u = base + ((k & 1) ? gridDim.x - 1 - blockIdx.x : blockIdx.x);
  return u < p.num_units ? static_cast<int>(u) : p.num_units;
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
  while (!mbar_wait_suspend(bar, parity, 20000u)) {
    if (globaltimer_ns() - t0 > limit) {
      atomicOr(&g_attn_status_word, kStatusTimeout);
      return;
    }
  }
}

// ---- softmax helpers (four threads per row, two rows per thread; see the
// softmax section of the kernel for the register layout)

// Load / fence half a score row block: BN/2 keys = BN/16 column groups.
template <int BN>
__device__ __forceinline__ void tmem_ld_half(uint32_t taddr, uint32_t* r) {
  if constexpr (BN == 256) {
    tmem_ld_16x256b_x16(taddr, r);
  } else if constexpr (BN == 128) {
    tmem_ld_16x256b_x8(taddr, r);
  } else {
    tmem_ld_16x256b_x4(taddr, r);
  }
}
template <int BN>
__device__ __forceinline__ void reg_fence_half(uint32_t* r) {
  if constexpr (BN == 256) {
    reg_fence64(r);
  } else if constexpr (BN == 128) {
    reg_fence32(r);
  } else {
    reg_fence16(r);
  }
}

// -inf for the keys outside each row's allowed columns, groups [G0, G1).
template <int G0, int G1>
__device__ __forceinline__ void mask_groups(float* s, int t0, int a_lo, int a_hi, int b_lo,
                                            int b_hi) {
#pragma unroll
  for (int m = G0; m < G1; ++m) {
    const int c = 8 * m + 2 * t0;
    if (c < a_lo || c >= a_hi) s[4 * m] = -INFINITY;
    if (c + 1 < a_lo || c + 1 >= a_hi) s[4 * m + 1] = -INFINITY;
    if (c < b_lo || c >= b_hi) s[4 * m + 2] = -INFINITY;
    if (c + 1 < b_lo || c + 1 >= b_hi) s[4 * m + 3] = -INFINITY;
  }
}

// Row maxima of the thread's two rows over the whole block, then across the
// four threads that share each row.
template <int BN>
__device__ __forceinline__ void row_max_pair(const float* s, float& mta, float& mtb) {
  float xa0 = s[0], xa1 = s[1], xb0 = s[2], xb1 = s[3];
#pragma unroll
  for (int m = 1; m < BN / 8; m += 2) {
    if (m + 1 < BN / 8) {
      xa0 = max3(xa0, s[4 * m], s[4 * m + 4]);
      xa1 = max3(xa1, s[4 * m + 1], s[4 * m + 5]);
      xb0 = max3(xb0, s[4 * m + 2], s[4 * m + 6]);
      xb1 = max3(xb1, s[4 * m + 3], s[4 * m + 7]);
    } else {
      xa0 = fmaxf(xa0, s[4 * m]);
      xa1 = fmaxf(xa1, s[4 * m + 1]);
      xb0 = fmaxf(xb0, s[4 * m + 2]);
      xb1 = fmaxf(xb1, s[4 * m + 3]);
    }
  }
  mta = fmaxf(xa0, xa1);
  mtb = fmaxf(xb0, xb1);
  mta = fmaxf(mta, __shfl_xor_sync(0xffffffffu, mta, 1));
  mtb = fmaxf(mtb, __shfl_xor_sync(0xffffffffu, mtb, 1));
  mta = fmaxf(mta, __shfl_xor_sync(0xffffffffu, mta, 2));
  mtb = fmaxf(mtb, __shfl_xor_sync(0xffffffffu, mtb, 2));
}

// p = 2^(s cl2 - m) for column groups [G0, G1) (multiples of 4), packed to bf16
// and written over the first half of S_t (group m -> packed column 4m + t0);
// l += p, lr += bf16(p), per row.
template <int G0, int G1, bool kPoly>
__device__ __forceinline__ void probabilities(const float* s, float cl2, float ma, float mb,
                                              uint32_t tS, float& l_a, float& l_b, float& lr_a,
                                              float& lr_b) {
#pragma unroll
  for (int ch = G0 / 4; ch < G1 / 4; ++ch) {
    uint32_t pk[8];
#pragma unroll
    for (int mm = 0; mm < 4; ++mm) {
      const int m = 4 * ch + mm;
      float x0, x1, x2, x3, p0, p1, p2, p3;
      if constexpr (kScalarMath) {
        x0 = fmaf(s[4 * m], cl2, -ma);
        x1 = fmaf(s[4 * m + 1], cl2, -ma);
        x2 = fmaf(s[4 * m + 2], cl2, -mb);
        x3 = fmaf(s[4 * m + 3], cl2, -mb);
      } else {
        fma2(x0, x1, s[4 * m], s[4 * m + 1], cl2, cl2, -ma, -ma);
        fma2(x2, x3, s[4 * m + 2], s[4 * m + 3], cl2, cl2, -mb, -mb);
      }
      if (kPoly && (m % kPolyEvery) == kPolyEvery - 1) {
        exp2_poly2(x0, x1, p0, p1);
        exp2_poly2(x2, x3, p2, p3);
      } else {
        p0 = ex2_approx(x0);
        p1 = ex2_approx(x1);
        p2 = ex2_approx(x2);
        p3 = ex2_approx(x3);
      }
      pk[2 * mm] = pack_bf16x2(p0, p1);
      pk[2 * mm + 1] = pack_bf16x2(p2, p3);
      if constexpr (kScalarMath) {
        l_a += p0;
        l_b += p2;
        l_a += p1;
        l_b += p3;
      } else {
        add2(l_a, l_b, l_a, l_b, p0, p2);
        add2(l_a, l_b, l_a, l_b, p1, p3);
      }
      acc_bf16x2_sum(lr_a, pk[2 * mm]);
      acc_bf16x2_sum(lr_b, pk[2 * mm + 1]);
    }
    tmem_st_16x128b_x4(tS + 16 * ch, pk);
  }
}

// Same as probabilities(), but the packed bf16 pairs stay in registers
// (pk[2 (m - G0) + {0, 1}]) for a later store_p().
template <int G0, int G1>
__device__ __forceinline__ void probabilities_regs(const float* s, float cl2, float ma, float mb,
                                                   uint32_t* pk, float& l_a, float& l_b,
                                                   float& lr_a, float& lr_b) {
#pragma unroll
  for (int m = G0; m < G1; ++m) {
    const float p0 = ex2_approx(fmaf(s[4 * m], cl2, -ma));
    const float p1 = ex2_approx(fmaf(s[4 * m + 1], cl2, -ma));
    const float p2 = ex2_approx(fmaf(s[4 * m + 2], cl2, -mb));
    const float p3 = ex2_approx(fmaf(s[4 * m + 3], cl2, -mb));
    const uint32_t a = pack_bf16x2(p0, p1), b = pack_bf16x2(p2, p3);
    pk[2 * (m - G0)] = a;
    pk[2 * (m - G0) + 1] = b;
    l_a += p0;
    l_b += p2;
    l_a += p1;
    l_b += p3;
    acc_bf16x2_sum(lr_a, a);
    acc_bf16x2_sum(lr_b, b);
  }
}
// Store the packed pairs of column groups [G0, G1) (multiples of 4).
template <int G0, int G1>
__device__ __forceinline__ void store_p(uint32_t tS, const uint32_t* pk) {
#pragma unroll
  for (int ch = G0 / 4; ch < G1 / 4; ++ch) tmem_st_16x128b_x4(tS + 16 * ch, pk + 8 * (ch - G0 / 4));
}

// O rows *= alpha (alpha_a for the thread's first row, alpha_b for its
// second), all D columns, through tensor memory.  The caller guarantees no MMA
// is writing O_t (its previous P.V product was issued before the S_t product
// the caller has waited for, and tcgen05 MMAs complete in order).
template <int D>
__device__ __forceinline__ void rescale_o_rows(uint32_t tO, float alpha_a, float alpha_b) {
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    uint32_t o[16];
    tmem_ld_16x256b_x4(tO + 32 * c, o);
    tmem_wait_ld();
    reg_fence16(o);
#pragma unroll
    for (int i = 0; i < 16; ++i)
      o[i] = __float_as_uint(__uint_as_float(o[i]) * ((i & 2) ? alpha_b : alpha_a));
    tmem_st_16x256b_x4(tO + 32 * c, o);
  }
}

// kStrided: q, k, v are 4-D tensor maps (d, rows, H, B) and out has element
// strides (row, head, batch); otherwise all four are dense [B, H, rows, d] and
// the maps 3-D (d, rows, B H).
template <int D, int BN, bool kStrided>
__global__ void __launch_bounds__(Layout<BN>::kThreads, 1)
    attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_o, const Params p) {
  using C = Cfg<D, BN>;
  using Lay = Layout<BN>;
  constexpr int kNQ = Lay::kNQ;
  constexpr int kProducerWarp = Lay::kProducerWarp;
  constexpr int kMmaWarp = Lay::kMmaWarp;
  constexpr int kSoftmaxWarps = Lay::kSoftmaxWarps;
  constexpr int kSoftmaxThreads = Lay::kSoftmaxThreads;
  extern __shared__ uint8_t smem_raw[];
  // 128-byte-swizzled tiles need 1024-byte-aligned shared-memory addresses
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::kSmemQ;
  uint8_t* sO = smem + C::kSmemQ + C::kSmemKV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kSmemQ + C::kSmemKV + C::kSmemO);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  auto bar = [&](int i) -> uint32_t { return smem_addr(&bars[i]); };

  if (threadIdx.x == 0) {
    grid_launch_dependents();
    for (int t = 0; t < kNQ; ++t) {
      mbar_init(bar(C::kBarQFull + t), 1);
      mbar_init(bar(C::kBarQEmpty + t), 1);
      mbar_init(bar(C::kBarSFull + t), 1);
      mbar_init(bar(C::kBarPFull + 2 * t), kSoftmaxThreads);
      mbar_init(bar(C::kBarPFull + 2 * t + 1), kSoftmaxThreads);
      mbar_init(bar(C::kBarOFull + t), 1);
      mbar_init(bar(C::kBarOEmpty + t), kSoftmaxThreads);
      mbar_init(bar(C::kBarTok + t), kSoftmaxWarps);
    }
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(C::kBarKVFull + s), 1);
      mbar_init(bar(C::kBarKVEmpty + s), 1);
    }
    mbar_init(bar(C::kBarDrain), 1);
    if constexpr (C::kDecouple) {
      for (int t = 0; t < kNQ; ++t) {
        mbar_init(bar(C::kBarSCons + t), kSoftmaxThreads);
        mbar_init(bar(C::kBarPEmpty + t), 1);
      }
    }
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
  if (warp >= kProducerWarp) {
    regs_shrink<Lay::kOtherRegs>();
    if (warp == kProducerWarp) {
      // ------------------------------------------------------------ producer
      // The whole warp walks the schedule (its counters stay warp-uniform);
      // one elected lane issues the copies.
      const bool leader = elect_one_sync();
      // In a dependent launch the set-up above overlapped the previous
      // kernel; its outputs are read from here on.  The other roles touch
      // global memory only after data these loads brought in.
      grid_dependency_wait();
      {
        int kv_it = 0;
        int q_cnt[kNQ] = {};
        bool ok = true;
        for (int k = 0, u = unit_of(0, p); ok && u < p.num_units; u = unit_of(++k, p)) {
          const Unit w = decode_unit<BN>(u, p);
          auto load_q = [&](int t) -> bool {
            if (!w.valid[t]) return true;
            if (!warp_wait(bar(C::kBarQEmpty + t), (q_cnt[t] & 1) ^ 1, abort_flag, limit))
              return false;
            if (leader) {
              mbar_arrive_expect_tx(bar(C::kBarQFull + t), C::kQTileBytes);
              const uint32_t dst = smem_addr(sQ + t * C::kQTileBytes);
  #pragma unroll
              for (int c = 0; c < C::kDChunks; ++c) {
                if constexpr (kStrided)
                  tma_load_4d(dst + c * kBM * 128, &tm_q, bar(C::kBarQFull + t), c * 64,
                              w.q_first[t], w.bh % p.H, w.bh / p.H);
                else
                  tma_load_3d(dst + c * kBM * 128, &tm_q, bar(C::kBarQFull + t), c * 64,
                              w.q_first[t], w.bh);
              }
            }
            __syncwarp();
            ++q_cnt[t];
            return true;
          };
          for (int t = 0; ok && t < kNQ; ++t) ok = load_q(t);
          for (int j = w.ulo; ok && j < w.uhi; ++j) {
  #pragma unroll 1
            for (int which = 0; which < 2; ++which) {
              const int s = kv_it % C::kStages;
              ok = warp_wait(bar(C::kBarKVEmpty + s), ((kv_it / C::kStages) & 1) ^ 1, abort_flag,
                             limit);
              if (!ok) break;
              if (leader) {
                mbar_arrive_expect_tx(bar(C::kBarKVFull + s), C::kKVTileBytes);
                const uint32_t dst = smem_addr(sKV + s * C::kKVTileBytes);
                const CUtensorMap* map = which == 0 ? &tm_k : &tm_v;
  #pragma unroll
                for (int c = 0; c < C::kDChunks; ++c)
                  if constexpr (kStrided)
                    tma_load_4d(dst + c * BN * 128, map, bar(C::kBarKVFull + s), c * 64, j * BN,
                                w.bh % p.H, w.bh / p.H);
                  else
                    tma_load_3d(dst + c * BN * 128, map, bar(C::kBarKVFull + s), c * 64, j * BN,
                                w.bh);
              }
              __syncwarp();
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
      // The whole warp walks the schedule, so that counters and descriptors
      // are warp-uniform (uniform registers); one elected lane issues each
      // tcgen05 instruction, and the commits, which track the MMAs of the
      // issuing thread.  With a single thread running the loop, every
      // descriptor had to be moved into the uniform datapath per instruction.
      const bool leader = elect_one_sync();
      {
        constexpr uint32_t idesc_s = idesc_bf16_f32(kBM, BN, false);
        constexpr uint32_t idesc_o = idesc_bf16_f32(kBM, D, true);
        constexpr uint32_t kStageUnits = C::kKVTileBytes >> 4;
        constexpr uint32_t kQTileUnits = C::kQTileBytes >> 4;
        // Shared-memory descriptors are linear in the start address (a field
        // in 16-byte units that cannot carry for addresses below 256 KB): keep
        // the common high word and the three low words, add offsets per K step.
        const uint32_t desc_hi = static_cast<uint32_t>(sdesc_sw128(0, 16, 1024) >> 32);
        const uint32_t lo_q = static_cast<uint32_t>(sdesc_sw128(smem_addr(sQ), 16, 1024));
        const uint32_t lo_k = static_cast<uint32_t>(sdesc_sw128(smem_addr(sKV), 16, 1024));
        const uint32_t lo_v = static_cast<uint32_t>(sdesc_sw128(smem_addr(sKV), BN * 128, 1024));
        auto desc = [&](uint32_t lo) -> uint64_t {
          return (static_cast<uint64_t>(desc_hi) << 32) | lo;
        };
        int kv_it = 0;
        uint32_t par_q = 0, par_p = 0, par_oe = 3;  // one phase bit per Q tile
        bool ok = true;
        EBH_TRACE_COUNTER;

        auto issue_s = [&](int t, int kst) {
          const uint32_t a0 = lo_q + t * kQTileUnits;
          const uint32_t b0 = lo_k + kst * kStageUnits;
          const uint32_t d = tmem + C::kColS + t * BN;
          if (leader) {
  #pragma unroll
            for (int k = 0; k < D / 16; ++k)
              mma_ss(d, desc(a0 + (((k / 4) * kBM * 128 + (k % 4) * 32) >> 4)),
                     desc(b0 + (((k / 4) * BN * 128 + (k % 4) * 32) >> 4)), idesc_s,
                     k > 0 ? 1u : 0u);
          }
          __syncwarp();
        };
        auto commit = [&](uint32_t b) {
          if (leader) mma_commit(b);
          __syncwarp();
        };
        // O_t (+)= P_t V_j in two halves of the keys: each half is issued as
        // soon as the softmax group has released that half of P_t.
        auto issue_pv = [&](int t, int vst, bool first) -> bool {
          const uint32_t b0 = lo_v + vst * kStageUnits;
          const uint32_t d = tmem + C::kColO + t * D;
          const uint32_t a =
              tmem + (C::kDecouple ? C::kColP + t * (BN / 2) : C::kColS + t * BN);
  #pragma unroll
          for (int h = 0; h < 2; ++h) {
            EBH_TRACE(kEvPWait + 10 * t, h);
            if (!warp_wait(bar(C::kBarPFull + 2 * t + h), (par_p >> t) & 1, abort_flag, limit))
              return false;
            EBH_TRACE(kEvPReady + 10 * t, h);
            if (h == 0 && first &&
                !warp_wait(bar(C::kBarOEmpty + t), (par_oe >> t) & 1, abort_flag, limit))
              return false;
            tc_fence_after();
            if (leader) {
  #pragma unroll
              for (int k = h * (BN / 32); k < (h + 1) * (BN / 32); ++k)
                mma_ts(d, a + k * 8, desc(b0 + ((k * 16 * 128) >> 4)), idesc_o,
                       (first && k == 0) ? 0u : 1u);
            }
            __syncwarp();
          }
          par_p ^= 1u << t;
          EBH_TRACE(kEvPVIssued + t, 0);
          return true;
        };

        if constexpr (C::kDecouple) {
          // S one block ahead: per step j, S_t(j+1) for both tiles (each as
          // soon as its softmax group has loaded S_t(j)), then P_t(j) V_j
          // for both.  Counters of S products issued and consumed run across
          // units, like the barriers' phases.
          uint32_t n_s0 = 0, n_s1 = 0;
          for (int k = 0, u = unit_of(0, p); ok && u < p.num_units; u = unit_of(++k, p)) {
            const TileWork w0 = decode_tile<BN>(u, 0, p);
            const TileWork w1 = decode_tile<BN>(u, 1, p);
            const int lo0 = w0.lo, hi0 = w0.valid ? w0.hi : w0.lo;
            const int lo1 = w1.lo, hi1 = w1.valid ? w1.hi : w1.lo;
            const bool has0 = hi0 > lo0, has1 = hi1 > lo1;
            const int ulo = has0 ? (has1 ? min(lo0, lo1) : lo0) : (has1 ? lo1 : 0);
            const int uhi = has0 ? (has1 ? max(hi0, hi1) : hi0) : (has1 ? hi1 : 0);
            const int kv0 = kv_it;  // ring index of K_ulo; V_j follows K_j
            kv_it += 2 * (uhi - ulo);
            auto ring_wait = [&](int i) -> bool {
              return warp_wait(bar(C::kBarKVFull + i % C::kStages), (i / C::kStages) & 1,
                               abort_flag, limit);
            };
            // S_t(j) into S_t's columns once the previous S_t has been loaded
            auto issue_s_ahead = [&](int t, int j, int kst) -> bool {
              const uint32_t n = t ? n_s1 : n_s0;
              if (n > 0 && !warp_wait(bar(C::kBarSCons + t), (n - 1) & 1, abort_flag, limit))
                return false;
              const int lo_t = t ? lo1 : lo0, hi_t = t ? hi1 : hi0;
              if (j == lo_t &&
                  !warp_wait(bar(C::kBarQFull + t), (par_q >> t) & 1, abort_flag, limit))
                return false;
              tc_fence_after();
              issue_s(t, kst);
              commit(bar(C::kBarSFull + t));
              if (j == hi_t - 1) commit(bar(C::kBarQEmpty + t));
              if (t)
                ++n_s1;
              else
                ++n_s0;
              return true;
            };
            auto s_step = [&](int j) -> bool {
              const int ki = kv0 + 2 * (j - ulo);
              if (!ring_wait(ki)) return false;
              const int kst = ki % C::kStages;
              if (j >= lo0 && j < hi0 && !issue_s_ahead(0, j, kst)) return false;
              if (j >= lo1 && j < hi1 && !issue_s_ahead(1, j, kst)) return false;
              commit(bar(C::kBarKVEmpty + kst));  // K_j no longer needed
              return true;
            };
            if (uhi > ulo) ok = s_step(ulo);
            for (int j = ulo; ok && j < uhi; ++j) {
              if (j + 1 < uhi && !(ok = s_step(j + 1))) break;
              const int vi = kv0 + 2 * (j - ulo) + 1;
              if (!(ok = ring_wait(vi))) break;
              const int vst = vi % C::kStages;
              if (j >= lo0 && j < hi0) {
                if (!(ok = issue_pv(0, vst, j == lo0))) break;
                commit(bar(C::kBarPEmpty + 0));
                if (j == hi0 - 1) commit(bar(C::kBarOFull + 0));
              }
              if (j >= lo1 && j < hi1) {
                if (!(ok = issue_pv(1, vst, j == lo1))) break;
                commit(bar(C::kBarPEmpty + 1));
                if (j == hi1 - 1) commit(bar(C::kBarOFull + 1));
              }
              commit(bar(C::kBarKVEmpty + vst));  // V_j no longer needed
            }
            const uint32_t used = (has0 ? 1u : 0u) | (has1 ? 2u : 0u);
            par_q ^= used;
            par_oe ^= used;
          }
        } else {
          // d = 128, and one-tile units: P over S_t, the groups take turns
          for (int k = 0, u = unit_of(0, p); ok && u < p.num_units; u = unit_of(++k, p)) {
            // key-block ranges of the two Q tiles (empty range: tile absent)
            int lo0, hi0, lo1 = 0, hi1 = 0;  // a one-tile unit has no tile 1
            {
              const TileWork w0 = decode_tile<BN>(u, 0, p);
              lo0 = w0.lo; hi0 = w0.valid ? w0.hi : w0.lo;
              if constexpr (kNQ == 2) {
                const TileWork w1 = decode_tile<BN>(u, 1, p);
                lo1 = w1.lo; hi1 = w1.valid ? w1.hi : w1.lo;
              }
            }
            const bool has0 = hi0 > lo0, has1 = hi1 > lo1;
            const int ulo = has0 ? (has1 ? min(lo0, lo1) : lo0) : (has1 ? lo1 : 0);
            const int uhi = has0 ? (has1 ? max(hi0, hi1) : hi0) : (has1 ? hi1 : 0);
            int pend_v = -1;  // ring stage of V_(j-1) still owed a P_1 . V product
            for (int j = ulo; ok && j < uhi; ++j) {
              const int kst = kv_it % C::kStages;
              const uint32_t kph = (kv_it / C::kStages) & 1;
              const int vst = (kv_it + 1) % C::kStages;
              const uint32_t vph = ((kv_it + 1) / C::kStages) & 1;
              kv_it += 2;
              EBH_TRACE(kEvKWait, j);
              if (!(ok = warp_wait(bar(C::kBarKVFull + kst), kph, abort_flag, limit))) break;
              EBH_TRACE(kEvKReady, j);
              const bool in0 = j >= lo0 && j < hi0, in1 = j >= lo1 && j < hi1;
              if (in0) {
                if (j == lo0 && !(ok = warp_wait(bar(C::kBarQFull + 0), par_q & 1, abort_flag,
                                                    limit)))
                  break;
                tc_fence_after();
                issue_s(0, kst);
                EBH_TRACE(kEvSIssued + 0, j);
                commit(bar(C::kBarSFull + 0));
                if (j == hi0 - 1) commit(bar(C::kBarQEmpty + 0));
              }
              if (pend_v >= 0) {
                if (!(ok = issue_pv(1, pend_v, j - 1 == lo1))) break;
                commit(bar(C::kBarKVEmpty + pend_v));
                if (j - 1 == hi1 - 1) commit(bar(C::kBarOFull + 1));
                pend_v = -1;
              }
              if (in1) {
                if (j == lo1 && !(ok = warp_wait(bar(C::kBarQFull + 1), (par_q >> 1) & 1,
                                                    abort_flag, limit)))
                  break;
                tc_fence_after();
                issue_s(1, kst);
                EBH_TRACE(kEvSIssued + 1, j);
                commit(bar(C::kBarSFull + 1));
                if (j == hi1 - 1) commit(bar(C::kBarQEmpty + 1));
              }
              commit(bar(C::kBarKVEmpty + kst));  // K_j no longer needed
              EBH_TRACE(kEvVWait, j);
              if (!(ok = warp_wait(bar(C::kBarKVFull + vst), vph, abort_flag, limit))) break;
              EBH_TRACE(kEvVReady, j);
              if (in0) {
                if (!(ok = issue_pv(0, vst, j == lo0))) break;
                if (j == hi0 - 1) commit(bar(C::kBarOFull + 0));
              }
              if (in1) {
                pend_v = vst;
              } else {
                commit(bar(C::kBarKVEmpty + vst));
              }
            }
            if (ok && pend_v >= 0) {
              if ((ok = issue_pv(1, pend_v, uhi - 1 == lo1))) {
                commit(bar(C::kBarKVEmpty + pend_v));
                if (uhi - 1 == hi1 - 1) commit(bar(C::kBarOFull + 1));
              }
            }
            // Q tiles and O accumulators used by this unit move to their next phase
            const uint32_t used = (has0 ? 1u : 0u) | (has1 ? 2u : 0u);
            par_q ^= used;
            par_oe ^= used;
          }
        }
        // No MMA may still be writing tensor memory when it is freed.
        commit(bar(C::kBarDrain));
        drain_wait(bar(C::kBarDrain), 0, limit);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    // Eight warps per Q tile, two per tensor-memory sub-partition (lanes
    // 32q..32q+15 and 32q+16..32q+31).  Four threads share a row: lane l holds
    // rows l/4 and l/4 + 8 of its warp's 16, and the key columns 8m + 2(l%4)
    // and 8m + 2(l%4) + 1 of every group of eight.
    regs_grow<Lay::kSoftmaxRegs>();
    const int t = warp / kSoftmaxWarps;
    const int wl = warp % kSoftmaxWarps;
    const int lbase = 32 * (warp % 4) + 16 * (wl / 4);  // first row (= lane) of this warp
    const int t0 = lane % 4;
    const int ra = lbase + lane / 4;                   // the thread's rows in the Q tile
    const int rb = ra + 8;
    const uint32_t lane_addr = static_cast<uint32_t>(lbase) << 16;
    const uint32_t tS = tmem + lane_addr + C::kColS + t * BN;
    const uint32_t tO = tmem + lane_addr + C::kColO + t * D;
    // P_t's bf16 pairs: over the first half of S_t, or in their own columns
    const uint32_t tP = C::kDecouple ? tmem + lane_addr + C::kColP + t * (BN / 2) : tS;
    uint32_t n_p = 0;  // P_t blocks written (own columns: P.V products awaited)
    const float cl2 = p.scale_log2;
    uint32_t phase = 0;  // bit 0: S_full parity, bit 1: O_full parity
    bool ok = true;
    // The two Q tiles take turns at the exponentials: tile 1 starts key block
    // j once tile 0 has finished its exponentials of block j, tile 0 starts
    // block j once tile 1 has finished block j - 1.  Each tile counts the
    // other's completions (one phase of kBarTok + tile per key block) to know
    // which phase to wait for.  Without the turns, both groups share the
    // exponential unit and finish together, and the tensor core then runs
    // all four products of the step with no softmax to overlap.
    const int other = t ^ 1;
    uint32_t tok_base = 0;  // key blocks the other tile finished in earlier units
    EBH_TRACE_COUNTER;

    for (int k = 0, u = unit_of(0, p); ok && u < p.num_units; u = unit_of(++k, p)) {
      const TileWork w = decode_tile<BN>(u, t, p);
      const TileWork wo = decode_tile<BN>(u, other, p);
      const int o_lo = wo.valid ? wo.lo : 0, o_hi = wo.valid ? wo.hi : 0;
      const uint32_t o_base = tok_base;
      tok_base += static_cast<uint32_t>(o_hi - o_lo);
      if (!w.valid) continue;
      const int row_a = w.q_first + ra, row_b = w.q_first + rb;
      int full_lo, full_hi;  // key blocks that need no element mask
      kv_full_range(p.Lk, w.q_first + p.q_shift, w.q_last + p.q_shift, p.mask_kind, p.window, BN,
                    full_lo, full_hi);
      // per row: running max (log2 units), sum of the probabilities against
      // it and sum of their bf16 roundings
      float m_a = -INFINITY, m_b = -INFINITY;
      float l_a = 0.f, l_b = 0.f, lr_a = 0.f, lr_b = 0.f;

      for (int j = w.lo; j < w.hi; ++j) {
        EBH_TRACE(kEvSWait, j);
        if (!(ok = warp_wait(bar(C::kBarSFull + t), phase & 1, abort_flag, limit))) break;
        EBH_TRACE(kEvSReady, j);
        phase ^= 1;
        tc_fence_after();
        // Scores in two halves of BN/2 keys: the second half's load overlaps
        // the first half's exponentials.
        constexpr int kHalf = BN / 16;  // column groups of 8 per half
        uint32_t sr[BN / 2];
        tmem_ld_half<BN>(tS, sr);
        if constexpr (!C::kDecouple) {
          const int jo = t == 0 ? j - 1 : j;  // the other tile's block that goes first
          if (jo >= o_lo && jo < o_hi) {
            const uint32_t kt = o_base + static_cast<uint32_t>(jo - o_lo);
            if (!(ok = warp_wait(bar(C::kBarTok + other), kt & 1, abort_flag, limit))) {
              tmem_wait_ld();
              break;
            }
          }
        }
        tmem_wait_ld();
        reg_fence_half<BN>(sr);
        if constexpr (C::kDecouple) {
          // P_t's columns and O_t are free once the previous P_t V product
          // has completed
          if (n_p > 0 &&
              !(ok = warp_wait(bar(C::kBarPEmpty + t), (n_p - 1) & 1, abort_flag, limit)))
            break;
          ++n_p;
        }
        tmem_ld_half<BN>(tS + BN / 2, sr + BN / 4);
        float* s = reinterpret_cast<float*>(sr);
        EBH_TRACE(kEvSLoaded, j);

        const bool full = j >= full_lo && j < full_hi;
        int a_lo = 0, a_hi = BN, b_lo = 0, b_hi = BN;
        if (!full) {
          row_allowed_cols(p.Lk, row_a + p.q_shift, j, p.mask_kind, p.window, BN, a_lo, a_hi);
          row_allowed_cols(p.Lk, row_b + p.q_shift, j, p.mask_kind, p.window, BN, b_lo, b_hi);
          mask_groups<0, kHalf>(s, t0, a_lo, a_hi, b_lo, b_hi);
        }
        EBH_TRACE(kEvMasked, j);

        // The branch must be warp-uniform: both sides run warp-collective
        // tensor-memory instructions and shuffles.
        bool released_a = false;  // first half of P already handed to the MMA warp
        if (__all_sync(0xffffffffu, m_a != -INFINITY && m_b != -INFINITY)) {
          // Speculate that the stale reference max still holds (the tile max
          // exceeds it by at most the threshold): the exponentials need not
          // wait for this tile's row max.
          const float l_a0 = l_a, l_b0 = l_b, lr_a0 = lr_a, lr_b0 = lr_b;
          EBH_TRACE(kEvMaxDone, j);
          if (full) {
            probabilities<0, kHalf, kPolyOn>(s, cl2, m_a, m_b, tP, l_a, l_b, lr_a, lr_b);
          } else {
            probabilities<0, kHalf, false>(s, cl2, m_a, m_b, tP, l_a, l_b, lr_a, lr_b);
          }
          EBH_TRACE(kEvHalf1, j);
          tmem_wait_ld();
          reg_fence_half<BN>(sr + BN / 4);
          if constexpr (C::kDecouple) {  // S_t's columns may take S_t(j+1)
            tc_fence_before();
            mbar_arrive(bar(C::kBarSCons + t));
          }
          EBH_TRACE(kEvHalf2Loaded, j);
          if (!full) mask_groups<kHalf, 2 * kHalf>(s, t0, a_lo, a_hi, b_lo, b_hi);
          float mta, mtb;
          row_max_pair<BN>(s, mta, mtb);
          mta *= cl2;
          mtb *= cl2;
          EBH_TRACE(kEvRowMax, j);
          const bool grow_a = mta > m_a + kRescaleThreshold;
          const bool grow_b = mtb > m_b + kRescaleThreshold;
          if (!__any_sync(0xffffffffu, grow_a || grow_b)) {
            // The speculation held.  Second half into registers; by then the
            // first half's stores have landed, so it is handed to the MMA
            // warp at once and its P.V product overlaps the second half's
            // stores.
            uint32_t pk2[BN / 8];
            probabilities_regs<kHalf, 2 * kHalf>(s, cl2, m_a, m_b, pk2, l_a, l_b, lr_a, lr_b);
            EBH_TRACE(kEvHalf2, j);
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::kBarTok + t));
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(C::kBarPFull + 2 * t));
            released_a = true;
            store_p<kHalf, 2 * kHalf>(tP, pk2);
          } else {
            // rare: redo the tile against the grown maximum
            float alpha_a = 1.f, alpha_b = 1.f;
            if (grow_a) {
              alpha_a = ex2_approx(m_a - mta);
              m_a = mta;
            }
            if (grow_b) {
              alpha_b = ex2_approx(m_b - mtb);
              m_b = mtb;
            }
            l_a = l_a0 * alpha_a;
            lr_a = lr_a0 * alpha_a;
            l_b = l_b0 * alpha_b;
            lr_b = lr_b0 * alpha_b;
            rescale_o_rows<D>(tO, alpha_a, alpha_b);
            probabilities<0, 2 * kHalf, false>(s, cl2, m_a, m_b, tP, l_a, l_b, lr_a, lr_b);
            EBH_TRACE(kEvHalf2, j);
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::kBarTok + t));
          }
        } else {
          // first key block with an allowed key for some row of this thread:
          // take the tile max as the reference before any exponential
          tmem_wait_ld();
          reg_fence_half<BN>(sr + BN / 4);
          if constexpr (C::kDecouple) {
            tc_fence_before();
            mbar_arrive(bar(C::kBarSCons + t));
          }
          if (!full) mask_groups<kHalf, 2 * kHalf>(s, t0, a_lo, a_hi, b_lo, b_hi);
          float mta, mtb;
          row_max_pair<BN>(s, mta, mtb);
          mta *= cl2;
          mtb *= cl2;
          float alpha_a = 1.f, alpha_b = 1.f;
          bool grow = false;
          if (m_a == -INFINITY) {
            m_a = mta;  // nothing accumulated for this row yet
          } else if (mta > m_a + kRescaleThreshold) {
            alpha_a = ex2_approx(m_a - mta);
            m_a = mta;
            grow = true;
          }
          if (m_b == -INFINITY) {
            m_b = mtb;
          } else if (mtb > m_b + kRescaleThreshold) {
            alpha_b = ex2_approx(m_b - mtb);
            m_b = mtb;
            grow = true;
          }
          if (__any_sync(0xffffffffu, grow)) {
            l_a *= alpha_a;
            lr_a *= alpha_a;
            l_b *= alpha_b;
            lr_b *= alpha_b;
            rescale_o_rows<D>(tO, alpha_a, alpha_b);
          }
          EBH_TRACE(kEvMaxDone, j);
          // a row with every key masked so far keeps m = -inf: subtract 0 so
          // that -inf - (-inf) never happens (its probabilities are all 0)
          probabilities<0, 2 * kHalf, false>(s, cl2, m_a == -INFINITY ? 0.f : m_a,
                                      m_b == -INFINITY ? 0.f : m_b, tP, l_a, l_b, lr_a, lr_b);
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(C::kBarTok + t));
        }
        tmem_wait_st();
        tc_fence_before();
        EBH_TRACE(kEvPWritten, j);
        if (!released_a) mbar_arrive(bar(C::kBarPFull + 2 * t));
        mbar_arrive(bar(C::kBarPFull + 2 * t + 1));
      }
      if (!ok) break;

      // ---- epilogue: O / lr -> bf16, LSE = ln 2 * (m + log2 l)
      EBH_TRACE(kEvEpilogue, 0);
      if (!(ok = warp_wait(bar(C::kBarOFull + t), (phase >> 1) & 1, abort_flag, limit))) break;
      phase ^= 2;
      tc_fence_after();
#pragma unroll
      for (int x = 1; x <= 2; x <<= 1) {
        l_a += __shfl_xor_sync(0xffffffffu, l_a, x);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, x);
        lr_a += __shfl_xor_sync(0xffffffffu, lr_a, x);
        lr_b += __shfl_xor_sync(0xffffffffu, lr_b, x);
      }
      // O is divided by the sum of exactly the (bf16) weights that multiplied
      // V, so the weights sum to one; LSE uses the unrounded sum.
      const float inv_a = lr_a > 0.f ? 1.f / lr_a : 0.f;
      const float inv_b = lr_b > 0.f ? 1.f / lr_b : 0.f;
      const bool ok_a = row_a < p.L, ok_b = row_b < p.L;
      const float lse_a = l_a > 0.f ? (m_a + log2f(l_a)) * 0.69314718055994531f : -INFINITY;
      const float lse_b = l_b > 0.f ? (m_b + log2f(l_b)) * 0.69314718055994531f : -INFINITY;
      // All of O_t's rows of this thread in one load; once it has landed the
      // accumulator is free for the next unit's first P.V product.
      uint32_t o[D / 2];
      if constexpr (D == 128) {
        tmem_ld_16x256b_x16(tO, o);
        tmem_wait_ld();
        reg_fence64(o);
      } else {
        tmem_ld_16x256b_x8(tO, o);
        tmem_wait_ld();
        reg_fence32(o);
      }
      tc_fence_before();
      mbar_arrive(bar(C::kBarOEmpty + t));
      // register 4m + {0, 1}: row a, columns 8m + 2 t0 + {0, 1}; 4m + {2, 3}: row b
      if (p.o_part == nullptr) {
        // O / l -> bf16 into this warp's 16-row staging box, laid out as the
        // TMA's 128-byte swizzle (16-byte unit u of row r at u ^ (r % 8)),
        // then one TMA store per 64-column chunk: coalesced full-line writes,
        // rows past L clipped by the tensor map.  The lane's rows in the box
        // are lane / 4 and lane / 4 + 8 (same r % 8), its 4-byte slot 4 t0.
        uint8_t* box = sO + warp * C::kOBoxBytes;
        const int r_box = lane / 4;
        const int warp_row0 = w.q_first + lbase;  // the box's first row in the head
#pragma unroll
        for (int c = 0; c < C::kDChunks; ++c) {
          if (lane == 0) bulk_wait_group_read0();  // the box's previous store has read it
          __syncwarp();
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int m = 8 * c + u;  // column group: columns 8m + 2 t0 + {0, 1}
            const uint32_t va = pack_bf16x2(__uint_as_float(o[4 * m]) * inv_a,
                                            __uint_as_float(o[4 * m + 1]) * inv_a);
            const uint32_t vb = pack_bf16x2(__uint_as_float(o[4 * m + 2]) * inv_b,
                                            __uint_as_float(o[4 * m + 3]) * inv_b);
            const int slot = ((u ^ (r_box & 7)) * 16) + 4 * t0;
            *reinterpret_cast<uint32_t*>(box + r_box * 128 + slot) = va;
            *reinterpret_cast<uint32_t*>(box + (r_box + 8) * 128 + slot) = vb;
          }
          fence_proxy_async_shared();
          __syncwarp();
          if (lane == 0 && warp_row0 < p.L) {
            if constexpr (kStrided)
              tma_store_4d(&tm_o, smem_addr(box), c * 64, warp_row0, w.bh % p.H, w.bh / p.H);
            else
              tma_store_3d(&tm_o, smem_addr(box), c * 64, warp_row0, w.bh);
            bulk_commit_group();
          }
        }
        if (t0 == 0 && p.lse != nullptr) {
          const size_t n_lse = static_cast<size_t>(p.BH) * p.L;
          if (ok_a && in_bounds(static_cast<size_t>(w.bh) * p.L + row_a, n_lse))
            p.lse[static_cast<size_t>(w.bh) * p.L + row_a] = lse_a;
          if (ok_b && in_bounds(static_cast<size_t>(w.bh) * p.L + row_b, n_lse))
            p.lse[static_cast<size_t>(w.bh) * p.L + row_b] = lse_b;
        }
      } else {
        // split-KV partial: fp32 O normalised within the split, and its LSE
        const size_t head = static_cast<size_t>(w.split) * p.BH + w.bh;
        float2* dst_a = reinterpret_cast<float2*>(
            p.o_part + (head * p.L + (ok_a ? row_a : 0)) * D);
        float2* dst_b = reinterpret_cast<float2*>(
            p.o_part + (head * p.L + (ok_b ? row_b : 0)) * D);
#pragma unroll
        for (int m = 0; m < D / 8; ++m) {
          const int col2 = 4 * m + t0;
          const size_t n_part = static_cast<size_t>(p.num_splits) * p.BH * p.L * (D / 2);
          if (ok_a && in_bounds((head * p.L + row_a) * (D / 2) + col2, n_part))
            dst_a[col2] = make_float2(__uint_as_float(o[4 * m]) * inv_a,
                                      __uint_as_float(o[4 * m + 1]) * inv_a);
          if (ok_b && in_bounds((head * p.L + row_b) * (D / 2) + col2, n_part))
            dst_b[col2] = make_float2(__uint_as_float(o[4 * m + 2]) * inv_b,
                                      __uint_as_float(o[4 * m + 3]) * inv_b);
        }
        if (t0 == 0) {
          const size_t n_lpart = static_cast<size_t>(p.num_splits) * p.BH * p.L;
          if (ok_a && in_bounds(head * p.L + row_a, n_lpart)) p.lse_part[head * p.L + row_a] = lse_a;
          if (ok_b && in_bounds(head * p.L + row_b, n_lpart)) p.lse_part[head * p.L + row_b] = lse_b;
        }
      }
      EBH_TRACE(kEvEpilogueDone, 0);
    }
  }

  // the epilogue's staging boxes must have been read before the CTA's shared
  // memory goes; the global writes complete with the kernel
  if (warp < kProducerWarp && lane == 0) bulk_wait_group_read0();
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

// bf16 tensor, boxes of `rows` x 64 columns of one head, 128-byte swizzle;
// rows past L read as zero.  map4: seen as (D, L, H, B) with element strides
// (row, head, batch); else dense, seen as (D, L, B H).
bool make_map(CUtensorMap* map, const void* base, int B, int H, int L, int D,
              const long long* stride, int rows, bool map4, cudaError_t* err) {
  EncodeTiledFn fn = encode_fn(err);
  if (!fn) return false;
  const cuuint64_t dims4[4] = {(cuuint64_t)D, (cuuint64_t)L, (cuuint64_t)H, (cuuint64_t)B};
  const cuuint64_t strides4[3] = {(cuuint64_t)stride[0] * 2, (cuuint64_t)stride[1] * 2,
                                  (cuuint64_t)stride[2] * 2};
  const cuuint64_t dims3[3] = {(cuuint64_t)D, (cuuint64_t)L, (cuuint64_t)B * H};
  const cuuint64_t strides3[2] = {(cuuint64_t)D * 2, (cuuint64_t)L * D * 2};
  const cuuint32_t box[4] = {64, (cuuint32_t)rows, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, map4 ? 4 : 3, const_cast<void*>(base),
                  map4 ? dims4 : dims3, map4 ? strides4 : strides3, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
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

// Launch with or without the programmatic-dependent-launch attribute (the
// kernel's own griddepcontrol instructions do the rest).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), int grid, int threads, int smem,
                          cudaStream_t stream, bool dependent, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <int D, int BN>
int launch_t(const FwdArgs& a, cudaStream_t stream, cudaError_t* err) {
  using C = Cfg<D, BN>;
  // dense inputs and output keep the 3-D maps and the plain epilogue (measured
  // 0.5-3.5 % faster than the strided instantiation on dense data)
  bool strided = false;
  for (int x = 0; x < 4; ++x) strided = strided || a.stride[x][0] != 0;
  using Lay = Layout<BN>;
  auto kernel = strided ? attn_fwd_sm100_kernel<D, BN, true> : attn_fwd_sm100_kernel<D, BN, false>;
  int device = 0;
  if ((*err = cudaGetDevice(&device)) != cudaSuccess) return ATTN_ERR_CUDA;
  {
    static std::mutex mu;
    static bool attr_set[64][2] = {};
    std::lock_guard<std::mutex> g(mu);
    if (device >= 64) {
      *err = cudaErrorInvalidDevice;
      return ATTN_ERR_CUDA;
    }
    if (!attr_set[device][strided]) {
      *err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  C::kSmemBytes);
      if (*err != cudaSuccess) return ATTN_ERR_CUDA;
      // The in-kernel register split assumes exactly kLaunchRegs per thread
      // at launch; refuse to launch a build where that does not hold.
      cudaFuncAttributes fa;
      if ((*err = cudaFuncGetAttributes(&fa, kernel)) != cudaSuccess) return ATTN_ERR_CUDA;
      if (fa.numRegs != Lay::kLaunchRegs) {
        *err = cudaErrorInvalidConfiguration;
        return ATTN_ERR_CUDA;
      }
      attr_set[device][strided] = true;
    }
  }
  const int nsm = sm_count(device, err);
  if (nsm <= 0) return ATTN_ERR_CUDA;

  const int BH = a.B * a.H;
  const int Lk = a.Lk > 0 ? a.Lk : a.L;
  // element strides (row, head, batch); zero: dense [B, H, rows, D]
  long long st[4][3];
  for (int x = 0; x < 4; ++x) {
    const long long rows = x == 1 || x == 2 ? Lk : a.L;
    const bool dense = a.stride[x][0] == 0;
    st[x][0] = dense ? D : a.stride[x][0];
    st[x][1] = dense ? rows * D : a.stride[x][1];
    st[x][2] = dense ? static_cast<long long>(a.H) * rows * D : a.stride[x][2];
  }
  CUtensorMap tq, tk, tv, to;
  if (!make_map(&tq, a.q, a.B, a.H, a.L, D, st[0], kBM, strided, err)) return ATTN_ERR_CUDA;
  // output: 16-row boxes, one per softmax warp's epilogue store
  if (!make_map(&to, a.out, a.B, a.H, a.L, D, st[3], Lay::kOBoxRows, strided, err))
    return ATTN_ERR_CUDA;
  if (!make_map(&tk, a.k, a.B, a.H, Lk, D, st[1], BN, strided, err)) return ATTN_ERR_CUDA;
  if (!make_map(&tv, a.v, a.B, a.H, Lk, D, st[2], BN, strided, err)) return ATTN_ERR_CUDA;

  Params p;
  p.out = a.out;
  p.lse = a.lse;
  p.o_row = st[3][0];
  p.o_head = st[3][1];
  p.o_batch = st[3][2];
  p.o_extent = static_cast<size_t>((a.B - 1) * st[3][2] + (a.H - 1) * st[3][1] +
                                   static_cast<long long>(a.L - 1) * st[3][0] + D);
  p.H = a.H;
  p.BH = BH;
  p.L = a.L;
  p.Lk = Lk;
  p.q_shift = a.q_shift;
  p.mask_kind = a.mask_kind;
  p.window = a.window;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.nqp = (a.L + Lay::kUnitRows - 1) / Lay::kUnitRows;
  p.num_splits = 1;
  p.split_blocks = 0;
  p.o_part = nullptr;
  p.lse_part = nullptr;
  if (a.o_part != nullptr) {
    p.num_splits = a.num_splits;
    p.split_blocks = a.split_keys / BN;
    p.o_part = a.o_part;
    p.lse_part = a.lse_part;
  }
  const long long units = static_cast<long long>(BH) * p.nqp * p.num_splits;
  if (units > 0x7fffffffLL) {
    *err = cudaErrorInvalidValue;
    return ATTN_ERR_UNSUPPORTED;
  }
  p.num_units = static_cast<int>(units);
  p.timeout_ns = a.timeout_ns;
  const int grid = p.num_units < nsm ? p.num_units : nsm;
  *err = launch_kernel(kernel, grid, Lay::kThreads, C::kSmemBytes, stream, a.dependent, tq, tk, tv,
                       to, p);
  return *err == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

int launch_fwd_bf16_sm100(const FwdArgs& a, cudaStream_t stream, cudaError_t* err) {
  *err = cudaSuccess;
  if (a.d == 128 && a.block_n == 128) return launch_t<128, 128>(a, stream, err);
  if (a.d == 128 && a.block_n == 64) return launch_t<128, 64>(a, stream, err);
  if (a.d == 128 && a.block_n == 256) return launch_t<128, 256>(a, stream, err);
  if (a.d == 64 && a.block_n == 128) return launch_t<64, 128>(a, stream, err);
  if (a.d == 64 && a.block_n == 64) return launch_t<64, 64>(a, stream, err);
  if (a.d == 64 && a.block_n == 256) return launch_t<64, 256>(a, stream, err);
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

// The backward's tensor-core kernels share this translation unit's helpers and
// its device status word.
#include "attn_bwd_sm100.cuh"
#include "linear_sm100.cuh"

#ifdef EBH_BOUNDS_CHECK
// Bounds-checking builds only: the number of refused out-of-range stores
// since the last reset.
extern "C" __attribute__((visibility("default"))) long long attn_debug_bounds_violations(
    int reset) {
  unsigned long long n = 0;
  if (cudaMemcpyFromSymbol(&n, ebh::g_bounds_violations, sizeof(n)) != cudaSuccess) return -1;
  if (reset) {
    const unsigned long long zero = 0;
    if (cudaMemcpyToSymbol(ebh::g_bounds_violations, &zero, sizeof(zero)) != cudaSuccess)
      return -1;
  }
  return static_cast<long long>(n);
}
#endif

#ifdef EBH_PIPELINE_TRACE
// Profiling builds only: copy out / clear the pipeline trace of CTA 0.
extern "C" __attribute__((visibility("default"))) int attn_pipeline_trace_read(
    unsigned long long* host) {
  return static_cast<int>(
      cudaMemcpyFromSymbol(host, ebh::g_pipeline_trace, sizeof(ebh::g_pipeline_trace)));
}
extern "C" __attribute__((visibility("default"))) int attn_pipeline_trace_clear() {
  static unsigned long long zero[20][ebh::kTraceLen];
  return static_cast<int>(cudaMemcpyToSymbol(ebh::g_pipeline_trace, zero, sizeof(zero)));
}
#endif
