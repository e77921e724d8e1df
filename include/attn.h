/*
 * attn.h -- C ABI of the exact blockwise multi-head attention forward
 * (libebh_attn.so).
 *
 * Operation.  For every batch b, head h and query row i:
 *     O[b,h,i,:] = sum_j softmax_j( scale * <Q[b,h,i,:], K[b,h,j,:]> + mask(i,j) ) V[b,h,j,:]
 *     LSE[b,h,i] = ln sum_{j allowed} exp( scale * <Q[b,h,i,:], K[b,h,j,:]> )
 * the formula softmax(Q K^T / sqrt(d_k)) V of the page "Transformer multi-head
 * attention, 8-head parallel computation: PyTorch implementation and CUDA
 * kernel optimisation" (lshu.cn), section 1, with the scores of disallowed keys
 * set to -inf before the softmax as in its section 2.2.  The result is exact
 * up to rounding: it is computed tile by tile over blocks of keys with a
 * running max and sum (the fused kernel of the page "Mosaic multi-GPU
 * sequence-sharded attention" (kwkr.cn), section 3.2, with the rescale that
 * sketch omits), so the L x L score matrix is never stored and memory stays
 * O(L), as the query-blockwise scheme of "Blockwise Parallel Transformer in
 * PyTorch" (qqiyuan.cn) intends.
 *
 * Masks.
 *   ATTN_MASK_NONE    every key j in [0, L)
 *   ATTN_MASK_CAUSAL  j <= i (diagonal included; queries and keys aligned)
 *   ATTN_MASK_WINDOW  |i - j| <= window, the band of "Attention optimisation
 *                     strategies and practice for long-sequence inference"
 *                     (trdm.cn), section 2.1, applied additively (-inf)
 *   ATTN_MASK_CAUSAL_WINDOW
 *                     i - window <= j <= i: that band's causal side only
 * Every mask allows the diagonal, so no row is ever fully masked.
 *
 * Layout.  q, k, v, out are dense row-major [B, H, L, d] arrays (d fastest,
 * then L, then H, then B) in device memory.  lse is a dense [B, H, L] fp32
 * array in device memory, or NULL to skip it.
 *
 * Ownership and execution.  The caller owns every buffer.  Each call only
 * enqueues work on `stream` (a cudaStream_t; NULL = the legacy default
 * stream) and returns: it never allocates or frees device memory and never
 * synchronises.  The buffers must stay valid until the work completes.  `out`
 * and `lse` must not overlap q, k, v or each other.  Calls are thread-safe.
 *
 * Errors.  Every argument is validated before anything is launched; a call
 * that returns an error has enqueued nothing (except ATTN_ERR_CUDA, which
 * reports a failed launch).  attn_strerror() names a status.  Waits inside
 * the kernels are bounded: if one runs out (a malfunction, never expected),
 * the kernel records ATTN_ERR_TIMEOUT in a per-device status word, releases
 * its resources and returns; attn_device_status() reads that word.
 */
#ifndef EBH_ATTN_H
#define EBH_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ATTN_ABI_VERSION 1

/* Symbol visibility: the library is built with hidden visibility by default
 * and exports exactly the entry points declared here. */
#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

/* Status codes returned by every entry point. */
enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID = 1,     /* null pointer, non-positive size, bad mask kind,
                               negative window, non-finite or non-positive
                               scale, overlapping outputs, bad block_n/dtype */
  ATTN_ERR_UNSUPPORTED = 2, /* head dim not supported by the chosen path, or
                               the current device is not sm_100 */
  ATTN_ERR_MISALIGNED = 3,  /* q/k/v/out not 16-byte aligned, lse not 4-byte */
  ATTN_ERR_CUDA = 4,        /* a CUDA runtime call failed; attn_last_cuda_error()
                               gives its code */
  ATTN_ERR_TIMEOUT = 5,     /* a bounded wait inside a kernel ran out */
  ATTN_ERR_SCRATCH_LIMIT = 6 /* the problem's partials do not fit the fixed
                               scratch of attn_fwd_splitkv_noalloc */
};

/* Mask kinds. */
enum { ATTN_MASK_NONE = 0, ATTN_MASK_CAUSAL = 1, ATTN_MASK_WINDOW = 2, ATTN_MASK_CAUSAL_WINDOW = 3 };

/* Element types. */
enum { ATTN_DTYPE_BF16 = 0, ATTN_DTYPE_F32 = 1 };

/* Tile classes returned by attn_kv_tile_class(). */
enum { ATTN_TILE_EMPTY = 0, ATTN_TILE_PARTIAL = 1, ATTN_TILE_FULL = 2 };

/*
 * bf16 forward on the sm_100a tensor cores (tcgen05 MMAs into tensor memory,
 * TMA-staged tiles).  q, k, v, out: bf16 [B,H,L,d], d in {64, 128}, 16-byte
 * aligned.  lse: fp32 [B,H,L] or NULL.  Products accumulate in fp32; the
 * softmax runs in fp32 with exp2; the probabilities are rounded to bf16 for
 * the P.V product; out is rounded to bf16 (nearest-even).  B, H, L >= 1 with
 * B*H <= 2^31-1; scale finite and > 0 (the pages use 1/sqrt(d)); window >= 0,
 * read only for the two window masks.  Keys are visited in blocks of 128.
 */
ATTN_API int attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
             int B, int H, int L, int d, float scale, int mask_kind, int window,
             void* stream);

/*
 * fp32 forward on the CUDA cores (exact fp32 arithmetic, expf): q, k, v, out
 * fp32 [B,H,L,d] with 1 <= d <= 256, 16-byte aligned; other arguments as for
 * attn_fwd.  This path keeps full fp32 precision (no TF32).
 */
ATTN_API int attn_fwd_f32(const float* q, const float* k, const float* v, float* out,
                 float* lse, int B, int H, int L, int d, float scale,
                 int mask_kind, int window, void* stream);

/* Full parameter set for attn_fwd_ex(). */
typedef struct attn_params {
  int dtype;              /* ATTN_DTYPE_BF16 or ATTN_DTYPE_F32 */
  const void* q;          /* [B,H,L,d] */
  const void* k;          /* [B,H,L,d] */
  const void* v;          /* [B,H,L,d] */
  void* out;              /* [B,H,L,d], same dtype as q */
  float* lse;             /* [B,H,L] fp32, or NULL */
  int B, H, L, d;
  float scale;
  int mask_kind;
  int window;
  int block_n;            /* keys per block on the bf16 path: 0 (auto = 128),
                             64, 128 or 256; must be 0 on the fp32 path.
                             64 and 128 run two 128-row query tiles per
                             work unit (their softmax overlaps the other
                             tile's products); 256 runs one query tile per
                             unit (S of 256 columns and O of d columns fill
                             the tensor memory), with no such overlap */
  uint64_t wait_timeout_ns; /* limit on each wait inside the kernel; 0 = 10 s */
} attn_params;

/* attn_fwd / attn_fwd_f32 with every knob exposed. */
ATTN_API int attn_fwd_ex(const attn_params* p, void* stream);

/*
 * bf16 forward on tensors in any (row, head, batch) layout with contiguous
 * head dim: element (b, h, i, c) of q sits at
 *   q + b strides[2] + h strides[1] + i strides[0] + c
 * and likewise k (strides[3..5]), v (strides[6..8]) and out (strides[9..11]),
 * all in elements.  For example [B, L, H, d] tensors have strides (H d, d,
 * L H d), and the thirds of a fused [B, L, 3, H, d] projection have (3 H d,
 * d, 3 L H d) from bases 0, H d and 2 H d.  Every stride is positive, a
 * multiple of 8 (16 bytes; the tensor-memory-access copy rule) and, for rows,
 * at least d.  lse stays dense [B, H, L] fp32 or NULL.  out may not overlap q,
 * k, v or lse; q, k, v may overlap each other.  Other arguments and errors as
 * attn_fwd_ex (bf16 only).
 */
ATTN_API int attn_fwd_strided(const attn_params* p, const int64_t* strides, void* stream);

/*
 * Forward for a block of query rows placed inside a longer key sequence:
 * q, out are [B, H, L, d] with L = p->L query rows, k, v are [B, H, kv_len, d],
 * lse is [B, H, L]; query row i sits at key position q_offset + i, and the
 * masks compare key positions with that position.  With q_offset = 0 and
 * kv_len = L this is attn_fwd_ex.  This is the local step of sequence-sharded
 * attention ("Mosaic multi-GPU sequence-sharded attention", section 2.1): a
 * rank holding query rows [r Ls, (r+1) Ls) runs it against the gathered keys.
 * Requires 0 <= q_offset and q_offset + L <= kv_len (every row keeps its own
 * key, so no row is fully masked); window masks are clamped to kv_len.
 * Both dtypes; other arguments and errors as attn_fwd_ex.
 */
ATTN_API int attn_fwd_rows(const attn_params* p, int kv_len, int q_offset, void* stream);

/*
 * Layout step of sequence-sharded attention: an all-gather of S sequence
 * shards of K (or V), each [B, H, Ls, d], leaves them rank-major,
 * gathered = [S, B, H, Ls, d]; this writes out = [B, H, S Ls, d], where shard
 * g's row c becomes key g Ls + c ("Mosaic multi-GPU sequence-sharded
 * attention", section 2.1).  elem_bytes 2 (bf16) or 4 (fp32); both buffers
 * device memory and disjoint.  Asynchronous on `stream`; allocates nothing.
 */
ATTN_API int attn_seq_unshard(const void* gathered, void* out, int S, int B, int H, int Ls, int d,
                              int elem_bytes, void* stream);

/* Static text for a status code (never NULL). */
ATTN_API const char* attn_strerror(int status);

/* The cudaError_t of the last ATTN_ERR_CUDA returned on this thread (0 if none). */
ATTN_API int attn_last_cuda_error(void);

/*
 * Reads, and if `reset` clears, the status word that kernels on `device` set
 * when a bounded wait ran out.  Returns ATTN_OK, ATTN_ERR_TIMEOUT, or
 * ATTN_ERR_CUDA if the device could not be queried.  Unlike every other entry
 * point this one synchronises with the device (it copies the word back).
 */
ATTN_API int attn_device_status(int device, int reset);

/*
 * Failure-detection self test: launches one CTA that waits on a barrier which
 * nothing ever arrives on, with the limit `limit_ns`; the wait runs out, the
 * kernel records ATTN_ERR_TIMEOUT in the device status word and returns
 * normally.  Used to test the bounded-wait path without hanging a GPU.
 */
ATTN_API int attn_selftest_wait_timeout(uint64_t limit_ns, void* stream);

/*
 * Host copies of the tile-skipping rule the kernels use.  Query rows
 * [q_first, q_last] (inclusive, q_last < L) meet key blocks of block_n keys;
 * attn_kv_tile_range() gives the half-open range [lo, hi) of key blocks that
 * hold at least one allowed key, and attn_kv_tile_class() classifies block j
 * as EMPTY (no allowed pair), PARTIAL (some pair masked, or keys past L) or
 * FULL (every pair allowed).  attn_kv_tile_range returns ATTN_ERR_INVALID on
 * bad arguments; attn_kv_tile_class returns -ATTN_ERR_INVALID (negative, so
 * it cannot be mistaken for a class).
 */
ATTN_API int attn_kv_tile_range(int L, int q_first, int q_last, int mask_kind, int window,
                       int block_n, int* lo, int* hi);
ATTN_API int attn_kv_tile_class(int L, int q_first, int q_last, int j, int mask_kind,
                       int window, int block_n);
/* The FULL blocks always form one contiguous run [lo, hi) (lo == hi: none);
 * the kernels test j against it instead of classifying every block. */
ATTN_API int attn_kv_full_range(int L, int q_first, int q_last, int mask_kind, int window,
                                int block_n, int* lo, int* hi);

/*
 * Split-KV forward (bf16 path).  The key blocks are cut into up to
 * num_splits (1..64, or ATTN_SPLITS_AUTO below) contiguous runs; every
 * (query tile, run) pair is an
 * independent work unit, which keeps all SMs busy when B*H*L/256 is small.
 * Each run writes an fp32 partial output normalised within the run and its
 * LSE into `workspace`, then attn_merge's rule combines the runs exactly
 * (the "tree reduction" of local attention results, page "Mosaic multi-GPU
 * sequence-sharded attention", section 2.1).  The workspace is device memory
 * owned by the caller, 256-byte aligned, at least
 * attn_splitkv_workspace_bytes(B, H, L, d, runs) bytes (runs = the number of
 * runs actually used, never more than num_splits; passing num_splits there is
 * always enough); it must not overlap any other argument.  Its contents on
 * entry do not matter.  With one run this is attn_fwd_ex and the workspace
 * is not touched.  Other arguments and errors as attn_fwd_ex.
 *
 * num_splits = ATTN_SPLITS_AUTO (0) lets the library choose from the
 * current device's SM count and the U = B*H*ceil(L/256) work units of one
 * run: floor(SMs / U) runs, at most ATTN_SPLITS_AUTO_MAX and at least one,
 * and at least two for a causal mask when U <= SMs (one unit per SM, so the
 * longest unit sets the time).  Measured on B200 (d=128, L2 flushed):
 * causal B=1 H=4 L=8192 (U=128) 453 -> 664-692 TFLOP/s with two runs; no
 * mask B=1 H=8 L=4096 (U=128) stays at one run (818-866; every split is
 * slower); U=32: four runs, causal B=1 H=1 L=8192 122 -> 305, no mask B=1
 * H=2 L=4096 227 -> 430.  attn_splitkv_workspace_bytes(..., 0) returns the
 * size for the current device's choice under a causal mask (never less than
 * under any other mask), or for ATTN_SPLITS_AUTO_MAX runs when no device
 * answers; query it on the device the call will run on.  The call reads the
 * SM count (ATTN_ERR_CUDA if that query fails).
 */
#define ATTN_SPLITS_AUTO 0
#define ATTN_SPLITS_AUTO_MAX 8
/* The automatic choice as a pure host function (no device call): the number
 * of key runs ATTN_SPLITS_AUTO takes for B, H, L and mask_kind (ATTN_MASK_*)
 * on a device with num_sms SMs, before the cut to whole key blocks (the call
 * never uses more runs than the problem has key blocks).  0 for arguments
 * outside B, H, L, num_sms >= 1 or an unknown mask_kind. */
ATTN_API int attn_splitkv_auto_runs(int B, int H, int L, int mask_kind, int num_sms);
ATTN_API size_t attn_splitkv_workspace_bytes(int B, int H, int L, int d, int num_splits);
ATTN_API int attn_fwd_splitkv(const attn_params* p, int num_splits, void* workspace,
                              size_t workspace_bytes, void* stream);

/*
 * Exact merge of partial results over disjoint key ranges:
 *   LSE_i = ln sum_s exp(LSE_s,i),  O_i = sum_s exp(LSE_s,i - LSE_i) O_s,i
 * over the splits s whose key range [split_bounds[s], split_bounds[s+1])
 * holds a key that row i may attend to under (mask_kind, window); other
 * splits are not read for that row.  o_parts: fp32 [S,B,H,L,d] (16-byte
 * aligned), each partial normalised within its range; lse_parts: fp32
 * [S,B,H,L].  split_bounds: host array of S+1 increasing key indices from 0
 * to L.  out: [B,H,L,d] in out_dtype (ATTN_DTYPE_BF16 rounds to nearest
 * even); lse: fp32 [B,H,L] or NULL.  d in {64, 128}, 1 <= S <= 64.
 * Asynchronous on `stream`; allocates nothing.
 */
ATTN_API int attn_merge(const float* o_parts, const float* lse_parts, int num_splits,
                        const int* split_bounds, int mask_kind, int window, void* out,
                        float* lse, int out_dtype, int B, int H, int L, int d, void* stream);

/*
 * attn_merge for rows placed inside a longer key sequence: row i of the L
 * rows sits at key position q_offset + i among kv_len keys, and split_bounds
 * (S+1 increasing key positions from 0 to kv_len) partition those keys.  A
 * split is read for a row only when its key range holds a key the row may
 * attend to.  0 <= q_offset, q_offset + L <= kv_len.  attn_merge is this call
 * with kv_len = L and q_offset = 0.  This is the combination step of
 * sequence-sharded attention ("Mosaic multi-GPU sequence-sharded attention",
 * section 2.1): each rank merges the partials of its rows over every key
 * shard.  Other arguments and errors as attn_merge.
 */
ATTN_API int attn_merge_rows(const float* o_parts, const float* lse_parts, int num_splits,
                             const int* split_bounds, int mask_kind, int window, void* out,
                             float* lse, int out_dtype, int B, int H, int L, int d, int kv_len,
                             int q_offset, void* stream);

/*
 * Partial forward of query rows against one block of keys, for merging with
 * attn_merge / attn_merge_rows: q is [B, H, L, d], k and v are [B, H, kv_len,
 * d] (bf16), and query row i sits at key position q_shift + i relative to
 * the first of these keys; q_shift may be negative or beyond kv_len (a key
 * shard that lies after or before the rows), and the masks compare those
 * positions.  Writes o_part: fp32 [B, H, L, d], the output over these keys
 * alone (normalised within them), and lse_part: fp32 [B, H, L], its
 * natural-log LSE.  A row with no allowed key among them gets O = 0 and LSE =
 * -inf when its 128-row tile has an allowed key for some other row; a tile
 * with no allowed key at all is not written (the merge's mask rule never
 * reads it).  p->out and p->lse are not used; p->block_n as attn_fwd_ex.
 * o_part (16-byte aligned) and lse_part (4-byte aligned) are device memory
 * and overlap nothing else; |q_shift| + L + kv_len must stay below 2^30.
 * This is the local step of sequence-sharded attention ("Mosaic multi-GPU
 * sequence-sharded attention", section 2.1) for one shard of the keys.
 * Asynchronous on `stream`; allocates nothing.  Errors as attn_fwd_ex.
 */
ATTN_API int attn_fwd_partial(const attn_params* p, int kv_len, int q_shift, float* o_part,
                              float* lse_part, void* stream);

/*
 * Split-KV forward with no workspace argument and no allocation.  The paper
 * has no counterpart to this call: it is a library convenience for callers
 * that cannot allocate device memory for attn_fwd_splitkv's workspace, such
 * as code running under a host framework whose caching allocator owns all
 * device memory, plugin interfaces that hand the library only its inputs and
 * outputs, and latency-critical loops where cudaMalloc/cudaFree (which may
 * synchronise the device) is not acceptable.
 *
 * It computes exactly what attn_fwd_splitkv computes, with the partials kept
 * in a fixed scratch array of ATTN_NOALLOC_SCRATCH_BYTES that the library's
 * device code carries on every device it is loaded on.  It calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *   - Limit: the partials of the runs actually used must fit, i.e.
 *     attn_splitkv_workspace_bytes(B, H, L, d, runs) <= ATTN_NOALLOC_SCRATCH_BYTES
 *     (at d=128 about 64K rows of B*H*L*runs); otherwise it returns
 *     ATTN_ERR_SCRATCH_LIMIT and enqueues nothing.  Every other argument is
 *     checked first, exactly as attn_fwd_splitkv checks it, so an invalid
 *     call gets ATTN_ERR_INVALID / UNSUPPORTED / MISALIGNED whatever its
 *     size.  With one run it is attn_fwd_ex and the scratch is not touched.
 *   - Set-up: the first call on a device (the current device) looks up the
 *     scratch's device address with cudaGetSymbolAddress, in the CUDA
 *     context current on the calling thread, and keeps it with that
 *     context's unique ID.  A later call reuses the address only while the
 *     same context is current; after cudaDeviceReset, or with another
 *     context made current on the device, the next call looks it up again
 *     (that call is again a set-up call).  Make every set-up call before any
 *     stream capture on that device.  A failed look-up returns ATTN_ERR_CUDA.
 *   - Concurrency: every call on a device uses the same scratch, so calls
 *     whose work may overlap on the GPU (unordered streams, several host
 *     threads) race and corrupt each other's results; order them, e.g. on
 *     one stream.
 * Nothing in the scratch needs to start at zero.  Other arguments and errors
 * as attn_fwd_splitkv.
 */
#define ATTN_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
ATTN_API int attn_fwd_splitkv_noalloc(const attn_params* p, int num_splits, void* stream);

/*
 * Backward of the forward by recomputation ("Attention optimisation
 * strategies and practice for long-sequence inference", section 3.1;
 * "Mosaic multi-GPU sequence-sharded attention", section 2.2): the weights
 * P_ij = exp(scale <q_i, k_j> - lse_i) are recomputed from Q, K and the
 * forward's LSE, never stored, and
 *   dV_j = sum_i P_ij dO_i,  dS_ij = P_ij (<dO_i, v_j> - <dO_i, O_i>),
 *   dQ_i = scale sum_j dS_ij k_j,  dK_j = scale sum_i dS_ij q_i.
 * p describes the forward call: q, k, v and p->out (the forward's O) in
 * p->dtype (bf16 or fp32), p->lse (the forward's LSE, required), the mask,
 * window and scale; p->block_n must be 0.  dout: dO, [B, H, L, d] in p->dtype,
 * 16-byte aligned.  dq, dk, dv: fp32 [B, H, L, d] outputs.  workspace:
 * device memory of at least attn_bwd_workspace_bytes(B, H, L) bytes.  No
 * output or the workspace may overlap any other argument.  d <= 128 (bf16:
 * 64 or 128).  fp32 arithmetic on the CUDA cores.  Asynchronous on `stream`.
 */
ATTN_API size_t attn_bwd_workspace_bytes(int B, int H, int L);
/* Host copy of the backward's rule: query rows [*r_lo, *r_hi) holding every
 * row that may attend to some key in [k_first, k_last] (inclusive, < L).
 * ATTN_ERR_INVALID on bad arguments. */
ATTN_API int attn_query_rows_for_keys(int L, int k_first, int k_last, int mask_kind, int window,
                                      int* r_lo, int* r_hi);
ATTN_API int attn_bwd(const attn_params* p, const void* dout, float* dq, float* dk, float* dv,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * The multi-head attention layer of "Transformer multi-head attention, 8-head
 * parallel computation" (lshu.cn), sections 2.1 and 2.2:
 *   qkv = x W_qkv^T + b_qkv; q, k, v = its three E-wide thirds, each split
 *   into H heads of d = E / H; context = attention(q, k, v) with scale
 *   1/sqrt(d) and the mask; y = context W_out^T + b_out.
 * x, y: bf16 [B, L, E]; w_qkv: bf16 [3E, E] (nn.Linear layout: row j makes
 * output feature j; rows [0, E) make q, [E, 2E) k, [2E, 3E) v); w_out: bf16
 * [E, E]; b_qkv [3E] and b_out [E]: bf16 or NULL.  d in {64, 128}; every
 * pointer 16-byte aligned.  The projections run in this library's
 * tensor-core GEMM (tcgen05 MMAs, fp32 accumulation in tensor memory, bias in
 * its epilogue, bf16 results); the attention runs in this library's kernel,
 * reading each head's q, k, v straight from the projection output and
 * writing the context in [B, L, H, d] (the head split and merge are its
 * strides).  The projection output and the context are bf16 in `workspace`:
 * device memory, 256-byte aligned, at least attn_mha_workspace_bytes(B, L, E)
 * bytes, disjoint from the other arguments.  A failed launch returns
 * ATTN_ERR_CUDA with its code in attn_last_cuda_error().  Asynchronous on
 * `stream`.
 */
typedef struct {
  const void* x;
  const void* w_qkv;
  const void* b_qkv;
  const void* w_out;
  const void* b_out;
  void* y;
  int B, L, E, H;
  int mask_kind;
  int window;
} attn_mha_params;
ATTN_API size_t attn_mha_workspace_bytes(int B, int L, int E);
ATTN_API int attn_mha_fwd(const attn_mha_params* p, void* workspace, size_t workspace_bytes,
                          void* stream);

/* ATTN_ABI_VERSION of the loaded library. */
ATTN_API int attn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* EBH_ATTN_H */
