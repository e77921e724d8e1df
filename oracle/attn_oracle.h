/*
 * attn_oracle.h -- fp64 CPU oracle for exact multi-head scaled-dot-product
 * attention forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes
 * or calls this code; only the tests, the smoke check and the bench's CPU
 * baseline leg load it.  It shares no source with the CUDA path.
 *
 * Sources (web pages, cited by title and section):
 *   [MHA-CUDA]  "Transformer multi-head attention, 8-head parallel computation:
 *               PyTorch implementation and CUDA kernel optimisation"
 *               (lshu.cn/news/104643): section 1 gives the formula
 *               softmax(Q K^T / sqrt(d_k)) V; section 2.2 masks scores with
 *               -inf before the softmax.
 *   [LONGSEQ]   "Attention optimisation strategies and practice for
 *               long-sequence inference" (trdm.cn/news/523779): section 2.1,
 *               sliding window, each token sees w tokens before and after.
 *   [BPT]       "Blockwise Parallel Transformer in PyTorch: solving the memory
 *               bottleneck of long-sequence modelling" (qqiyuan.cn): the
 *               query-blockwise attention function (every query block sees
 *               all keys, tail block clipped at L) and the note that blockwise
 *               softmax needs its own normalisation.
 *   [MOSAIC]    "Mosaic multi-GPU sequence-sharded attention"
 *               (kwkr.cn/news/57053): section 3.2, the fused kernel that walks
 *               K/V tiles keeping a running max and sum; section 5.1, NaN from
 *               exp overflow on long sequences, cured by log-space arithmetic.
 *
 * Layout: q, k, v are [B, H, L, d] row-major (d fastest), given as float
 * (bf16 inputs are widened exactly).  out is [B, H, L, d] double, lse is
 * [B, H, L] double (natural-log log-sum-exp of the scaled logits over the
 * allowed keys).  Every function returns 0 on success, -1 on a bad argument,
 * -2 if memory for scratch rows could not be obtained.
 */
#ifndef ATTN_ORACLE_H
#define ATTN_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  ORACLE_MASK_NONE = 0,   /* every key */
  ORACLE_MASK_CAUSAL = 1, /* key j <= query i */
  ORACLE_MASK_WINDOW = 2, /* |i - j| <= window */
  /* i - window <= j <= i: the band of [LONGSEQ] section 2.1 kept on the
   * causal side only (the page's tril(w).triu(-w) with tril at diagonal 0) */
  ORACLE_MASK_CAUSAL_WINDOW = 3
};

/* The plain definition, one query row at a time, rows spread over nthreads. */
int oracle_attn_fwd(const float* q, const float* k, const float* v, double* out,
                    double* lse, int64_t B, int64_t H, int64_t L, int64_t d,
                    double scale, int mask_kind, int64_t window, int nthreads);

/* The definition on selected rows only: row r of the result is query row
 * row_idx[r] of head bh_idx[r] (bh = b * H + h).  out is [nrows, d]. */
int oracle_attn_rows(const float* q, const float* k, const float* v,
                     const int64_t* bh_idx, const int64_t* row_idx,
                     int64_t nrows, double* out, double* lse, int64_t B,
                     int64_t H, int64_t L, int64_t d, double scale,
                     int mask_kind, int64_t window, int nthreads);

/* K/V-blockwise online softmax [MOSAIC 3.2, with the running-max rescale the
 * page leaves out]: keys are visited in blocks of `block`; a running max m,
 * running sum l and unnormalised accumulator are rescaled whenever m grows. */
int oracle_attn_kv_blockwise(const float* q, const float* k, const float* v,
                             double* out, double* lse, int64_t B, int64_t H,
                             int64_t L, int64_t d, double scale, int mask_kind,
                             int64_t window, int64_t block);

/* Query-blockwise attention [BPT]: query rows in blocks of `block` (the last
 * block clipped at L); each block forms its full score rows against all keys,
 * masks, normalises them and multiplies by V. */
int oracle_attn_q_blockwise(const float* q, const float* k, const float* v,
                            double* out, double* lse, int64_t B, int64_t H,
                            int64_t L, int64_t d, double scale, int mask_kind,
                            int64_t window, int64_t block);

/* The definition restricted to keys [key_lo, key_hi) (a key shard's partial
 * result, [MOSAIC 2.1]): out normalised within the range, lse over the range;
 * rows with no allowed key in it get out = 0, lse = -inf. */
int oracle_attn_partial(const float* q, const float* k, const float* v, double* out,
                        double* lse, int64_t B, int64_t H, int64_t L, int64_t d,
                        double scale, int mask_kind, int64_t window, int64_t key_lo,
                        int64_t key_hi);

/* The multi-head attention layer of [MHA-CUDA] sections 2.1-2.2: x [B, L, E],
 * w_qkv [3E, E] and w_out [E, E] in nn.Linear layout, b_qkv [3E] and b_out [E]
 * (NULL: zero), H heads of d = E / H; y [B, L, E] double. */
int oracle_mha_fwd(const float* x, const float* w_qkv, const float* b_qkv, const float* w_out,
                   const float* b_out, double* y, int64_t B, int64_t L, int64_t E, int64_t H,
                   int mask_kind, int64_t window);

/* Backward by recomputation ([LONGSEQ] 3.1, [MOSAIC] 2.2): dQ, dK, dV of the
 * definition given dO, all [B, H, L, d] (dq, dk, dv in double). */
int oracle_attn_bwd(const float* q, const float* k, const float* v, const float* dout,
                    double* dq, double* dk, double* dv, int64_t B, int64_t H, int64_t L,
                    int64_t d, double scale, int mask_kind, int64_t window);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_ORACLE_H */
