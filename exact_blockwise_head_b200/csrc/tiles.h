// tiles.h -- which key blocks a block of query rows must visit, and which of
// them need an element-wise mask.  Shared by the host API (exported for
// tests) and the kernels, so both apply one rule.
//
// Masks: causal keeps key j <= query i; window keeps |i - j| <= w, the band of
// "Attention optimisation strategies and practice for long-sequence inference"
// (trdm.cn), section 2.1; causal window keeps that band's causal side only,
// i - w <= j <= i.  Skipping blocks with no allowed pair is what makes the
// windows cost O(L w) instead of O(L^2), the point of that section.
#pragma once

#ifdef __CUDACC__
#define EBH_HD __host__ __device__ __forceinline__
#else
#define EBH_HD inline
#endif

namespace ebh {

enum : int { kMaskNone = 0, kMaskCausal = 1, kMaskWindow = 2, kMaskCausalWindow = 3 };
enum : int { kTileEmpty = 0, kTilePartial = 1, kTileFull = 2 };

// Key blocks [lo, hi) holding at least one allowed key for some query row in
// [q_first, q_last] (inclusive; q_last < L).  `window` must be >= 0.
EBH_HD void kv_tile_range(int L, int q_first, int q_last, int mask_kind,
                          int window, int bn, int& lo, int& hi) {
  const int nkv = (L + bn - 1) / bn;
  lo = 0;
  hi = nkv;
  if (mask_kind == kMaskCausal) {
    const int h = q_last / bn + 1;
    hi = h < nkv ? h : nkv;
  } else if (mask_kind == kMaskWindow) {
    const long long a = (long long)q_first - window;
    lo = a <= 0 ? 0 : (int)(a / bn);
    const long long b = (long long)q_last + window;
    const long long h = b / bn + 1;
    hi = h < nkv ? (int)h : nkv;
  } else if (mask_kind == kMaskCausalWindow) {
    const long long a = (long long)q_first - window;
    lo = a <= 0 ? 0 : (int)(a / bn);
    const int h = q_last / bn + 1;
    hi = h < nkv ? h : nkv;
  }
}

// Class of key block j for rows [q_first, q_last]: FULL when every pair is
// allowed and every key is < L, EMPTY when no pair is allowed, else PARTIAL.
EBH_HD int kv_tile_class(int L, int q_first, int q_last, int j, int mask_kind,
                         int window, int bn) {
  const long long k0 = (long long)j * bn;
  const long long k1 = k0 + bn - 1;  // inclusive
  if (k0 >= L || j < 0) return kTileEmpty;
  if (mask_kind == kMaskCausal) {
    if (k0 > q_last) return kTileEmpty;
    if (k1 < L && k1 <= q_first) return kTileFull;
    return kTilePartial;
  }
  if (mask_kind == kMaskWindow) {
    if (k0 > (long long)q_last + window || k1 < (long long)q_first - window) return kTileEmpty;
    if (k1 < L && (long long)q_last - k0 <= window && k1 - (long long)q_first <= window)
      return kTileFull;
    return kTilePartial;
  }
  if (mask_kind == kMaskCausalWindow) {
    if (k0 > q_last || k1 < (long long)q_first - window) return kTileEmpty;
    if (k1 < L && k1 <= q_first && (long long)q_last - k0 <= window) return kTileFull;
    return kTilePartial;
  }
  return k1 < L ? kTileFull : kTilePartial;
}

// Key blocks [flo, fhi) in which every pair of rows [q_first, q_last] and
// keys is allowed and every key is < L (the FULL blocks of kv_tile_class, which
// always form one contiguous run; flo == fhi when there are none).
EBH_HD void kv_full_range(int L, int q_first, int q_last, int mask_kind, int window, int bn,
                          int& flo, int& fhi) {
  long long lo = 0, hi = L / bn;  // blocks entirely below L
  if (mask_kind == kMaskCausal) {
    // (j + 1) bn - 1 <= q_first
    const long long h = ((long long)q_first + 1) / bn;
    if (h < hi) hi = h;
  } else if (mask_kind == kMaskWindow) {
    // q_last - j bn <= w  and  (j + 1) bn - 1 - q_first <= w
    const long long a = (long long)q_last - window;
    if (a > 0) lo = (a + bn - 1) / bn;
    const long long h = ((long long)q_first + window + 1) / bn;
    if (h < hi) hi = h;
  } else if (mask_kind == kMaskCausalWindow) {
    // q_last - j bn <= w  and  (j + 1) bn - 1 <= q_first
    const long long a = (long long)q_last - window;
    if (a > 0) lo = (a + bn - 1) / bn;
    const long long h = ((long long)q_first + 1) / bn;
    if (h < hi) hi = h;
  }
  if (hi < lo) hi = lo;
  flo = (int)lo;
  fhi = (int)hi;
}

// Allowed key columns [c_lo, c_hi) of row i inside key block j (block of bn
// keys starting at j*bn), clipped to the keys < L.
EBH_HD void row_allowed_cols(int L, int i, int j, int mask_kind, int window,
                             int bn, int& c_lo, int& c_hi) {
  const long long k0 = (long long)j * bn;
  long long lo = 0, hi = bn;
  if (L - k0 < hi) hi = L - k0;
  if (mask_kind == kMaskCausal) {
    const long long h = (long long)i - k0 + 1;
    if (h < hi) hi = h;
  } else if (mask_kind == kMaskWindow) {
    const long long h = (long long)i + window - k0 + 1;
    if (h < hi) hi = h;
    const long long l = (long long)i - window - k0;
    if (l > lo) lo = l;
  } else if (mask_kind == kMaskCausalWindow) {
    const long long h = (long long)i - k0 + 1;
    if (h < hi) hi = h;
    const long long l = (long long)i - window - k0;
    if (l > lo) lo = l;
  }
  if (hi < lo) hi = lo;
  if (lo > bn) lo = bn;
  if (hi < 0) hi = 0;
  c_lo = (int)lo;
  c_hi = (int)hi;
}

// Query rows [r_lo, r_hi) (half-open, clipped to [0, L)) holding at least one
// row that may attend to some key in [k_first, k_last] (inclusive, < L): the
// rows a key block's gradients gather from.
EBH_HD void query_rows_for_keys(int L, int k_first, int k_last, int mask_kind, int window,
                                int& r_lo, int& r_hi) {
  long long lo = 0, hi = L;  // half-open
  if (mask_kind == kMaskCausal) {
    lo = k_first;
  } else if (mask_kind == kMaskWindow) {
    lo = (long long)k_first - window;
    hi = (long long)k_last + window + 1;
  } else if (mask_kind == kMaskCausalWindow) {
    lo = k_first;
    hi = (long long)k_last + window + 1;
  }
  if (lo < 0) lo = 0;
  if (hi > L) hi = L;
  if (hi < lo) hi = lo;
  r_lo = (int)lo;
  r_hi = (int)hi;
}

// May query row i attend to key j (both < L)?
EBH_HD bool pair_allowed(int i, int j, int mask_kind, int window) {
  if (mask_kind == kMaskCausal) return j <= i;
  if (mask_kind == kMaskWindow) return (long long)i - j <= window && (long long)j - i <= window;
  if (mask_kind == kMaskCausalWindow) return j <= i && (long long)i - j <= window;
  return true;
}

}  // namespace ebh
