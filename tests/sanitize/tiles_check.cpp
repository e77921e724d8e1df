// Host check of the tile rules in csrc/tiles.h against a brute-force mask,
// built with AddressSanitizer and UndefinedBehaviorSanitizer by
// tests/test_sanitizers.py.  Exit status 0 means every rule matched.
#include <cstdio>
#include <vector>

#include "tiles.h"

using namespace ebh;

static bool allowed(int i, int j, int kind, int w) {
  if (kind == kMaskCausal) return j <= i;
  if (kind == kMaskWindow) return i - j <= w && j - i <= w;
  if (kind == kMaskCausalWindow) return j <= i && i - j <= w;
  return true;
}

int main() {
  int bad = 0;
  const int Ls[] = {1, 2, 63, 64, 65, 127, 128, 129, 200, 257};
  const int bns[] = {32, 64, 128};
  const int windows[] = {0, 1, 5, 63, 64, 130, 1000};
  for (int L : Ls)
    for (int kind = 0; kind <= 3; ++kind)
      for (int w : windows) {
        if ((kind == kMaskNone || kind == kMaskCausal) && w != 0) continue;
        for (int bn : bns) {
          const int nkv = (L + bn - 1) / bn;
          for (int q0 = 0; q0 < L; q0 += bn) {
            const int q1 = q0 + bn - 1 < L - 1 ? q0 + bn - 1 : L - 1;
            int lo, hi, flo, fhi;
            kv_tile_range(L, q0, q1, kind, w, bn, lo, hi);
            kv_full_range(L, q0, q1, kind, w, bn, flo, fhi);
            for (int j = 0; j < nkv; ++j) {
              int n_allowed = 0, n_pairs = 0;
              for (int i = q0; i <= q1; ++i)
                for (int c = j * bn; c < (j + 1) * bn; ++c) {
                  ++n_pairs;
                  if (c < L && allowed(i, c, kind, w)) ++n_allowed;
                }
              const int want = n_allowed == 0 ? kTileEmpty
                                              : (n_allowed == n_pairs ? kTileFull : kTilePartial);
              const int got = kv_tile_class(L, q0, q1, j, kind, w, bn);
              if (got != want || ((lo <= j && j < hi) != (want != kTileEmpty)) ||
                  ((flo <= j && j < fhi) != (want == kTileFull))) {
                if (bad++ < 10)
                  std::printf("L=%d kind=%d w=%d bn=%d q0=%d j=%d: class %d want %d\n", L, kind, w,
                              bn, q0, j, got, want);
              }
              for (int i = q0; i <= q1; ++i) {
                int c_lo, c_hi;
                row_allowed_cols(L, i, j, kind, w, bn, c_lo, c_hi);
                for (int c = 0; c < bn; ++c) {
                  const bool in = c >= c_lo && c < c_hi;
                  const bool ok = j * bn + c < L && allowed(i, j * bn + c, kind, w);
                  if (in != ok && bad++ < 10)
                    std::printf("row cols L=%d kind=%d w=%d i=%d j=%d c=%d\n", L, kind, w, i, j, c);
                }
              }
            }
            // the backward's rule: rows that may attend to keys [q0, q1]
            int r_lo, r_hi;
            query_rows_for_keys(L, q0, q1, kind, w, r_lo, r_hi);
            int first = -1, last = -1;
            for (int i = 0; i < L; ++i)
              for (int c = q0; c <= q1; ++c)
                if (allowed(i, c, kind, w)) {
                  if (first < 0) first = i;
                  last = i;
                }
            if (first >= 0 && (r_lo != first || r_hi != last + 1) && bad++ < 10)
              std::printf("query rows L=%d kind=%d w=%d keys=%d: [%d,%d) want [%d,%d]\n", L, kind,
                          w, q0, r_lo, r_hi, first, last);
          }
        }
      }
  std::printf("tile rules: %d mismatches\n", bad);
  return bad == 0 ? 0 : 1;
}
