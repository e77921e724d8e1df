"""The pins are strong enough: plant a plausible mistake in a COPY of the
oracle's source, compile it on the CPU, and check that some pin fails.

Nothing here touches the committed oracle; each mutant lives in a temp dir.
"""
import os
import shutil
import subprocess

import pytest

import oracle
from tests import _pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.c")
HDR = os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.h")

# (name, text in the source, replacement) -- each a mistake a careful reader
# might still make: a dropped term, a wrong sign or index, a transposed operand.
MUTANTS = [
    ("dropped_scale", "s[j] = scale * dot;", "s[j] = dot;"),
    ("causal_sign", "return j <= i;", "return j >= i;"),
    ("window_off_by_one", "(i - j <= window) && (j - i <= window)",
     "(i - j < window) && (j - i <= window)"),
    ("lse_log2", "*lse = m + log(l);", "*lse = m + log2(l);"),
    ("lse_without_max", "*lse = m + log(l);", "*lse = log(l);"),
    ("key_row_is_query_row", "const float* kj = kh + j * d;", "const float* kj = kh + i * d;"),
    ("value_row_is_query_row", "const float* vj = vh + j * d;", "const float* vj = vh + i * d;"),
    ("no_normalisation", "for (int64_t c = 0; c < d; ++c) o[c] /= l;", ""),
    ("q_k_transposed_index", "dot += (double)qi[c] * (double)kj[c];",
     "dot += (double)qi[c] * (double)kh[c * d + (j % d)];"),
    ("kv_no_rescale", "for (int64_t c = 0; c < d; ++c) acc[c] *= alpha;", ""),
    ("kv_sum_not_rescaled", "l *= alpha;", ""),
    ("q_block_tail_dropped", "int64_t i1 = i0 + block < L ? i0 + block : L;",
     "int64_t i1 = i0 + block < L ? i0 + block : L - 1;"),
    ("causal_window_two_sided", "(j <= i) && (i - j <= window)", "(i - j <= window)"),
    ("causal_window_off_by_one", "(j <= i) && (i - j <= window)", "(j <= i) && (i - j < window)"),
    ("mha_out_bias_dropped", "double acc = b_out ? (double)b_out[j] : 0.0;", "double acc = 0.0;"),
    ("mha_k_read_from_q_block", "qkv + (b * L + j) * 3 * E + E + h * d;",
     "qkv + (b * L + j) * 3 * E + h * d;"),
    ("mha_head_offset_wrong", "const double* qi = qkv + (b * L + i) * 3 * E + h * d;",
     "const double* qi = qkv + (b * L + i) * 3 * E + h;"),
    ("bwd_D_sign", "const double ds = P[j] * (dP[j] - D);", "const double ds = P[j] * (dP[j] + D);"),
    ("bwd_dk_missing_scale", "dk[head + j * d + c] += scale * ds * (double)qi[c];",
     "dk[head + j * d + c] += ds * (double)qi[c];"),
    ("bwd_dv_at_query_row", "dv[head + j * d + c] += P[j] * (double)gi[c];",
     "dv[head + i * d + c] += P[j] * (double)gi[c];"),
    ("partial_not_normalised", "for (int64_t c = 0; c < d; ++c) o[c] /= l;\n      lse[bh * L + i]",
     "lse[bh * L + i]"),
    ("partial_range_shifted", "for (int64_t j = key_lo; j < key_hi; ++j) {\n        if (!allowed(i, j, mask_kind, window)) continue;\n        double dot = 0.0;\n        for (int64_t c = 0; c < d; ++c) dot += (double)qi[c] * (double)kh[j * d + c];\n        double p",
     "for (int64_t j = key_lo + 1; j < key_hi; ++j) {\n        if (!allowed(i, j, mask_kind, window)) continue;\n        double dot = 0.0;\n        for (int64_t c = 0; c < d; ++c) dot += (double)qi[c] * (double)kh[j * d + c];\n        double p"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(old, new)
    shutil.copy(HDR, tmp_path / "attn_oracle.h")
    (tmp_path / "attn_oracle.c").write_text(mutated)
    so = tmp_path / f"mutant_{name}.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                    "-ffp-contract=off", "-o", str(so), str(tmp_path / "attn_oracle.c"), "-lm"],
                   check=True)
    orc = oracle.load_variant(str(so))
    failures = []
    for pin in _pins.ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, RuntimeError, IndexError, ValueError):
            failures.append(pin.__name__)
    assert failures, f"mutant {name} passed every pin"
