"""Pins for the fp64 oracle: facts fixed by the pages and by mathematics.

Each pin takes an object with the oracle's four functions (``attention``,
``attention_rows``, ``attention_kv_blockwise``, ``attention_q_blockwise``) and
raises AssertionError when the oracle disagrees with what the pages fix.  The
pins never retype the oracle's own formula: they use a pure-Python brute force
built the way the pages build their masks, closed forms, invariants and
special cases that reduce to something simpler.

Pages (cited by title and section):
  [MHA-CUDA] "Transformer multi-head attention, 8-head parallel computation:
             PyTorch implementation and CUDA kernel optimisation", section 1
             (formula), section 2.2 (scores masked with -inf).
  [LONGSEQ]  "Attention optimisation strategies and practice for long-sequence
             inference", section 2.1 (band mask ones(n,n).tril(w).triu(-w)).
  [BPT]      "Blockwise Parallel Transformer in PyTorch", the query-blockwise
             function (tail block clipped at L) and the numerical-stability note.
  [MOSAIC]   "Mosaic multi-GPU sequence-sharded attention", section 3.2 (K/V
             tiles with running max and sum), section 5.1 (overflow -> NaN).
"""
from __future__ import annotations

import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# --------------------------------------------------------------------------
# third implementation: pure Python, dense mask built literally, no max
# subtraction, exactly rounded sums (math.fsum)
# --------------------------------------------------------------------------
def dense_mask(L, mask, window):
    """0/1 matrix: causal is tril(diagonal=0); window is tril(diagonal=w) times
    triu(diagonal=-w) as [LONGSEQ 2.1] builds it; causal_window is that band
    with its upper side at the diagonal, tril(diagonal=0) times triu(diagonal=-w)."""
    M = [[1] * L for _ in range(L)]
    for i in range(L):
        for j in range(L):
            if mask == "causal":
                M[i][j] = 1 if j - i <= 0 else 0
            elif mask == "window":
                tril = 1 if j - i <= window else 0
                triu = 1 if j - i >= -window else 0
                M[i][j] = tril * triu
            elif mask == "causal_window":
                tril = 1 if j - i <= 0 else 0
                triu = 1 if j - i >= -window else 0
                M[i][j] = tril * triu
    return M


def brute_force_head(q, k, v, scale, mask, window):
    """softmax(q k^T scale + log M) v for one head given as nested lists."""
    L, d = len(q), len(q[0])
    M = dense_mask(L, mask, window)
    out, lse = [], []
    for i in range(L):
        e = []
        for j in range(L):
            if M[i][j]:
                s = scale * math.fsum(q[i][c] * k[j][c] for c in range(d))
                e.append(math.exp(s))
            else:
                e.append(0.0)
        Z = math.fsum(e)
        out.append([math.fsum(e[j] * v[j][c] for j in range(L)) / Z for c in range(d)])
        lse.append(math.log(Z))
    return out, lse


def _rand(shape, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal(shape) * scale).astype(np.float32)


def _close(a, b, rtol, atol, what):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    err = np.abs(a - b)
    bad = err > atol + rtol * np.abs(b)
    assert not bad.any(), f"{what}: max err {err.max():.3e} at {np.argwhere(bad)[0]}"


# --------------------------------------------------------------------------
# pins
# --------------------------------------------------------------------------
def pin_brute_force(orc):
    """Tiny inputs against the pure-Python brute force, every mask kind."""
    cases = []
    for L in (1, 2, 3, 5, 8, 17):
        for d in (1, 2, 4):
            cases.append((L, d))
    seed = 100
    for L, d in cases:
        for mask, window in (("none", 0), ("causal", 0), ("window", 0), ("window", 1),
                             ("window", 3), ("causal_window", 0), ("causal_window", 2)):
            seed += 1
            q = _rand((1, 1, L, d), seed)
            k = _rand((1, 1, L, d), seed + 1000)
            v = _rand((1, 1, L, d), seed + 2000)
            scale = 0.3 + (seed % 7) * 0.11  # not 1/sqrt(d): a dropped scale shows
            out, lse = orc.attention(q, k, v, scale=scale, mask=mask, window=window)
            bo, bl = brute_force_head(q[0, 0].tolist(), k[0, 0].tolist(), v[0, 0].tolist(),
                                      scale, mask, window)
            _close(out[0, 0], bo, 1e-12, 1e-13, f"brute force out L={L} d={d} {mask}{window}")
            _close(lse[0, 0], bl, 1e-12, 1e-13, f"brute force lse L={L} d={d} {mask}{window}")


def load_golden():
    path = os.path.join(GOLDEN, "hand_case_L2_d1.txt")
    rows, inputs = [], {}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if "=" in line and line.split("=")[0].strip() in ("q", "k", "v"):
                key, vals = line.split("=")
                inputs[key.strip()] = [float(x) for x in vals.split()]
                continue
            mask, window, row, exp_out, exp_lse = (x.strip() for x in line.split("|"))
            env = {"e": math.e, "log": math.log}
            rows.append((mask, int(window), int(row), eval(exp_out, {}, env),
                         eval(exp_lse, {}, env)))
    return inputs, rows


def pin_golden(orc):
    """The hand-derived L=2, d=1 case of tests/golden/hand_case_L2_d1.txt."""
    inputs, rows = load_golden()
    q = np.array(inputs["q"], np.float32).reshape(1, 1, 2, 1)
    k = np.array(inputs["k"], np.float32).reshape(1, 1, 2, 1)
    v = np.array(inputs["v"], np.float32).reshape(1, 1, 2, 1)
    for mask, window, row, eo, el in rows:
        out, lse = orc.attention(q, k, v, scale=1.0, mask=mask, window=window)
        assert abs(out[0, 0, row, 0] - eo) <= 1e-15 * max(1.0, abs(eo)), (mask, row, out, eo)
        assert abs(lse[0, 0, row] - el) <= 1e-15 * max(1.0, abs(el)), (mask, row, lse, el)


def pin_kv_blockwise(orc):
    """[MOSAIC 3.2]: the K/V-blockwise online softmax equals the unblocked
    definition for every block size 1..L, and for large blocks at L=512."""
    L, d = 40, 6
    q, k, v = _rand((1, 2, L, d), 1), _rand((1, 2, L, d), 2), _rand((1, 2, L, d), 3)
    for mask, window in (("none", 0), ("causal", 0), ("window", 4), ("causal_window", 6)):
        ref = orc.attention(q, k, v, mask=mask, window=window)
        for block in range(1, L + 1):
            got = orc.attention_kv_blockwise(q, k, v, block, mask=mask, window=window)
            _close(got[0], ref[0], 1e-12, 1e-13, f"kv-blockwise out b={block} {mask}")
            _close(got[1], ref[1], 1e-12, 1e-13, f"kv-blockwise lse b={block} {mask}")
    L, d = 512, 16
    q, k, v = _rand((1, 1, L, d), 4), _rand((1, 1, L, d), 5), _rand((1, 1, L, d), 6)
    for mask, window in (("none", 0), ("causal", 0), ("window", 37), ("causal_window", 100)):
        ref = orc.attention(q, k, v, mask=mask, window=window)
        for block in (1, 7, 64, 128, 256, 1000):
            got = orc.attention_kv_blockwise(q, k, v, block, mask=mask, window=window)
            _close(got[0], ref[0], 1e-12, 1e-13, f"kv-blockwise L=512 b={block} {mask}")
            _close(got[1], ref[1], 1e-12, 1e-13, f"kv-blockwise L=512 lse b={block} {mask}")


def pin_q_blockwise(orc):
    """[BPT]: query blocks that see every key, tail clipped at L, give the
    unblocked result for every block size."""
    L, d = 29, 5
    q, k, v = _rand((2, 1, L, d), 7), _rand((2, 1, L, d), 8), _rand((2, 1, L, d), 9)
    for mask, window in (("none", 0), ("causal", 0), ("window", 2), ("causal_window", 3)):
        ref = orc.attention(q, k, v, mask=mask, window=window)
        for block in list(range(1, L + 2)) + [256]:
            got = orc.attention_q_blockwise(q, k, v, block, mask=mask, window=window)
            _close(got[0], ref[0], 1e-12, 1e-13, f"q-blockwise out b={block} {mask}")
            _close(got[1], ref[1], 1e-12, 1e-13, f"q-blockwise lse b={block} {mask}")


def _probabilities(orc, q, k, scale, mask, window):
    """Read the softmax matrix through the public call: with d_v = L and V the
    identity, output row i is probability row i."""
    B, H, L, d = q.shape
    # q, k have head dim d; V must share it, so embed: use d = L by padding q, k.
    qp = np.zeros((B, H, L, L), np.float32)
    kp = np.zeros((B, H, L, L), np.float32)
    qp[..., :d] = q
    kp[..., :d] = k
    eye = np.broadcast_to(np.eye(L, dtype=np.float32), (B, H, L, L)).copy()
    out, lse = orc.attention(qp, kp, eye, scale=scale, mask=mask, window=window)
    return out, lse


def pin_probability_rows(orc):
    """Probability rows sum to 1, are >= 0, and are exactly 0 on masked keys."""
    L, d = 24, 4
    q, k = _rand((1, 2, L, d), 10, 2.0), _rand((1, 2, L, d), 11, 2.0)
    for mask, window in (("none", 0), ("causal", 0), ("window", 3), ("causal_window", 4)):
        P, _ = _probabilities(orc, q, k, 0.5, mask, window)
        M = np.array(dense_mask(L, mask, window), bool)
        assert (P >= 0).all()
        assert np.abs(P.sum(-1) - 1.0).max() <= 1e-14, mask
        assert (P[..., ~M] == 0.0).all(), mask
        assert (P[..., M] > 0.0).all(), mask


def pin_identical_keys(orc):
    """All keys equal -> uniform weights over the allowed set: O_i is the mean
    of the allowed V rows and LSE_i = s + ln|A_i|."""
    L, d = 33, 8
    q = _rand((1, 1, L, d), 12)
    k = np.broadcast_to(_rand((1, 1, 1, d), 13), (1, 1, L, d)).copy()
    v = _rand((1, 1, L, d), 14)
    scale = 0.7
    M_all = {m: np.array(dense_mask(L, m, w), bool) for m, w in
             (("none", 0), ("causal", 0), ("window", 5), ("causal_window", 7))}
    for mask, window in (("none", 0), ("causal", 0), ("window", 5), ("causal_window", 7)):
        out, lse = orc.attention(q, k, v, scale=scale, mask=mask, window=window)
        M = M_all[mask]
        for i in range(L):
            sel = v[0, 0][M[i]].astype(np.float64)
            _close(out[0, 0, i], sel.mean(0), 1e-13, 1e-14, f"identical keys {mask} row {i}")
            s = scale * float(np.dot(q[0, 0, i].astype(np.float64), k[0, 0, 0].astype(np.float64)))
            assert abs(lse[0, 0, i] - (s + math.log(M[i].sum()))) <= 1e-12 * max(1, abs(s))


def pin_constant_v(orc):
    """All value rows equal to c -> every output row is c, whatever Q, K, mask."""
    L, d = 50, 7
    q, k = _rand((2, 2, L, d), 15, 3.0), _rand((2, 2, L, d), 16, 3.0)
    c = _rand((1, 1, 1, d), 17)
    v = np.broadcast_to(c, (2, 2, L, d)).copy()
    for mask, window in (("none", 0), ("causal", 0), ("window", 6), ("causal_window", 6)):
        out, _ = orc.attention(q, k, v, mask=mask, window=window)
        _close(out, np.broadcast_to(c.astype(np.float64), out.shape), 1e-14, 1e-14,
               f"constant V {mask}")


def pin_special_cases(orc):
    """w=0 passes V through; w >= L-1 is no mask; causal row 0 is v_0;
    Q=0 gives the mean over the allowed set with LSE ln|A|; permuting K and V
    rows together leaves the unmasked result alone; heads are independent."""
    L, d = 21, 6
    q, k, v = _rand((1, 1, L, d), 18), _rand((1, 1, L, d), 19), _rand((1, 1, L, d), 20)
    scale = 0.4
    out, lse = orc.attention(q, k, v, scale=scale, mask="window", window=0)
    _close(out, v.astype(np.float64), 1e-15, 0.0, "w=0 -> V")
    s_ii = scale * np.einsum("bhld,bhld->bhl", q.astype(np.float64), k.astype(np.float64))
    _close(lse, s_ii, 1e-14, 1e-15, "w=0 -> lse = s_ii")
    ref = orc.attention(q, k, v, scale=scale, mask="none")
    for w in (L - 1, L, 10 * L):
        got = orc.attention(q, k, v, scale=scale, mask="window", window=w)
        _close(got[0], ref[0], 0.0, 0.0, f"w={w} -> none")
        _close(got[1], ref[1], 0.0, 0.0, f"w={w} -> none lse")
    out, lse = orc.attention(q, k, v, scale=scale, mask="causal")
    _close(out[0, 0, 0], v[0, 0, 0].astype(np.float64), 0.0, 0.0, "causal row 0")
    _close(lse[0, 0, 0], s_ii[0, 0, 0], 1e-15, 0.0, "causal row 0 lse")
    # the causal side of the band: w=0 keeps only the diagonal, w >= L-1 is causal
    out, lse = orc.attention(q, k, v, scale=scale, mask="causal_window", window=0)
    _close(out, v.astype(np.float64), 1e-15, 0.0, "causal w=0 -> V")
    _close(lse, s_ii, 1e-14, 1e-15, "causal w=0 -> lse = s_ii")
    ref_c = orc.attention(q, k, v, scale=scale, mask="causal")
    for w in (L - 1, L, 10 * L):
        got = orc.attention(q, k, v, scale=scale, mask="causal_window", window=w)
        _close(got[0], ref_c[0], 0.0, 0.0, f"causal w={w} -> causal")
        _close(got[1], ref_c[1], 0.0, 0.0, f"causal w={w} -> causal lse")
    zq = np.zeros_like(q)
    for mask, window in (("none", 0), ("causal", 0), ("window", 3), ("causal_window", 4)):
        out, lse = orc.attention(zq, k, v, scale=scale, mask=mask, window=window)
        M = np.array(dense_mask(L, mask, window), bool)
        for i in range(L):
            _close(out[0, 0, i], v[0, 0][M[i]].astype(np.float64).mean(0), 1e-13, 1e-14,
                   f"Q=0 mean {mask} {i}")
            assert abs(lse[0, 0, i] - math.log(M[i].sum())) <= 1e-14
    perm = np.random.default_rng(21).permutation(L)
    got = orc.attention(q, k[:, :, perm], v[:, :, perm], scale=scale, mask="none")
    _close(got[0], ref[0], 1e-13, 1e-14, "permutation")
    _close(got[1], ref[1], 1e-13, 1e-14, "permutation lse")
    # heads and batches are independent
    B, H = 2, 3
    q3, k3, v3 = _rand((B, H, L, d), 22), _rand((B, H, L, d), 23), _rand((B, H, L, d), 24)
    full = orc.attention(q3, k3, v3, scale=scale, mask="causal")
    for b in range(B):
        for h in range(H):
            one = orc.attention(q3[b:b + 1, h:h + 1], k3[b:b + 1, h:h + 1],
                                v3[b:b + 1, h:h + 1], scale=scale, mask="causal")
            _close(full[0][b, h], one[0][0, 0], 0.0, 0.0, "head independence")
            _close(full[1][b, h], one[1][0, 0], 0.0, 0.0, "head independence lse")


def pin_overflow(orc):
    """[MOSAIC 5.1]: logits scaled far up (Q x8, x64, x1000) stay finite, the
    probability rows still sum to 1 and outputs stay inside the hull of V."""
    L, d = 64, 64
    k, v = _rand((1, 2, L, d), 25), _rand((1, 2, L, d), 26)
    for mult in (8.0, 64.0, 1000.0):
        q = _rand((1, 2, L, d), 27, mult)
        for mask, window in (("none", 0), ("causal", 0), ("window", 9), ("causal_window", 9)):
            out, lse = orc.attention(q, k, v, mask=mask, window=window)
            assert np.isfinite(out).all() and np.isfinite(lse).all(), (mult, mask)
            M = np.array(dense_mask(L, mask, window), bool)
            for i in range(L):
                sel = v[0, :, M[i]].astype(np.float64)  # [n, H, d] after fancy indexing
                lo, hi = sel.min(0), sel.max(0)
                assert (out[0, :, i] >= lo - 1e-12).all() and (out[0, :, i] <= hi + 1e-12).all()
        P, lse = _probabilities(orc, q[..., :8], k[..., :8], 1.0, "causal", 0)
        assert np.isfinite(P).all() and np.isfinite(lse).all()
        assert np.abs(P.sum(-1) - 1.0).max() <= 1e-13, mult


def pin_rows_match(orc):
    """The selected-rows call returns the same rows as the whole-problem call."""
    B, H, L, d = 1, 3, 70, 8
    q, k, v = _rand((B, H, L, d), 28), _rand((B, H, L, d), 29), _rand((B, H, L, d), 30)
    for mask, window in (("none", 0), ("causal", 0), ("window", 11), ("causal_window", 11)):
        full_o, full_l = orc.attention(q, k, v, mask=mask, window=window)
        bh = [0, 0, 1, 2, 2, 2]
        rows = [0, 69, 5, 0, 34, 69]
        o, l = orc.attention_rows(q, k, v, bh, rows, mask=mask, window=window)
        for n, (b_h, r) in enumerate(zip(bh, rows)):
            _close(o[n], full_o[0, b_h, r], 0.0, 0.0, "rows vs full")
            assert l[n] == full_l[0, b_h, r]


def pin_partials_merge_to_definition(orc):
    """[MOSAIC 2.1]: partial results over disjoint key ranges combine into the
    whole: LSE = ln sum_s e^LSE_s and O = sum_s e^(LSE_s - LSE) O_s.  Ranges
    that hold no allowed key of a row give LSE_s = -inf (weight 0)."""
    L, d = 45, 6
    q, k, v = _rand((1, 2, L, d), 31), _rand((1, 2, L, d), 32), _rand((1, 2, L, d), 33)
    for mask, window in (("none", 0), ("causal", 0), ("window", 4), ("causal_window", 9)):
        full_o, full_l = orc.attention(q, k, v, mask=mask, window=window)
        for bounds in ([0, 45], [0, 20, 45], [0, 1, 2, 44, 45], [0, 7, 14, 21, 28, 35, 45]):
            parts = [orc.attention_partial(q, k, v, a, b, mask=mask, window=window)
                     for a, b in zip(bounds[:-1], bounds[1:])]
            lses = np.stack([p[1] for p in parts])
            mx = lses.max(0)
            w = np.exp(lses - mx)
            lse = mx + np.log(w.sum(0))
            o = sum(np.exp(p[1] - lse)[..., None] * p[0] for p in parts)
            _close(lse, full_l, 1e-13, 1e-13, f"merged lse {mask} {bounds}")
            _close(o, full_o, 1e-13, 1e-13, f"merged out {mask} {bounds}")
    # an empty range is all -inf / 0
    o, l = orc.attention_partial(q, k, v, 10, 10, mask="causal")
    assert np.isneginf(l).all() and (o == 0).all()
    # causal: row 3 has no allowed key in [20, 45)
    o, l = orc.attention_partial(q, k, v, 20, 45, mask="causal")
    assert np.isneginf(l[0, :, 3]).all() and (o[0, :, 3] == 0).all()


ALL_PINS = [pin_brute_force, pin_golden, pin_kv_blockwise, pin_q_blockwise,
            pin_probability_rows, pin_identical_keys, pin_constant_v, pin_special_cases,
            pin_overflow, pin_rows_match, pin_partials_merge_to_definition]


# --------------------------------------------------------------------------
# the multi-head attention layer [MHA-CUDA 2.1, 2.2]
# --------------------------------------------------------------------------
def brute_force_mha(x, w_qkv, b_qkv, w_out, b_out, H, mask, window):
    """The page's layer with plain Python loops, one step per line of its
    forward: Linear(E, 3E), chunk into q, k, v, split heads, masked softmax
    attention with 1/sqrt(d), merge heads, Linear(E, E)."""
    B, L, E = len(x), len(x[0]), len(x[0][0])
    d = E // H
    M = dense_mask(L, mask, window)

    def linear(rows, W, b):
        return [[math.fsum([rows[r][c] * W[j][c] for c in range(len(rows[0]))])
                 + (b[j] if b is not None else 0.0) for j in range(len(W))]
                for r in range(len(rows))]

    y = []
    for bb in range(B):
        qkv = linear(x[bb], w_qkv, b_qkv)
        q = [row[0:E] for row in qkv]
        k = [row[E:2 * E] for row in qkv]
        v = [row[2 * E:3 * E] for row in qkv]
        ctx = [[0.0] * E for _ in range(L)]
        for h in range(H):
            cols = range(h * d, (h + 1) * d)
            for i in range(L):
                e = [math.exp(math.fsum([q[i][c] * k[j][c] for c in cols]) / math.sqrt(d))
                     if M[i][j] else 0.0 for j in range(L)]
                Z = math.fsum(e)
                for c in cols:
                    ctx[i][c] = math.fsum([e[j] * v[j][c] for j in range(L)]) / Z
        y.append(linear(ctx, w_out, b_out))
    return y


def pin_mha_brute_force(orc):
    """The layer against the pure-Python restatement of the page's forward."""
    rng = np.random.default_rng(40)
    for (B, L, E, H), (mask, window) in (((1, 4, 4, 2), ("none", 0)), ((2, 5, 6, 3), ("causal", 0)),
                                         ((1, 6, 4, 1), ("window", 1)),
                                         ((1, 5, 8, 2), ("causal_window", 2))):
        x = rng.standard_normal((B, L, E)).astype(np.float32)
        w_qkv = (rng.standard_normal((3 * E, E)) * 0.5).astype(np.float32)
        b_qkv = rng.standard_normal(3 * E).astype(np.float32)
        w_out = (rng.standard_normal((E, E)) * 0.5).astype(np.float32)
        b_out = rng.standard_normal(E).astype(np.float32)
        y = orc.mha(x, w_qkv, b_qkv, w_out, b_out, H, mask=mask, window=window)
        ref = brute_force_mha(x.tolist(), w_qkv.tolist(), b_qkv.tolist(), w_out.tolist(),
                              b_out.tolist(), H, mask, window)
        _close(y, ref, 1e-12, 1e-12, f"mha brute force {B, L, E, H} {mask}")
        y0 = orc.mha(x, w_qkv, None, w_out, None, H, mask=mask, window=window)
        ref0 = brute_force_mha(x.tolist(), w_qkv.tolist(), None, w_out.tolist(), None, H, mask,
                               window)
        _close(y0, ref0, 1e-12, 1e-12, f"mha brute force, no biases {mask}")


def pin_mha_identity_projections(orc):
    """With W_qkv = [I; I; I], W_out = I and zero biases the layer is the
    attention of x split into heads, merged back (checked against the pinned
    attention functions)."""
    B, L, E, H = 2, 30, 12, 3
    d = E // H
    x = _rand((B, L, E), 41)
    eye = np.eye(E, dtype=np.float32)
    y = orc.mha(x, np.concatenate([eye, eye, eye]), None, eye, None, H, mask="causal")
    heads = x.reshape(B, L, H, d).transpose(0, 2, 1, 3).copy()
    o, _ = orc.attention(heads, heads, heads, scale=1.0 / math.sqrt(d), mask="causal")
    _close(y, o.transpose(0, 2, 1, 3).reshape(B, L, E), 1e-13, 1e-13, "identity projections")


ALL_PINS += [pin_mha_brute_force, pin_mha_identity_projections]


# --------------------------------------------------------------------------
# backward by recomputation [LONGSEQ 3.1], [MOSAIC 2.2]
# --------------------------------------------------------------------------
def _grid_values(shape, seed):
    """Values k / 64, |k| <= 64: x +- 2^-12 is exact in fp32, so central
    differences see exactly the perturbation they intend."""
    rng = np.random.default_rng(seed)
    return (rng.integers(-64, 65, size=shape) / 64.0).astype(np.float32)


def pin_backward_finite_differences(orc):
    """dQ, dK, dV against central differences of the (pinned) forward:
    f = sum(G * O), df/dx ~ (f(x + e) - f(x - e)) / 2e with e = 2^-12."""
    B, H, L, d = 1, 1, 5, 3
    eps = 2.0 ** -12
    for mask, window in (("none", 0), ("causal", 0), ("window", 1), ("causal_window", 2)):
        q, k, v, g = (_grid_values((B, H, L, d), s) for s in (50, 51, 52, 53))
        scale = 0.7
        dq, dk, dv = orc.attention_backward(q, k, v, g, scale=scale, mask=mask, window=window)

        def f(q_, k_, v_):
            o, _ = orc.attention(q_, k_, v_, scale=scale, mask=mask, window=window)
            return math.fsum((o * g.astype(np.float64)).ravel().tolist())

        for name, arr, grad in (("dq", q, dq), ("dk", k, dk), ("dv", v, dv)):
            num = np.zeros_like(grad)
            for idx in np.ndindex(arr.shape):
                up, dn = arr.copy(), arr.copy()
                up[idx] += eps
                dn[idx] -= eps
                args_up = [q, k, v]
                args_dn = [q, k, v]
                pos = {"dq": 0, "dk": 1, "dv": 2}[name]
                args_up[pos], args_dn[pos] = up, dn
                num[idx] = (f(*args_up) - f(*args_dn)) / (2 * eps)
            _close(grad, num, 1e-5, 1e-6, f"finite differences {name} {mask}")


def pin_backward_invariants(orc):
    """Constant V: the output ignores Q and K, so dQ = dK = 0.  A common shift
    of every key leaves each row's softmax unchanged, so sum_j dK_j = 0.
    Rows of P sum to 1, so sum_j dV_j = sum_i dO_i."""
    B, H, L, d = 2, 2, 37, 8
    q, k, g = _rand((B, H, L, d), 54), _rand((B, H, L, d), 55), _rand((B, H, L, d), 56)
    for mask, window in (("none", 0), ("causal", 0), ("window", 5), ("causal_window", 7)):
        c = np.broadcast_to(_rand((B, H, 1, d), 57), (B, H, L, d)).copy()
        dq, dk, _ = orc.attention_backward(q, k, c, g, mask=mask, window=window)
        assert np.abs(dq).max() <= 1e-13 and np.abs(dk).max() <= 1e-13, mask
        v = _rand((B, H, L, d), 58)
        dq, dk, dv = orc.attention_backward(q, k, v, g, mask=mask, window=window)
        assert np.abs(dk.sum(axis=2)).max() <= 1e-12, mask
        _close(dv.sum(axis=2), g.astype(np.float64).sum(axis=2), 1e-12, 1e-12,
               f"sum dV = sum dO {mask}")


ALL_PINS += [pin_backward_finite_differences, pin_backward_invariants]
