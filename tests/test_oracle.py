"""Pins for the float64 oracle, each against something other than the oracle.

Every check here is a closed form, an invariant of the definition, a hand-
worked value, brute force, finite differences, or an independent library
routine (torch's float64 CPU SDPA with autograd).  A dropped term, a wrong
sign, a wrong index or a transposed operand in the oracle fails at least one.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import (alibi_slope_gradient, attention_backward, attention_forward,
                    attention_probs, dense_bias_gradient, fire_gradients, fire_table,
                    head_scores, rel_table_gradient, t5_relative_bucket, t5_table_gradient,
                    visibility_mask)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def qkv(B=2, L=12, Hq=4, Hkv=2, d=8, seed=0):
    return (rnd((B, L, Hq, d), seed), rnd((B, L, Hkv, d), seed + 1),
            rnd((B, L, Hkv, d), seed + 2), rnd((B, L, Hq, d), seed + 3))


# ---------------------------------------------------------------- buckets
def test_t5_buckets_hand_worked():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "t5_buckets.txt"))
            if l.strip() and not l.startswith("#")]
    rel = np.array([int(r[0]) for r in rows])
    want = np.array([int(r[1]) for r in rows])
    got = t5_relative_bucket(rel, 32, 128, True)
    assert np.array_equal(got, want), list(zip(rel, got, want))


def test_t5_buckets_integer_thresholds():
    # The log-form boundaries for (32, 128) are n = 8,12,16,23,32,46,64,91
    # (solve 8*16^(k/8) for k = 0..7 and round up): every n in [0, 5000].
    thr = [8, 12, 16, 23, 32, 46, 64, 91]
    n = np.arange(0, 5001)
    want = np.where(n < 8, n, 7 + np.searchsorted(thr, n, side="right"))
    want = np.minimum(want, 15)
    assert np.array_equal(t5_relative_bucket(-n, 32, 128, True), want)
    want_pos = np.where(n > 0, want + 16, 0)
    assert np.array_equal(t5_relative_bucket(n, 32, 128, True), want_pos)


def _golden_sections(name):
    """{(num_buckets, max_distance, bidirectional): (rel, bucket)} of a golden file."""
    out, cur = {}, None
    for line in open(os.path.join(GOLDEN, name)):
        f = line.split()
        if not f or f[0].startswith("#"):
            continue
        if f[0] == "config":
            cur = (int(f[1]), int(f[2]), bool(int(f[3])))
            out[cur] = ([], [])
            continue
        out[cur][0].append(int(f[0]))
        out[cur][1].append(int(f[1]))
    return out


def test_t5_buckets_other_settings_hand_worked():
    # The decoder (unidirectional) form and the non-default bucket settings
    # the GPU bucket test uses, against thresholds solved by hand: both sides
    # of every threshold of the 32-bucket decoder table, keys after the query
    # (bucket 0), the caps, and the exact-tie distances 32, 64, 128 of the
    # (64, 256) table.
    secs = _golden_sections("t5_buckets_more.txt")
    assert set(secs) == {(32, 128, False), (16, 40, True), (64, 256, True), (8, 20, True),
                         (128, 1000, False)}
    for (nb, md, bidir), (rel, want) in secs.items():
        got = t5_relative_bucket(np.array(rel), nb, md, bidir)
        assert np.array_equal(got, np.array(want)), \
            [(r, g, w) for r, g, w in zip(rel, got, want) if g != w]


def test_t5_buckets_decoder_thresholds_every_distance():
    # 32 decoder buckets: the hand-solved first distance of each log bucket
    # (16 * 8^(k/16) rounded up), checked for every n in [0, 5000]; every key
    # after the query is bucket 0.
    thr = [16, 19, 21, 24, 27, 31, 35, 40, 46, 52, 59, 67, 77, 87, 99, 113]
    n = np.arange(0, 5001)
    want = np.where(n < 16, n, 15 + np.searchsorted(thr, n, side="right"))
    want = np.minimum(want, 31)
    assert np.array_equal(t5_relative_bucket(-n, 32, 128, False), want)
    assert (t5_relative_bucket(np.arange(1, 3000), 32, 128, False) == 0).all()


# ---------------------------------------------------------------- masks
def test_mask_brute_force():
    L = 9
    for causal in (False, True):
        for wl in (-1, 0, 2, 8):
            for wr in (-1, 0, 3):
                m = visibility_mask(L, causal, wl, wr)
                for i in range(L):
                    for j in range(L):
                        ok = (not causal or j <= i) and (wl < 0 or j >= i - wl) \
                            and (wr < 0 or j <= i + wr)
                        assert m[i, j] == ok


# ---------------------------------------------------------------- softmax
@pytest.mark.parametrize("causal,wl", [(False, -1), (True, -1), (True, 3)])
def test_probability_rows_sum_to_one(causal, wl):
    q, k, _, _ = qkv()
    for b in range(2):
        for hq in range(4):
            P = attention_probs(q, k, b, hq, causal=causal, window_left=wl)
            assert np.allclose(P.sum(1), 1.0, atol=1e-13)
            assert (P >= 0).all()
            M = visibility_mask(12, causal, wl)
            assert (P[~M] == 0).all()


def test_row_constant_bias_is_invariant():
    q, k, v, do = qkv()
    B, L, Hq = 2, 12, 4
    c = rnd((B, Hq, L, 1), 7) * np.ones((1, 1, 1, L))
    O0, _ = attention_forward(q, k, v, causal=True)
    O1, _ = attention_forward(q, k, v, causal=True, bias=c)
    g0 = attention_backward(q, k, v, do, causal=True)
    g1 = attention_backward(q, k, v, do, causal=True, bias=c)
    assert np.allclose(O0, O1, atol=1e-12)
    for a, b_ in zip(g0, g1):
        assert np.allclose(a, b_, atol=1e-11)


# ---------------------------------------------------------------- causal
def test_causal_first_and_last_rows():
    # codelab section 7: the first query sees only itself, the last sees all.
    q, k, v, _ = qkv()
    Oc, _ = attention_forward(q, k, v, causal=True)
    Of, _ = attention_forward(q, k, v, causal=False)
    G = 2
    for hq in range(4):
        assert np.array_equal(Oc[:, 0, hq], v[:, 0, hq // G])
    assert np.allclose(Oc[:, -1], Of[:, -1], atol=1e-14)
    assert not np.allclose(Oc[:, 0], Of[:, 0], atol=1e-3)


def test_lower_triangular_dense_bias_equals_causal():
    q, k, v, do = qkv()
    L = 12
    tri = np.where(np.tril(np.ones((L, L), bool)), 0.0, -np.inf)[None, None]
    Oc, Lc = attention_forward(q, k, v, causal=True)
    Ob, Lb = attention_forward(q, k, v, causal=False, bias=tri)
    assert np.allclose(Oc, Ob, atol=1e-14) and np.allclose(Lc, Lb, atol=1e-14)
    gc = attention_backward(q, k, v, do, causal=True)
    gb = attention_backward(q, k, v, do, causal=False, bias=tri)
    for a, b_ in zip(gc, gb):
        assert np.allclose(a, b_, atol=1e-13)


# ---------------------------------------------------------------- window
def test_window_at_least_L_minus_1_equals_causal():
    q, k, v, do = qkv()
    Oc, Lc = attention_forward(q, k, v, causal=True)
    for wl in (11, 12, 4096):
        Ow, Lw = attention_forward(q, k, v, causal=True, window_left=wl)
        assert np.array_equal(Oc, Ow) and np.array_equal(Lc, Lw)
    Ow, _ = attention_forward(q, k, v, causal=True, window_left=10)
    assert not np.allclose(Oc, Ow)   # wl = L-2 drops key 0 from the last row


def test_window_zero_closed_form():
    # Each query sees only its own key: O = V_g, dQ = dK = 0, dV = group sum of dO.
    q, k, v, do = qkv()
    O, LSE = attention_forward(q, k, v, causal=True, window_left=0)
    dq, dk, dv = attention_backward(q, k, v, do, causal=True, window_left=0)
    G = 2
    for hq in range(4):
        assert np.allclose(O[:, :, hq], v[:, :, hq // G], atol=1e-15)
        s = np.einsum("bld,bld->bl", q[:, :, hq], k[:, :, hq // G]) / math.sqrt(8)
        assert np.allclose(LSE[:, hq], s, atol=1e-13)
    assert np.allclose(dq, 0, atol=1e-15) and np.allclose(dk, 0, atol=1e-15)
    want = do.reshape(2, 12, 2, G, 8).sum(3)
    assert np.allclose(dv, want, atol=1e-13)


# ---------------------------------------------------------------- closed forms
def test_zero_q_gives_mean_of_visible_values():
    _, k, v, _ = qkv()
    q = np.zeros((2, 12, 4, 8))
    O, LSE = attention_forward(q, k, v, causal=True, window_left=3)
    M = visibility_mask(12, True, 3)
    n = M.sum(1)
    for hq in range(4):
        want = np.einsum("ij,bjd->bid", M / n[:, None], v[:, :, hq // 2])
        assert np.allclose(O[:, :, hq], want, atol=1e-14)
        assert np.allclose(LSE[:, hq], np.log(n)[None], atol=1e-14)


def test_constant_v_and_single_key():
    q, k, _, _ = qkv()
    v = np.full((2, 12, 2, 8), 3.25)
    O, _ = attention_forward(q, k, v, causal=False)
    assert np.allclose(O, 3.25, atol=1e-14)
    q1, k1, v1, _ = qkv(L=1)
    O1, L1 = attention_forward(q1, k1, v1)
    for hq in range(4):
        assert np.array_equal(O1[:, 0, hq], v1[:, 0, hq // 2])
        s = (q1[:, 0, hq] * k1[:, 0, hq // 2]).sum(-1) / math.sqrt(8)
        assert np.allclose(L1[:, hq, 0], s, atol=1e-14)


def test_fully_masked_row_is_zero():
    q, k, v, do = qkv()
    bias = np.zeros((1, 1, 12, 12))
    bias[..., 5, :] = -np.inf
    O, LSE = attention_forward(q, k, v, bias=bias)
    assert (O[:, 5] == 0).all() and np.isneginf(LSE[:, :, 5]).all()
    dq, dk, dv = attention_backward(q, k, v, do, bias=bias)
    assert (dq[:, 5] == 0).all()
    assert np.isfinite(dk).all() and np.isfinite(dv).all()


# ---------------------------------------------------------------- GQA / MQA
@pytest.mark.parametrize("Hkv", [1, 2, 4])
def test_gqa_equals_mha_with_repeated_kv(Hkv):
    q, k, v, do = qkv(Hkv=Hkv)
    G = 4 // Hkv
    kr, vr = np.repeat(k, G, axis=2), np.repeat(v, G, axis=2)
    O, LSE = attention_forward(q, k, v, causal=True)
    Or, LSEr = attention_forward(q, kr, vr, causal=True)
    assert np.array_equal(O, Or) and np.array_equal(LSE, LSEr)
    dq, dk, dv = attention_backward(q, k, v, do, causal=True)
    dqr, dkr, dvr = attention_backward(q, kr, vr, do, causal=True)
    assert np.allclose(dq, dqr, atol=1e-14)
    assert np.allclose(dk, dkr.reshape(2, 12, Hkv, G, 8).sum(3), atol=1e-13)
    assert np.allclose(dv, dvr.reshape(2, 12, Hkv, G, 8).sum(3), atol=1e-13)


def test_row_subset_matches_full():
    q, k, v, _ = qkv(L=20)
    table = rnd((32, 4), 2)
    O, LSE = attention_forward(q, k, v, causal=True, window_left=6, t5_table=table)
    rows = [0, 3, 19, 7]
    Os, LSEs = attention_forward(q, k, v, causal=True, window_left=6, t5_table=table,
                                 query_rows=rows, batches=[1])
    assert np.array_equal(Os[1, rows], O[1, rows]) and np.array_equal(LSEs[1][:, rows], LSE[1][:, rows])
    assert np.isnan(Os[1, 1]).all() and np.isnan(Os[0]).all()


def test_subset_matches_full():
    q, k, v, do = qkv()
    O, LSE = attention_forward(q, k, v, causal=True)
    Os, LSEs = attention_forward(q, k, v, causal=True, batches=[1], kv_heads=[0])
    assert np.array_equal(Os[1, :, :2], O[1, :, :2]) and np.isnan(Os[0]).all()
    g = attention_backward(q, k, v, do, causal=True)
    gs = attention_backward(q, k, v, do, causal=True, batches=[1], kv_heads=[0])
    assert np.array_equal(gs[0][1, :, :2], g[0][1, :, :2])
    assert np.array_equal(gs[1][1, :, 0], g[1][1, :, 0])


# ---------------------------------------------------------------- biases
def test_constant_t5_table_is_no_bias():
    q, k, v, do = qkv()
    table = np.tile(rnd((1, 4), 3), (32, 1))      # constant per head
    O0, _ = attention_forward(q, k, v)
    O1, _ = attention_forward(q, k, v, t5_table=table)
    assert np.allclose(O0, O1, atol=1e-13)


def test_dense_bias_equals_expanded_t5_bias():
    q, k, v, do = qkv(L=40)
    table = rnd((32, 4), 5)
    L = 40
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    # expand by brute force with the hand-worked threshold rule
    thr = [8, 12, 16, 23, 32, 46, 64, 91]
    dense = np.zeros((1, 4, L, L))
    for a in range(L):
        for c in range(L):
            r = c - a
            n = abs(r)
            bk = n if n < 8 else min(7 + sum(n >= t for t in thr), 15)
            bk += 16 if r > 0 else 0
            dense[0, :, a, c] = table[bk, :]
    O1, L1 = attention_forward(q, k, v, t5_table=table)
    O2, L2 = attention_forward(q, k, v, bias=dense)
    assert np.allclose(O1, O2, atol=1e-14) and np.allclose(L1, L2, atol=1e-14)
    g1 = attention_backward(q, k, v, do, t5_table=table)
    g2 = attention_backward(q, k, v, do, bias=dense)
    for a, b_ in zip(g1, g2):
        assert np.allclose(a, b_, atol=1e-13)


# ---------------------------------------------------------------- gradients
def _loss(q, k, v, do, kw):
    O, _ = attention_forward(q, k, v, **kw)
    return float(np.sum(O * do))


@pytest.mark.parametrize("kw", [
    dict(causal=True),
    dict(causal=True, window_left=2),
    dict(causal=False, window_left=1, window_right=3),
    dict(causal=False, t5_table="t5"),
    dict(causal=False, bias="dense"),
])
def test_gradients_central_differences(kw):
    B, L, Hq, Hkv, d = 1, 6, 4, 2, 3
    q, k, v, do = qkv(B, L, Hq, Hkv, d, seed=11)
    kw = dict(kw)
    if kw.get("t5_table") == "t5":
        kw["t5_table"] = rnd((32, Hq), 4)
    if kw.get("bias") == "dense":
        kw["bias"] = rnd((B, Hq, L, L), 4)
    dq, dk, dv = attention_backward(q, k, v, do, **kw)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = x.copy(); xp[idx] += h
            xm = x.copy(); xm[idx] -= h
            args = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            argm = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            num[idx] = (_loss(*args, do, kw) - _loss(*argm, do, kw)) / (2 * h)
        err = np.max(np.abs(num - g)) / max(1.0, np.max(np.abs(g)))
        assert err < 1e-6, (name, err)


def test_dense_bias_gradient_central_differences():
    B, L, Hq, Hkv, d = 1, 5, 2, 1, 3
    q, k, v, do = qkv(B, L, Hq, Hkv, d, seed=21)
    bias = rnd((B, Hq, L, L), 9)
    *_, dB = attention_backward(q, k, v, do, causal=True, bias=bias, return_dbias=True)
    h = 1e-6
    M = visibility_mask(L, True)
    for hq in range(Hq):
        for i in range(L):
            for j in range(L):
                bp = bias.copy(); bp[0, hq, i, j] += h
                bm = bias.copy(); bm[0, hq, i, j] -= h
                num = (_loss(q, k, v, do, dict(causal=True, bias=bp))
                       - _loss(q, k, v, do, dict(causal=True, bias=bm))) / (2 * h)
                want = dB[0, hq, i, j] if M[i, j] else 0.0
                assert abs(num - want) < 1e-7


@pytest.mark.parametrize("bias_shape", [(1, 2, 5, 5), (2, 1, 5, 5), (1, 1, 5, 5),
                                        (2, 2, 1, 5), (1, 1, 1, 5)])
def test_broadcast_bias_gradient_central_differences(bias_shape):
    # A broadcast bias feeds every (b, h, i) it is broadcast over, so its
    # gradient is the sum of dS over those copies.
    B, L, Hq, Hkv, d = 2, 5, 2, 1, 3
    q, k, v, do = qkv(B, L, Hq, Hkv, d, seed=23)
    bias = rnd(bias_shape, 10)
    kw = dict(causal=False, window_left=3, window_right=1, bias=bias)
    *_, dS = attention_backward(q, k, v, do, return_dbias=True, **kw)
    g = dense_bias_gradient(dS, bias_shape)
    assert g.shape == bias_shape
    h = 1e-6
    it = np.nditer(bias, flags=["multi_index"])
    for _ in it:
        idx = it.multi_index
        bp = bias.copy(); bp[idx] += h
        bm = bias.copy(); bm[idx] -= h
        num = (_loss(q, k, v, do, {**kw, "bias": bp})
               - _loss(q, k, v, do, {**kw, "bias": bm})) / (2 * h)
        assert abs(num - g[idx]) < 1e-7, (idx, num, g[idx])


@pytest.mark.parametrize("bidirectional,causal", [(True, False), (True, True), (False, True),
                                                  (False, False)])
def test_t5_table_gradient_central_differences(bidirectional, causal):
    # 8 buckets over distances up to 11 with max_distance 6: exact, log-wide
    # and clamped buckets all occur, on both sides when bidirectional.
    B, L, Hq, Hkv, d = 2, 12, 2, 2, 3
    nb, md = 8, 6
    q, k, v, do = qkv(B, L, Hq, Hkv, d, seed=31)
    table = rnd((nb, Hq), 12)
    kw = dict(causal=causal, t5_table=table, t5_num_buckets=nb, t5_max_distance=md,
              t5_bidirectional=bidirectional)
    *_, dS = attention_backward(q, k, v, do, return_dbias=True, **kw)
    g = t5_table_gradient(dS, nb, md, bidirectional)
    h = 1e-6
    for kb in range(nb):
        for hq in range(Hq):
            tp = table.copy(); tp[kb, hq] += h
            tm = table.copy(); tm[kb, hq] -= h
            num = (_loss(q, k, v, do, {**kw, "t5_table": tp})
                   - _loss(q, k, v, do, {**kw, "t5_table": tm})) / (2 * h)
            assert abs(num - g[kb, hq]) < 1e-7, (kb, hq, num, g[kb, hq])
    # softmax rows sum to one, so each row of dS sums to zero, and so do the
    # table gradient's columns (every (i, j) lands in exactly one bucket)
    assert np.allclose(g.sum(axis=0), 0.0, atol=1e-12)


@pytest.mark.parametrize("bidirectional", [True, False])
def test_every_t5_bucket_is_one_range_of_distances(bidirectional):
    # The T5 table gradient adds up per-diagonal sums over one contiguous
    # range of r = j - i per bucket; that needs the bucket to be monotone in
    # |r| on each side of 0 with disjoint ids across the sides.
    L = 3000
    r = np.arange(-(L - 1), L)
    for nb in (4, 8, 16, 32, 64, 128):
        for md in (nb, 2 * nb, 128, 1000, 5000):
            if md <= (nb // 2 if bidirectional else nb) // 2:
                continue
            b = t5_relative_bucket(r, nb, md, bidirectional)
            for k in np.unique(b):
                idx = np.nonzero(b == k)[0]
                assert idx[-1] - idx[0] + 1 == idx.size, (nb, md, k)


# ---------------------------------------------------------------- ALiBi
def test_alibi_zero_slopes_is_no_bias():
    q, k, v, do = qkv(1, 9, 2, 1, 4, seed=41)
    a = attention_forward(q, k, v, causal=True, alibi_slopes=np.zeros(2))
    b = attention_forward(q, k, v, causal=True)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_causal_alibi_is_a_key_position_bias():
    # Softmax ignores a constant added to a whole row, and under a causal
    # mask -m (i - j) = m j - m i: causal ALiBi must equal the bias m j, with
    # LSE lower by m i.  A sign error or a dropped |.| breaks this.
    B, L, Hq, Hkv, d = 2, 11, 3, 1, 5
    q, k, v, do = qkv(B, L, Hq, Hkv, d, seed=43)
    m = np.array([0.5, 0.25, 0.125])
    O1, lse1 = attention_forward(q, k, v, causal=True, alibi_slopes=m)
    keybias = m[None, :, None, None] * np.arange(L)[None, None, None, :] * np.ones((1, Hq, L, L))
    O2, lse2 = attention_forward(q, k, v, causal=True, bias=keybias)
    assert np.allclose(O1, O2, atol=1e-12)
    shift = m[None, :, None] * np.arange(L)[None, None, :]
    assert np.allclose(lse1, lse2 - shift, atol=1e-12)


def test_bidirectional_alibi_is_symmetric_under_reversal():
    # |j - i| is unchanged when both positions are mirrored, so reversing the
    # sequence reverses the outputs; a one-sided (j - i) form would not.
    B, L, Hq, Hkv, d = 1, 10, 2, 2, 4
    q, k, v, do = qkv(B, L, Hq, Hkv, d, seed=47)
    m = np.array([0.7, 0.3])
    O, lse = attention_forward(q, k, v, alibi_slopes=m)
    Or, lser = attention_forward(q[:, ::-1], k[:, ::-1], v[:, ::-1], alibi_slopes=m)
    assert np.allclose(O, Or[:, ::-1], atol=1e-12)
    assert np.allclose(lse, lser[:, :, ::-1], atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_alibi_slope_gradient_central_differences(causal):
    B, L, Hq, Hkv, d = 2, 8, 2, 1, 3
    q, k, v, do = qkv(B, L, Hq, Hkv, d, seed=53)
    m = np.array([0.6, 0.2])
    kw = dict(causal=causal, alibi_slopes=m)
    dq, dk, dv, dS = attention_backward(q, k, v, do, return_dbias=True, **kw)
    g = alibi_slope_gradient(dS)
    h = 1e-6
    for hq in range(Hq):
        mp = m.copy(); mp[hq] += h
        mm = m.copy(); mm[hq] -= h
        num = (_loss(q, k, v, do, {**kw, "alibi_slopes": mp})
               - _loss(q, k, v, do, {**kw, "alibi_slopes": mm})) / (2 * h)
        assert abs(num - g[hq]) < 1e-7, (hq, num, g[hq])
    # and dQ / dK / dV through the ALiBi bias, as for the other biases
    for name, x, gx in (("q", q, dq), ("k", k, dk)):
        idx = (1, 3, 1 if name == "q" else 0, 2)
        xp = x.copy(); xp[idx] += h
        xm = x.copy(); xm[idx] -= h
        args = (xp, k, v) if name == "q" else (q, xp, v)
        argm = (xm, k, v) if name == "q" else (q, xm, v)
        num = (_loss(*args, do, kw) - _loss(*argm, do, kw)) / (2 * h)
        assert abs(num - gx[idx]) < 1e-7


# ------------------------------------------------- cross-attention (Lk != L)
def test_cross_attention_single_query_brute_force():
    # one query row over 7 keys of another sequence, summed term by term
    rng = np.random.default_rng(61)
    q = rng.standard_normal((1, 1, 2, 3))
    k = rng.standard_normal((1, 7, 1, 3))
    v = rng.standard_normal((1, 7, 1, 4))
    bias = rng.standard_normal((1, 2, 1, 7))
    O, lse = attention_forward(q, k, v, bias=bias)
    for h in range(2):
        s = [sum(q[0, 0, h, c] * k[0, j, 0, c] for c in range(3)) / math.sqrt(3)
             + bias[0, h, 0, j] for j in range(7)]
        w = [math.exp(x) for x in s]
        z = sum(w)
        assert abs(lse[0, h, 0] - math.log(z)) < 1e-12
        for c in range(4):
            assert abs(O[0, 0, h, c] - sum(w[j] * v[0, j, 0, c] for j in range(7)) / z) < 1e-12


def test_cross_attention_key_permutation():
    # permuting keys, values and the bias's key axis together leaves O and
    # LSE unchanged; a bias read along the wrong axis would not follow
    rng = np.random.default_rng(67)
    q = rng.standard_normal((2, 5, 2, 4))
    k = rng.standard_normal((2, 9, 1, 4))
    v = rng.standard_normal((2, 9, 1, 4))
    bias = rng.standard_normal((2, 2, 5, 9))
    perm = rng.permutation(9)
    O, lse = attention_forward(q, k, v, bias=bias)
    Op, lsep = attention_forward(q, k[:, perm], v[:, perm], bias=bias[..., perm])
    assert np.allclose(O, Op, atol=1e-12) and np.allclose(lse, lsep, atol=1e-12)


@pytest.mark.parametrize("kw", [dict(), dict(bias="dense"), dict(t5="t5"),
                                dict(window_left=2, window_right=3)])
def test_cross_attention_gradients_central_differences(kw):
    B, Lq, Lk, Hq, Hkv, d = 1, 4, 7, 2, 1, 3
    rng = np.random.default_rng(71)
    q = rng.standard_normal((B, Lq, Hq, d))
    k = rng.standard_normal((B, Lk, Hkv, d))
    v = rng.standard_normal((B, Lk, Hkv, d))
    do = rng.standard_normal((B, Lq, Hq, d))
    kw = dict(kw)
    if kw.pop("bias", None):
        kw["bias"] = rng.standard_normal((B, Hq, Lq, Lk))
    if kw.pop("t5", None):
        kw.update(t5_table=rng.standard_normal((8, Hq)), t5_num_buckets=8, t5_max_distance=6)
    dq, dk, dv, dS = attention_backward(q, k, v, do, return_dbias=True, **kw)
    assert dq.shape == q.shape and dk.shape == k.shape and dS.shape == (B, Hq, Lq, Lk)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = x.copy(); xp[idx] += h
            xm = x.copy(); xm[idx] -= h
            args = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            argm = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            num[idx] = (_loss(*args, do, kw) - _loss(*argm, do, kw)) / (2 * h)
        assert np.max(np.abs(num - g)) < 1e-6 * max(1.0, np.max(np.abs(g))), name
    if "bias" in kw:
        for idx in ((0, 0, 1, 5), (0, 1, 3, 0)):
            bp = kw["bias"].copy(); bp[idx] += h
            bm = kw["bias"].copy(); bm[idx] -= h
            num = (_loss(q, k, v, do, {**kw, "bias": bp})
                   - _loss(q, k, v, do, {**kw, "bias": bm})) / (2 * h)
            assert abs(num - dS[idx]) < 1e-7


def test_D_two_ways():
    # rowsum(P * dP) = rowsum(dO * O) for every row.
    q, k, v, do = qkv()
    O, _ = attention_forward(q, k, v, causal=True)
    for b in range(2):
        for hq in range(4):
            P = attention_probs(q, k, b, hq, causal=True)
            dP = do[b, :, hq] @ v[b, :, hq // 2].T
            assert np.allclose((P * dP).sum(1), (do[b, :, hq] * O[b, :, hq]).sum(1), atol=1e-13)


# ---------------------------------------------------------------- library
@pytest.mark.parametrize("causal,wl,wr,bias_kind,Hkv", [
    (False, -1, -1, None, 4), (True, -1, -1, None, 2), (True, 5, -1, None, 1),
    (False, 4, 2, None, 4), (False, -1, -1, "t5", 4), (True, -1, -1, "dense", 2),
])
def test_matches_torch_float64_sdpa(causal, wl, wr, bias_kind, Hkv):
    B, L, Hq, d = 2, 33, 4, 16
    q, k, v, do = qkv(B, L, Hq, Hkv, d, seed=3)
    kw = dict(causal=causal, window_left=wl, window_right=wr)
    add = np.where(visibility_mask(L, causal, wl, wr), 0.0, -np.inf)[None, None]
    if bias_kind == "t5":
        table = rnd((32, Hq), 8)
        kw["t5_table"] = table
        rel = np.arange(L)[None, :] - np.arange(L)[:, None]
        # torch side indexes the table with its own integer bucket rule
        thr = torch.tensor([8, 12, 16, 23, 32, 46, 64, 91])
        n = torch.from_numpy(np.abs(rel))
        bk = torch.where(n < 8, n, torch.clamp(7 + torch.bucketize(n, thr, right=True), max=15))
        bk = bk + torch.from_numpy((rel > 0).astype(np.int64)) * 16
        add = add + torch.from_numpy(table)[bk].permute(2, 0, 1).numpy()[None]
    elif bias_kind == "dense":
        bias = rnd((B, Hq, L, L), 8)
        kw["bias"] = bias
        add = add + bias
    G = Hq // Hkv
    tq = torch.tensor(q, requires_grad=True)
    tk = torch.tensor(k, requires_grad=True)
    tv = torch.tensor(v, requires_grad=True)
    kr = tk.repeat_interleave(G, dim=2)
    vr = tv.repeat_interleave(G, dim=2)
    out = torch.nn.functional.scaled_dot_product_attention(
        tq.transpose(1, 2), kr.transpose(1, 2), vr.transpose(1, 2),
        attn_mask=torch.tensor(np.broadcast_to(add, (B, Hq, L, L)).copy()))
    out = out.transpose(1, 2)
    out.backward(torch.tensor(do))
    O, LSE = attention_forward(q, k, v, **kw)
    dq, dk, dv = attention_backward(q, k, v, do, **kw)
    assert np.allclose(O, out.detach().numpy(), atol=1e-12)
    assert np.allclose(dq, tq.grad.numpy(), atol=1e-11)
    assert np.allclose(dk, tk.grad.numpy(), atol=1e-11)
    assert np.allclose(dv, tv.grad.numpy(), atol=1e-11)
    # LSE against torch's own logsumexp of the same scores
    s = torch.einsum("blhd,bmhd->bhlm", tq.detach(), kr.detach()) / math.sqrt(d)
    s = s + torch.tensor(add)
    assert np.allclose(LSE, torch.logsumexp(s, dim=-1).numpy(), atol=1e-12)


def test_head_scores_masked_entries():
    q, k, _, _ = qkv()
    S = head_scores(q, k, 0, 1, scale=0.5, causal=True)
    assert np.isneginf(S[0, 1:]).all()
    assert math.isclose(S[3, 2], 0.5 * float(q[0, 3, 1] @ k[0, 2, 0]), rel_tol=1e-14)


# ------------------------------------------------------ packed sequences
from oracle import (attention_backward_packed, attention_forward_packed,  # noqa: E402
                    packed_positions, packed_visibility_mask)


def _packed(lq, lk, Hq=4, Hkv=2, d=8, seed=0):
    cq = np.concatenate([[0], np.cumsum(lq)]).astype(int)
    ck = np.concatenate([[0], np.cumsum(lk)]).astype(int)
    q = rnd((cq[-1], Hq, d), seed)
    k = rnd((ck[-1], Hkv, d), seed + 1)
    v = rnd((ck[-1], Hkv, d), seed + 2)
    do = rnd((cq[-1], Hq, d), seed + 3)
    return cq, ck, q, k, v, do


def test_packed_mask_brute_force():
    cq, ck = [0, 3, 3, 7], [0, 2, 5, 9]
    for causal, wl, wr in ((False, -1, -1), (True, -1, -1), (True, 1, -1), (False, 0, 2)):
        m = packed_visibility_mask(cq, ck, causal, wl, wr)
        for r in range(7):
            for c in range(9):
                bq = max(b for b in range(3) if cq[b] <= r and r < cq[b + 1])
                bk = max(b for b in range(3) if ck[b] <= c and c < ck[b + 1])
                i, j = r - cq[bq], c - ck[bk]
                ok = bq == bk and (not causal or j <= i) and (wl < 0 or j >= i - wl) \
                    and (wr < 0 or j <= i + wr)
                assert m[r, c] == ok, (r, c)
    seq, pos = packed_positions([0, 2, 2, 5])
    assert seq.tolist() == [0, 0, 2, 2, 2] and pos.tolist() == [0, 1, 0, 1, 2]


@pytest.mark.parametrize("kw", [dict(causal=True), dict(causal=False),
                                dict(causal=True, window_left=2),
                                dict(causal=False, t5_table=True),
                                dict(causal=True, alibi=True)])
def test_packed_equals_each_sequence_alone(kw):
    # The packed reading reduces to the pinned dense oracle run on each
    # sequence by itself (positions from 0), including an empty sequence, a
    # single-row one and sequences of keys longer / shorter than the queries.
    lq, lk = [5, 0, 1, 9, 4], [5, 0, 3, 9, 2]
    cq, ck, q, k, v, do = _packed(lq, lk)
    extra = dict(kw)
    if extra.pop("t5_table", False):
        extra["t5_table"] = rnd((32, 4), 9)
    if extra.pop("alibi", False):
        extra["alibi_slopes"] = np.array([0.5, 0.25, 0.125, 0.0625])
    O, LSE = attention_forward_packed(q, k, v, cq, ck, **extra)
    dQ, dK, dV = attention_backward_packed(q, k, v, do, cq, ck, **extra)
    for b in range(len(lq)):
        q0, q1, k0, k1 = cq[b], cq[b + 1], ck[b], ck[b + 1]
        if q1 == q0:
            continue
        if k1 == k0:
            assert (O[q0:q1] == 0).all() and np.isneginf(LSE[:, q0:q1]).all()
            continue
        Ob, Lb = attention_forward(q[None, q0:q1], k[None, k0:k1], v[None, k0:k1], **extra)
        gq, gk, gv = attention_backward(q[None, q0:q1], k[None, k0:k1], v[None, k0:k1],
                                        do[None, q0:q1], **extra)
        assert np.allclose(O[q0:q1], Ob[0], atol=1e-12)
        assert np.allclose(LSE[:, q0:q1], Lb[0], atol=1e-12)
        assert np.allclose(dQ[q0:q1], gq[0], atol=1e-11)
        assert np.allclose(dK[k0:k1], gk[0], atol=1e-11)
        assert np.allclose(dV[k0:k1], gv[0], atol=1e-11)


def test_packed_sequences_do_not_see_each_other():
    cq, ck, q, k, v, do = _packed([6, 4, 7], [6, 4, 7])
    O0, _ = attention_forward_packed(q, k, v, cq, ck, causal=True)
    g0 = attention_backward_packed(q, k, v, do, cq, ck, causal=True)
    k2, v2 = k.copy(), v.copy()
    k2[ck[1]:ck[2]] += 5.0          # change every key and value of the middle sequence
    v2[ck[1]:ck[2]] -= 3.0
    O1, _ = attention_forward_packed(q, k2, v2, cq, ck, causal=True)
    g1 = attention_backward_packed(q, k2, v2, do, cq, ck, causal=True)
    for lo, hi in ((cq[0], cq[1]), (cq[2], cq[3])):
        assert np.array_equal(O0[lo:hi], O1[lo:hi])
        assert np.array_equal(g0[0][lo:hi], g1[0][lo:hi])
    assert not np.allclose(O0[cq[1]:cq[2]], O1[cq[1]:cq[2]])


def test_packed_gradients_central_differences():
    cq, ck, q, k, v, do = _packed([3, 2], [2, 4], Hq=2, Hkv=1, d=3, seed=4)
    kw = dict(causal=False, t5_table=rnd((8, 2), 5), t5_num_buckets=8, t5_max_distance=20)

    def loss(q_, k_, v_):
        O, _ = attention_forward_packed(q_, k_, v_, cq, ck, **kw)
        return float(np.sum(O * do))
    dQ, dK, dV = attention_backward_packed(q, k, v, do, cq, ck, **kw)
    h = 1e-6
    for arr, grad, which in ((q, dQ, 0), (k, dK, 1), (v, dV, 2)):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            a = [q.copy(), k.copy(), v.copy()]
            a[which][idx] += h
            up = loss(*a)
            a[which][idx] -= 2 * h
            num[idx] = (up - loss(*a)) / (2 * h)
        assert np.allclose(grad, num, rtol=1e-6, atol=1e-8), which


# ------------------------------------------- relative-position table, FIRE
def test_rel_table_equals_the_dense_bias_it_expands_to():
    # cross-attention shape, so a wrong offset or a swapped i / j shows
    B, L, Lk, Hq, Hkv, d = 1, 6, 9, 2, 1, 4
    q = rnd((B, L, Hq, d), 71)
    k, v = rnd((B, Lk, Hkv, d), 72), rnd((B, Lk, Hkv, d), 73)
    do = rnd((B, L, Hq, d), 74)
    table = rnd((L + Lk - 1, Hq), 75)
    dense = np.zeros((1, Hq, L, Lk))
    for h in range(Hq):
        for i in range(L):
            for j in range(Lk):
                dense[0, h, i, j] = table[j - i + L - 1, h]     # entry j - i + L - 1
    for causal in (False, True):
        O1, L1 = attention_forward(q, k, v, causal=causal, rel_table=table)
        O2, L2 = attention_forward(q, k, v, causal=causal, bias=dense)
        assert np.allclose(O1, O2, atol=1e-14) and np.allclose(L1, L2, atol=1e-14)
        g1 = attention_backward(q, k, v, do, causal=causal, rel_table=table)
        g2 = attention_backward(q, k, v, do, causal=causal, bias=dense)
        for a, b_ in zip(g1, g2):
            assert np.allclose(a, b_, atol=1e-13)


def test_rel_table_of_t5_buckets_is_the_t5_bias():
    # a table filled from the (golden-pinned) T5 buckets gives the T5 bias
    q, k, v, do = qkv(B=1, L=10, Hq=2, Hkv=2, d=4, seed=81)
    t5 = rnd((32, 2), 82)
    rel = np.arange(-9, 10)
    table = t5[t5_relative_bucket(rel, 32, 128, True), :]
    O1, _ = attention_forward(q, k, v, rel_table=table)
    O2, _ = attention_forward(q, k, v, t5_table=t5)
    assert np.allclose(O1, O2, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_rel_table_gradient_central_differences(causal):
    B, L, Hq, Hkv, d = 2, 7, 2, 1, 3
    q, k, v, do = qkv(B, L, Hq, Hkv, d, seed=91)
    table = rnd((2 * L - 1, Hq), 92)
    kw = dict(causal=causal, rel_table=table)
    *_, dS = attention_backward(q, k, v, do, return_dbias=True, **kw)
    g = rel_table_gradient(dS)
    h = 1e-6
    for r, hq in [(0, 0), (L - 1, 1), (L + 2, 0), (2 * L - 2, 1), (3, 1)]:
        tp = table.copy(); tp[r, hq] += h
        tm = table.copy(); tm[r, hq] -= h
        num = (_loss(q, k, v, do, {**kw, "rel_table": tp})
               - _loss(q, k, v, do, {**kw, "rel_table": tm})) / (2 * h)
        assert abs(num - g[r, hq]) < 1e-7, (r, hq, num, g[r, hq])
    if causal:
        assert np.all(g[L:, :] == 0.0)          # keys after the query see nothing


def test_fire_table_hand_worked():
    # c = 1, threshold 15: psi(t) = log(t + 1), psi(15) = log 16, so the
    # distances 0, 1, 3, 15 map to x = 0, 1/4, 1/2, 1 exactly.  With
    # w1 = (1, -1), b1 = (0, 1/2), w2 = (2, 3), b2 = 1/4:
    #   f(x) = 2 relu(x) + 3 relu(1/2 - x) + 1/4
    #   f(0) = 1.75, f(1/4) = 0.5 + 0.75 + 0.25 = 1.5,
    #   f(1/2) = 1 + 0 + 0.25 = 1.25, f(1) = 2 + 0 + 0.25 = 2.25
    t = fire_table(16, 16, 1.0, 15.0, [1.0, -1.0], [0.0, 0.5], [[2.0, 3.0]], [0.25])
    assert t.shape == (31, 1)
    for dist, want in ((0, 1.75), (1, 1.5), (3, 1.25), (15, 2.25)):
        assert abs(t[15 + dist, 0] - want) < 1e-12 and abs(t[15 - dist, 0] - want) < 1e-12


def test_fire_threshold_reading():
    # the threshold must cover every query position: max(T, i) = T then
    fire_table(8, 8, 1.0, 7.0, [1.0], [0.0], [[1.0]], [0.0])
    with pytest.raises(ValueError):
        fire_table(8, 8, 1.0, 6.0, [1.0], [0.0], [[1.0]], [0.0])


def test_fire_gradients_central_differences():
    rng = np.random.default_rng(97)
    L, Lk, W, H = 9, 12, 5, 3
    params = dict(w1=rng.standard_normal(W), b1=rng.standard_normal(W) * 0.5,
                  w2=rng.standard_normal((H, W)), b2=rng.standard_normal(H))
    c, thr = 0.7, 11.0
    g = rng.standard_normal((L + Lk - 1, H))

    def loss(p, c_, t_):
        return float(np.sum(g * fire_table(L, Lk, c_, t_, p["w1"], p["b1"], p["w2"], p["b2"])))

    grads = fire_gradients(g, L, Lk, c, thr, **params)
    h = 1e-6
    for name in ("w1", "b1", "w2", "b2"):
        flat = params[name].reshape(-1)
        for idx in range(flat.size):
            pp = {n: a.copy() for n, a in params.items()}
            pm = {n: a.copy() for n, a in params.items()}
            pp[name].reshape(-1)[idx] += h
            pm[name].reshape(-1)[idx] -= h
            num = (loss(pp, c, thr) - loss(pm, c, thr)) / (2 * h)
            assert abs(num - grads[name].reshape(-1)[idx]) < 1e-6, (name, idx)
    num_c = (loss(params, c + h, thr) - loss(params, c - h, thr)) / (2 * h)
    num_t = (loss(params, c, thr + h) - loss(params, c, thr - h)) / (2 * h)
    assert abs(num_c - grads["c"]) < 1e-6 and abs(num_t - grads["threshold"]) < 1e-6
