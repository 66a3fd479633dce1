"""GPU parity of the bias gradients (sdpa_bwd_bias_grad) against the float64
oracle: a dense bias's gradient is dS, summed over the indices the bias is
broadcast along; a T5 table's gradient is dS summed per bucket of j - i; the
ALiBi slopes' gradient is -sum |j - i| dS per head.

Tolerances.  dS = P (dP - D) with D = rowsum(dO * O) formed from the stored
bf16 O, so D_i carries the rounding of O: with unit roundoff u = 2^-8 (bf16,
round to nearest even) each O_id is off by at most u |O_id|, and under the
probabilistic model of rounding errors (independent, uniform, standard
deviation u |O_id| / sqrt(3)) D_i is off by about u sqrt(sum_d (dO_id O_id)^2
/ 3).  dS_ij inherits P_ij times that, unscaled -- dQ = scale dS K divides it
by sqrt(d), which is why the other gradients do not feel it.  Let
    e_i = 4 u sqrt(sum_d (dO_id O_id)^2)      (about seven standard deviations).
An output that sums dS over a set of entries takes, from each query row
(b, h, i), the row's one D error times the P mass of its entries in the set:
w_row = e_i * sum of P_ij over those entries (weighted by |j - i| for the
ALiBi slopes).  Rows round independently, so
the rows' terms add in quadrature, and the bound is
    |err| <= 1e-2 + 1e-2 |ref| + sqrt(sum over rows of w_row^2)
(for a full-shape dense bias one row and one entry: 1e-2 + 1e-2 |dS| + P e).
The other rounding in dS (fp32 P and dP) and in the fp32 sums is orders of
magnitude smaller and sits inside the relative term.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import ATOL, RTOL, assert_close, case_inputs, mask_kw
from oracle import (alibi_slope_gradient, attention_backward, attention_forward,
                    attention_probs, dense_bias_gradient, t5_relative_bucket,
                    t5_table_gradient, visibility_mask)
from scaled_dot_product_bwd_b200 import sdpa_bwd, sdpa_bwd_bias_grad, sdpa_fwd
from scaled_dot_product_bwd_b200.inputs import Inputs

pytestmark = pytest.mark.gpu

CASES = {
    # full-shape dense bias: dS written straight into dbias
    "dense_full_causal_d128": dict(B=2, Hq=2, Hkv=1, L=200, d=128, causal=True, bias="dense"),
    # the bias staged by TMA (d = 64); a window leaves key tiles to zero-fill
    "dense_full_window_d64": dict(B=1, Hq=3, Hkv=3, L=260, d=64, causal=True, wl=70,
                                  bias="dense"),
    # broadcast biases: dS staged, then reduced over heads / batch / both
    "dense_heads_bcast_d64": dict(B=2, Hq=4, Hkv=2, L=132, d=64, bias="dense",
                                  bias_shape=(2, 1, 132, 132)),
    "dense_batch_bcast_causal_d128": dict(B=3, Hq=2, Hkv=2, L=144, d=128, causal=True,
                                          bias="dense", bias_shape=(1, 2, 144, 144)),
    "dense_all_bcast_window_d64": dict(B=2, Hq=2, Hkv=1, L=132, d=64, wl=40, wr=20,
                                       bias="dense", bias_shape=(1, 1, 132, 132)),
    # T5 tables; L = 301 leaves a ragged last tile and rows not a multiple of 4
    "t5_bidir_d64": dict(B=2, Hq=4, Hkv=4, L=301, d=64, bias="t5"),
    "t5_bidir_causal_gqa_d128": dict(B=1, Hq=2, Hkv=1, L=270, d=128, causal=True, bias="t5"),
    "t5_unidir_causal_d64": dict(B=2, Hq=2, Hkv=2, L=280, d=64, causal=True, bias="t5",
                                 t5_bidirectional=False),
    # short max distances: the capped bucket starts at distance 16 (16
    # buckets, max distance 24) or 14 (8 buckets, max distance 20), so most
    # 32 x 32 pieces of dS lie in one bucket, on both sides of the diagonal
    "t5_bidir_short_d64": dict(B=2, Hq=2, Hkv=2, L=330, d=64, bias="t5", t5_nb=16, t5_md=24),
    "t5_unidir_short_d64": dict(B=1, Hq=2, Hkv=2, L=300, d=64, bias="t5", t5_nb=8, t5_md=20,
                                t5_bidirectional=False),
    "t5_unidir_short_causal_d128": dict(B=1, Hq=2, Hkv=1, L=300, d=128, causal=True, bias="t5",
                                        t5_nb=8, t5_md=20, t5_bidirectional=False),
    # ALiBi slopes: dm_h = -sum |j - i| dS
    "alibi_bidir_d64": dict(B=2, Hq=4, Hkv=4, L=301, d=64, bias="alibi"),
    "alibi_causal_gqa_d128": dict(B=1, Hq=2, Hkv=1, L=270, d=128, causal=True, bias="alibi"),
}


def run_cuda_bias_grad(c, inp, bias=None):
    dev = torch.device("cuda")
    q, k, v, do = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.do))
    if bias is None and inp.bias is not None:
        bias = inp.bias.to(dev)
    table = inp.t5_table.to(dev) if inp.t5_table is not None else None
    slopes = inp.alibi_slopes.to(dev) if inp.alibi_slopes is not None else None
    kw = dict(mask_kw(c), bias=bias, t5_table=table, alibi_slopes=slopes)
    o, lse = sdpa_fwd(q, k, v, **kw)
    dq, dk, dv, dbias = sdpa_bwd_bias_grad(q, k, v, o, do, lse, **kw)
    dq0, dk0, dv0 = sdpa_bwd(q, k, v, o, do, lse, **kw)
    torch.cuda.synchronize()
    out = {n: t.float().cpu().numpy() for n, t in
           dict(dq=dq, dk=dk, dv=dv, dq0=dq0, dk0=dk0, dv0=dv0).items()}
    out["dbias"] = dbias.cpu().numpy()
    return out


def oracle_ds(c, inp):
    kw = dict(mask_kw(c), bias=inp.bias, t5_table=inp.t5_table,
              alibi_slopes=inp.alibi_slopes)
    dq, dk, dv, dS = attention_backward(inp.q, inp.k, inp.v, inp.do, return_dbias=True, **kw)
    return dict(dq=dq, dk=dk, dv=dv), dS


U_BF16 = 2.0 ** -8


def row_error_scale(c, inp):
    """e_i of the module docstring, [B, Hq, L], from the oracle's O and dO."""
    kw = dict(mask_kw(c), bias=inp.bias, t5_table=inp.t5_table,
              alibi_slopes=inp.alibi_slopes, rel_table=getattr(inp, "rel_table", None))
    O, _ = attention_forward(inp.q, inp.k, inp.v, **kw)          # [B, L, Hq, d]
    dO = inp.do.double().numpy()
    e = 4 * U_BF16 * np.sqrt(np.sum((dO * O) ** 2, axis=-1))     # [B, L, Hq]
    return e.transpose(0, 2, 1)


def expected_bias_grad(c, inp, dS):
    """Oracle gradient and the sum over rows of w_row^2 (module docstring)."""
    kw = dict(mask_kw(c), bias=inp.bias, t5_table=inp.t5_table,
              alibi_slopes=inp.alibi_slopes)
    e = row_error_scale(c, inp)
    B, Hq, L = e.shape
    if c["bias"] == "dense":
        shape = tuple(inp.bias.shape)
        w2 = np.empty((B, Hq, L, L))      # each output entry holds one entry per row
        for b in range(B):
            for h in range(Hq):
                w2[b, h] = (attention_probs(inp.q, inp.k, b, h, **kw) * e[b, h, :, None]) ** 2
        return dense_bias_gradient(dS, shape), dense_bias_gradient(w2, shape)
    if c["bias"] == "alibi":
        dist = np.abs(np.arange(L)[None, :] - np.arange(L)[:, None])
        q2 = np.zeros(Hq)
        for b in range(B):
            for h in range(Hq):
                P = attention_probs(inp.q, inp.k, b, h, **kw)
                q2[h] += np.sum((e[b, h] * (P * dist).sum(axis=1)) ** 2)
        return alibi_slope_gradient(dS), q2
    bidir = c.get("t5_bidirectional", True)
    nb, md = c.get("t5_nb", 32), c.get("t5_md", 128)
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    cell = (i * nb + t5_relative_bucket(j - i, nb, md, bidir)).ravel()
    q2 = np.zeros((nb, Hq))
    for b in range(B):
        for h in range(Hq):
            P = attention_probs(inp.q, inp.k, b, h, **kw)
            mass = np.bincount(cell, weights=P.ravel(), minlength=L * nb).reshape(L, nb)
            q2[:, h] += np.sum((mass * e[b, h, :, None]) ** 2, axis=0)
    return t5_table_gradient(dS, nb, md, bidir), q2


def tolerance(ref, q2):
    return ATOL + RTOL * np.abs(ref) + np.sqrt(q2)


def check_bias_grad(got, ref, tol):
    err = np.abs(got.astype(np.float64) - ref)
    bad = ~(err <= tol)
    assert not bad.any(), (f"dbias: {int(bad.sum())} of {bad.size} outside tolerance, "
                           f"max err {err.max():.3e}, first bad ref {ref[bad][:4]} "
                           f"got {got[bad][:4]}")


@pytest.mark.parametrize("name", list(CASES))
def test_bias_grad_parity(name):
    c = CASES[name]
    inp = case_inputs(c)
    got = run_cuda_bias_grad(c, inp)
    ref, dS = oracle_ds(c, inp)
    assert_close(got, ref, names=("dq", "dk", "dv"))
    # the dS output changes nothing else: dQ, dK, dV are those of sdpa_bwd, bit for bit
    for n in ("dq", "dk", "dv"):
        assert np.array_equal(got[n], got[n + "0"]), n
    want, q2 = expected_bias_grad(c, inp, dS)
    assert got["dbias"].shape == want.shape
    check_bias_grad(got["dbias"], want, tolerance(want, q2))
    if c["bias"] == "dense" and want.shape == dS.shape:
        # masked keys, including whole key tiles the mask skips, are exactly 0
        M = visibility_mask(c["L"], c.get("causal", False), c.get("wl", -1), c.get("wr", -1))
        assert (got["dbias"][:, :, ~M] == 0).all()


def test_padded_dense_bias_gradient():
    # a bias whose rows are padded (stride L + 4): the gradient takes the
    # same layout and leaves the padding untouched
    c = dict(B=2, Hq=2, Hkv=2, L=136, d=64, causal=True, bias="dense")
    inp = case_inputs(c)
    L = c["L"]
    dev = torch.device("cuda")
    store = torch.full((2, 2, L, L + 4), 7.0, device=dev)
    store[..., :L] = inp.bias.to(dev)
    bias = store[..., :L]
    dbias_store = torch.full((2, 2, L, L + 4), 5.0, device=dev)
    q, k, v, do = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.do))
    kw = dict(mask_kw(c), bias=bias)
    o, lse = sdpa_fwd(q, k, v, **kw)
    *_, dbias = sdpa_bwd_bias_grad(q, k, v, o, do, lse, dbias=dbias_store[..., :L], **kw)
    torch.cuda.synchronize()
    assert (dbias_store[..., L:] == 5.0).all()
    _, dS = oracle_ds(c, inp)
    want, q2 = expected_bias_grad(c, inp, dS)
    check_bias_grad(dbias.cpu().numpy(), want, tolerance(want, q2))


@pytest.mark.parametrize("name", ["dense_full_window_d64", "dense_heads_bcast_d64",
                                  "t5_bidir_d64", "t5_bidir_short_d64", "alibi_causal_gqa_d128"])
def test_bias_grad_bitwise_repeatable(name):
    c = CASES[name]
    inp = case_inputs(c)
    first = run_cuda_bias_grad(c, inp)
    for _ in range(2):
        again = run_cuda_bias_grad(c, inp)
        for n in first:
            assert np.array_equal(first[n], again[n]), n


def test_bias_grad_of_expanded_bias():
    # a torch-expanded bias (stride 0 over heads) behaves as a broadcast one
    c = dict(B=2, Hq=3, Hkv=3, L=128, d=64, bias="dense", bias_shape=(2, 1, 128, 128))
    inp = case_inputs(c)
    bias = inp.bias.cuda().expand(2, 3, 128, 128)
    got = run_cuda_bias_grad(c, inp, bias=bias)
    _, dS = oracle_ds(c, inp)
    want, q2 = expected_bias_grad(c, inp, dS)
    check_bias_grad(got["dbias"][:, :1], want, tolerance(want, q2))


@pytest.mark.slow
def test_t5_table_gradient_full_size():
    # the T5 workload at full size (B16 H12 L1024 d64, 32 buckets, max
    # distance 128): every (b, i, j) enters the table gradient, so the
    # oracle's dS is formed for the whole batch, one batch entry at a time
    c = dict(B=16, Hq=12, Hkv=12, L=1024, d=64, bias="t5")
    inp = case_inputs(c)
    got = run_cuda_bias_grad(c, inp)
    again = run_cuda_bias_grad(c, inp)
    assert np.array_equal(got["dbias"], again["dbias"])
    ref = np.zeros((32, 12))
    q2 = np.zeros((32, 12))
    for b in range(c["B"]):
        sub = Inputs(inp.q[b:b + 1], inp.k[b:b + 1], inp.v[b:b + 1], inp.do[b:b + 1],
                     inp.t5_table, None)
        _, dS = oracle_ds(dict(c, B=1), sub)
        want, w2 = expected_bias_grad(dict(c, B=1), sub, dS)
        ref += want
        q2 += w2
    check_bias_grad(got["dbias"], ref, tolerance(ref, q2))


@pytest.mark.slow
def test_dense_bias_gradient_full_size_sampled():
    # the dense-bias workload at full size (B16 H12 L1024 d64, bias
    # [16, 12, 1024, 1024]): dbias = dS checked on two sampled heads of one
    # batch entry, and the whole array bitwise repeatable
    c = dict(B=16, Hq=12, Hkv=12, L=1024, d=64, bias="dense")
    inp = case_inputs(c)
    got = run_cuda_bias_grad(c, inp)
    again = run_cuda_bias_grad(c, inp)
    assert np.array_equal(got["dbias"], again["dbias"])
    b = 7
    sub = Inputs(inp.q[b:b + 1], inp.k[b:b + 1], inp.v[b:b + 1], inp.do[b:b + 1], None,
                 inp.bias[b:b + 1])
    kw = dict(mask_kw(c), bias=sub.bias)
    *_, dS = attention_backward(sub.q, sub.k, sub.v, sub.do, return_dbias=True,
                                kv_heads=[3, 10], **kw)
    O, _ = attention_forward(sub.q, sub.k, sub.v, kv_heads=[3, 10], **kw)
    dO = sub.do.double().numpy()
    for h in (3, 10):
        e = 4 * U_BF16 * np.sqrt(np.sum((dO[0, :, h] * O[0, :, h]) ** 2, axis=-1))
        P = attention_probs(sub.q, sub.k, 0, h, **kw)
        ref = dS[0, h]
        check_bias_grad(got["dbias"][b, h], ref, tolerance(ref, (P * e[:, None]) ** 2))
