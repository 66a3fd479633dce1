"""GPU parity of the relative-position table bias (SDPA_BIAS_REL) and of FIRE
against the float64 oracle: forward and backward through the table, the
table's gradient from sdpa_bwd_bias_grad, FIRE's table and the gradients of
its parameters, and bitwise repeats.

Tolerances: O, dQ, dK, dV as every parity test (1e-2 + 1e-2 |ref|, LSE
1e-3).  The table gradient sums dS over a diagonal, so it carries the
rounding of D = rowsum(dO * O) from the stored bf16 O exactly as the T5
table gradient does (tests/test_gpu_bias_grad.py derives the bound): per
table row r the rows' terms e_i P_{i, i+r} add in quadrature.  FIRE's table
and gradients are float32 arithmetic on float32 weights: their bound is
float32 rounding of the log, the MLP and the sums over at most 2L - 1 rows,
1e-5 + 1e-5 |ref| for the table and 1e-4 + 1e-4 |ref| for the gradients.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import assert_close, mask_kw
from oracle import (attention_backward, attention_forward, attention_probs, fire_gradients,
                    fire_table, rel_table_gradient)
from scaled_dot_product_bwd_b200 import (sdpa_bwd, sdpa_bwd_bias_grad, sdpa_fire_backward,
                                         sdpa_fire_table, sdpa_fwd)
from scaled_dot_product_bwd_b200.inputs import make_fire_params, make_inputs
from test_gpu_bias_grad import check_bias_grad, row_error_scale, tolerance

pytestmark = pytest.mark.gpu

CASES = {
    # L = 300 leaves ragged tiles; cross-attention reads the table's other rows
    "rel_bidir_d64": dict(B=2, Hq=4, Hkv=2, L=300, d=64),
    "rel_causal_gqa_d128": dict(B=1, Hq=4, Hkv=1, L=270, d=128, causal=True),
    "rel_window_d64": dict(B=1, Hq=2, Hkv=2, L=390, d=64, causal=True, wl=100),
    "rel_cross_d64": dict(B=2, Hq=2, Hkv=1, L=200, Lk=330, d=64),
    "rel_cross_causal_d128": dict(B=1, Hq=2, Hkv=2, L=260, Lk=150, d=128, causal=True),
}


def _inputs(c, seed=0):
    return make_inputs(c["B"], c["L"], c["Hq"], c["Hkv"], c["d"], seed=seed, Lk=c.get("Lk"),
                       rel_table=True)


def _run(c, inp, table=None):
    dev = torch.device("cuda")
    q, k, v, do = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.do))
    table = inp.rel_table.to(dev) if table is None else table
    kw = dict(mask_kw(c), rel_table=table)
    o, lse = sdpa_fwd(q, k, v, **kw)
    dq, dk, dv = sdpa_bwd(q, k, v, o, do, lse, **kw)
    torch.cuda.synchronize()
    return {n: t.float().cpu().numpy() for n, t in
            dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv).items()}


def _oracle(c, inp, table):
    kw = dict(mask_kw(c), rel_table=table)
    O, LSE = attention_forward(inp.q, inp.k, inp.v, **kw)
    dq, dk, dv = attention_backward(inp.q, inp.k, inp.v, inp.do, **kw)
    return dict(o=O, lse=LSE, dq=dq, dk=dk, dv=dv)


@pytest.mark.parametrize("name", list(CASES))
def test_rel_table_parity(name):
    c = CASES[name]
    inp = _inputs(c)
    got = _run(c, inp)
    assert_close(got, _oracle(c, inp, inp.rel_table))


def test_rel_table_bitwise_repeatable():
    c = CASES["rel_causal_gqa_d128"]
    inp = _inputs(c)
    first = _run(c, inp)
    again = _run(c, inp)
    for n in first:
        assert np.array_equal(first[n], again[n]), n


@pytest.mark.parametrize("name", ["rel_bidir_d64", "rel_causal_gqa_d128", "rel_window_d64"])
def test_rel_table_gradient(name):
    c = CASES[name]
    inp = _inputs(c)
    dev = torch.device("cuda")
    q, k, v, do = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.do))
    table = inp.rel_table.to(dev)
    kw = dict(mask_kw(c), rel_table=table)
    o, lse = sdpa_fwd(q, k, v, **kw)
    dq, dk, dv, dtable = sdpa_bwd_bias_grad(q, k, v, o, do, lse, **kw)
    dq0, dk0, dv0 = sdpa_bwd(q, k, v, o, do, lse, **kw)
    again = sdpa_bwd_bias_grad(q, k, v, o, do, lse, **kw)[3]
    torch.cuda.synchronize()
    for a, b in ((dq, dq0), (dk, dk0), (dv, dv0), (dtable, again)):
        assert torch.equal(a, b)
    okw = dict(mask_kw(c), rel_table=inp.rel_table)
    *_, dS = attention_backward(inp.q, inp.k, inp.v, inp.do, return_dbias=True, **okw)
    want = rel_table_gradient(dS)
    # per table row r: sum over rows of (e_i P_{i, i + r})^2
    e = row_error_scale(c, inp)
    B, Hq, L = e.shape
    q2 = np.zeros_like(want)
    rows = np.arange(L)[:, None]
    cols = np.arange(L)[None, :]
    idx = (cols - rows + L - 1).ravel()
    for b in range(B):
        for h in range(Hq):
            P = attention_probs(inp.q, inp.k, b, h, **okw)
            np.add.at(q2[:, h], idx, ((P * e[b, h, :, None]) ** 2).ravel())
    check_bias_grad(dtable.cpu().numpy(), want, tolerance(want, q2))


# --------------------------------------------------------------------- FIRE
FIRE = dict(width=32, heads=4, c=0.5)


def _fire(L, Lk, seed=0, threshold=None):
    prm = make_fire_params(FIRE["width"], FIRE["heads"], seed=seed)
    thr = float(L - 1 if threshold is None else threshold)
    return prm, thr


def test_fire_table_matches_oracle():
    L, Lk = 700, 500
    prm, thr = _fire(L, Lk)
    dev = torch.device("cuda")
    got = sdpa_fire_table(*(prm[n].to(dev) for n in ("w1", "b1", "w2", "b2")), FIRE["c"], thr,
                          L, Lk).cpu().numpy()
    want = fire_table(L, Lk, FIRE["c"], thr, *(prm[n].double().numpy()
                                               for n in ("w1", "b1", "w2", "b2")))
    err = np.abs(got - want)
    assert np.all(err <= 1e-5 + 1e-5 * np.abs(want)), err.max()


def test_fire_backward_matches_oracle_and_repeats():
    L, Lk = 600, 600
    prm, thr = _fire(L, Lk, seed=3, threshold=800)
    g = torch.Generator().manual_seed(11)
    d_table = torch.randn(L + Lk - 1, FIRE["heads"], generator=g, dtype=torch.float32)
    dev = torch.device("cuda")
    args = [prm[n].to(dev) for n in ("w1", "b1", "w2", "b2")] + [FIRE["c"], thr, L, Lk]
    got = sdpa_fire_backward(*args, d_table.to(dev))
    again = sdpa_fire_backward(*args, d_table.to(dev))
    for n in got:
        assert torch.equal(got[n], again[n]), n
    want = fire_gradients(d_table.double().numpy(), L, Lk, FIRE["c"], thr,
                          *(prm[n].double().numpy() for n in ("w1", "b1", "w2", "b2")))
    for n in ("w1", "b1", "w2", "b2"):
        a, b = got[n].cpu().numpy(), want[n]
        assert np.all(np.abs(a - b) <= 1e-4 + 1e-4 * np.abs(b)), (n, np.abs(a - b).max())
    ct = got["c_threshold"].cpu().numpy()
    for i, n in enumerate(("c", "threshold")):
        assert abs(ct[i] - want[n]) <= 1e-4 + 1e-4 * abs(want[n]), (n, ct[i], want[n])


def test_attention_with_fire_bias():
    # FIRE's table from the GPU drives the relative-position kernels
    c = dict(B=1, Hq=4, Hkv=2, L=256, d=64, causal=True)
    inp = make_inputs(c["B"], c["L"], c["Hq"], c["Hkv"], c["d"], seed=5)
    prm, thr = _fire(c["L"], c["L"], seed=7)
    dev = torch.device("cuda")
    table = sdpa_fire_table(*(prm[n].to(dev) for n in ("w1", "b1", "w2", "b2")), FIRE["c"], thr,
                            c["L"], c["L"])
    got = _run(c, inp, table=table)
    ref_table = fire_table(c["L"], c["L"], FIRE["c"], thr,
                           *(prm[n].double().numpy() for n in ("w1", "b1", "w2", "b2")))
    assert_close(got, _oracle(c, inp, ref_table))


def test_fire_threshold_below_the_queries_is_refused():
    from scaled_dot_product_bwd_b200 import SdpaError
    prm, _ = _fire(64, 64)
    dev = torch.device("cuda")
    with pytest.raises(SdpaError) as e:
        sdpa_fire_table(*(prm[n].to(dev) for n in ("w1", "b1", "w2", "b2")), 1.0, 10.0, 64, 64)
    assert e.value.status == 2
