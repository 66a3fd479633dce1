"""GPU parity of packed variable-length batches (sdpa_fwd_varlen /
sdpa_bwd_varlen) against the float64 oracle's packed reading: sequences end
to end on one axis, positions from 0 in each, no attention across
sequences.  Ragged lengths include an empty sequence, single rows, lengths
one past a tile and several tiles, and keys of other lengths than the
queries.

Tolerance.  O and LSE take the fixed bound (1e-2 + 1e-2 |ref|; 1e-3).  The
gradients take it plus the rounding the kernels' bf16 operands add, derived
from the arithmetic (the reading that the bias-gradient tests use for dS):
with u = 2^-8, D_i = rowsum(dO * O) is formed from the stored bf16 O, off by
e_i = 4 u sqrt(sum_c (dO_ic O_ic)^2); dS_ij is rounded to bf16 for the MMAs
(4 u |dS_ij| / sqrt 3 at four standard deviations), so each dS entry is off
by about delta_ij = P_ij e_i + 4 u |dS_ij| / sqrt 3, and P is rounded to
bf16 for dV (4 u P_ij / sqrt 3).  Entries of a sum round independently, so
    dQ_ic: scale sqrt(sum_j (delta_ij K_jc)^2)
    dK_jc: scale sqrt(sum_i (delta_ij Q_ic)^2)
    dV_jc: sqrt(sum_i (4 u P_ij dO_ic / sqrt 3)^2)
are added to the fixed bound.  Where every key is shared by few queries
these terms are far below 1e-2; a sequence whose queries outnumber its keys
(200 queries over 7 keys here) piles them onto each key.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import ATOL, LSE_ATOL, RTOL
from oracle import attention_backward_packed, attention_forward_packed
from scaled_dot_product_bwd_b200 import sdpa_bwd_varlen, sdpa_fwd_varlen
from scaled_dot_product_bwd_b200.inputs import cu_seqlens, make_inputs

pytestmark = pytest.mark.gpu

CASES = {
    "self_causal_d128": dict(lq=[37, 300, 1, 129, 0, 255], Hq=4, Hkv=2, d=128, causal=True),
    "self_bidir_t5_d64": dict(lq=[128, 17, 400, 1, 96], Hq=2, Hkv=2, d=64, bias="t5"),
    "self_window_mqa_d128": dict(lq=[500, 3, 260], Hq=4, Hkv=1, d=128, causal=True, wl=64),
    "cross_bidir_d64": dict(lq=[50, 200, 1, 130], lk=[300, 7, 129, 0], Hq=2, Hkv=1, d=64),
    "cross_alibi_causal_d128": dict(lq=[140, 260], lk=[70, 400], Hq=2, Hkv=2, d=128,
                                    causal=True, bias="alibi"),
}


U_BF16 = 2.0 ** -8


def rounding_allowance(q, k, do, O, P, dS, scale):
    """The derived terms of the module docstring for dQ, dK, dV."""
    q, k, do = (t.double().numpy() for t in (q, k, do))
    Hq, Hkv = q.shape[1], k.shape[1]
    G = Hq // Hkv
    e = 4 * U_BF16 * np.sqrt(np.sum((do * O) ** 2, axis=-1))          # [Tq, Hq]
    vq = np.zeros(q.shape)
    vk = np.zeros(k.shape)
    vv = np.zeros(k.shape)
    r = 4 * U_BF16 / np.sqrt(3.0)
    for hq in range(Hq):
        g = hq // G
        dd = P[hq] * e[:, hq, None] + r * np.abs(dS[hq])
        vq[:, hq, :] = scale ** 2 * ((dd ** 2) @ (k[:, g, :] ** 2))
        vk[:, g, :] += scale ** 2 * ((dd ** 2).T @ (q[:, hq, :] ** 2))
        vv[:, g, :] += (r ** 2) * ((P[hq] ** 2).T @ (do[:, hq, :] ** 2))
    return dict(dq=np.sqrt(vq), dk=np.sqrt(vk), dv=np.sqrt(vv))


def _close(name, got, ref, atol, extra=0.0):
    got = got.float().cpu().numpy()
    both_inf = np.isinf(ref) & (ref == got)
    with np.errstate(invalid="ignore"):  # inf - inf where both agree: masked below
        err = np.where(both_inf, 0.0, np.abs(got - ref))
    tol = atol + (RTOL * np.abs(ref) if atol == ATOL else 0.0) + extra
    bad = ~(err <= tol)
    where = [tuple(int(x) for x in ix) for ix in np.argwhere(bad)[:6]]
    assert not bad.any(), (f"{name}: {int(bad.sum())} of {bad.size} outside, max "
                           f"{np.nanmax(err):.3e}; first at {where}: ref "
                           f"{[float(ref[w]) for w in where]} got {[float(got[w]) for w in where]}")


def _run(c, seed=0):
    lq = c["lq"]
    lk = c.get("lk", lq)
    tq, tk = sum(lq), sum(lk)
    inp = make_inputs(1, tq, c["Hq"], c["Hkv"], c["d"], seed=seed, Lk=tk,
                      t5_buckets=32 if c.get("bias") == "t5" else 0, alibi=c.get("bias") == "alibi")
    q, k, v, do = (t[0] for t in (inp.q, inp.k, inp.v, inp.do))
    cq, ck = cu_seqlens(lq), cu_seqlens(lk)
    kw = dict(causal=c.get("causal", False), window_left=c.get("wl", -1))
    dev = torch.device("cuda")
    gkw = dict(kw)
    okw = dict(kw)
    if inp.t5_table is not None:
        gkw["t5_table"] = inp.t5_table.to(dev)
        okw["t5_table"] = inp.t5_table
    if inp.alibi_slopes is not None:
        gkw["alibi_slopes"] = inp.alibi_slopes.to(dev)
        okw["alibi_slopes"] = inp.alibi_slopes
    args = [t.to(dev) for t in (q, k, v)]
    cqd, ckd = cq.to(dev), ck.to(dev)
    o, lse = sdpa_fwd_varlen(*args, cqd, ckd, max(lq), max(lk), **gkw)
    dq, dk, dv = sdpa_bwd_varlen(*args, o, do.to(dev), lse, cqd, ckd, max(lq), max(lk), **gkw)
    torch.cuda.synchronize()
    got = dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv)
    return got, (q, k, v, do, cq.numpy(), ck.numpy(), okw)


@pytest.mark.parametrize("name", list(CASES))
def test_varlen_parity(name):
    got, (q, k, v, do, cq, ck, okw) = _run(CASES[name])
    O, LSE = attention_forward_packed(q, k, v, cq, ck, **okw)
    dQ, dK, dV, P, dS = attention_backward_packed(q, k, v, do, cq, ck,
                                                  return_intermediates=True, **okw)
    extra = rounding_allowance(q, k, do, O, P, dS, 1.0 / np.sqrt(q.shape[-1]))
    _close("o", got["o"], O, ATOL)
    _close("lse", got["lse"], LSE, LSE_ATOL)
    _close("dq", got["dq"], dQ, ATOL, extra["dq"])
    _close("dk", got["dk"], dK, ATOL, extra["dk"])
    _close("dv", got["dv"], dV, ATOL, extra["dv"])


def test_varlen_bitwise_repeatable():
    a, _ = _run(CASES["self_causal_d128"])
    b, _ = _run(CASES["self_causal_d128"])
    for n in a:
        assert torch.equal(a[n], b[n]), n
