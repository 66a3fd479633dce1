"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
binding and the float64 oracle on the same seeded inputs, then compare."""
from __future__ import annotations

import numpy as np
import torch

from oracle import attention_backward, attention_forward
from scaled_dot_product_bwd_b200 import sdpa_bwd, sdpa_fwd
from scaled_dot_product_bwd_b200.inputs import make_inputs

ATOL, RTOL = 1e-2, 1e-2      # O, dQ, dK, dV: |err| <= 1e-2 + 1e-2 |ref|
LSE_ATOL = 1e-3


def case_inputs(c):
    return make_inputs(c["B"], c["L"], c["Hq"], c["Hkv"], c["d"], seed=c.get("seed", 0),
                       t5_buckets=c.get("t5_nb", 32) if c.get("bias") == "t5" else 0,
                       dense_bias=c.get("bias") == "dense",
                       bias_shape=c.get("bias_shape"), alibi=c.get("bias") == "alibi",
                       Lk=c.get("Lk"))


def mask_kw(c):
    """Mask, scale and T5 options of a case (the same keywords on both sides)."""
    kw = dict(causal=c.get("causal", False), window_left=c.get("wl", -1),
              window_right=c.get("wr", -1))
    if "scale" in c:
        kw["scale"] = c["scale"]
    if "t5_bidirectional" in c:
        kw["t5_bidirectional"] = c["t5_bidirectional"]
    if "t5_nb" in c:
        kw["t5_num_buckets"] = c["t5_nb"]
    if "t5_md" in c:
        kw["t5_max_distance"] = c["t5_md"]
    return kw


def run_cuda(c, inp, backward=True):
    dev = torch.device("cuda")
    q, k, v, do = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.do))
    bias = inp.bias.to(dev) if inp.bias is not None else None
    table = inp.t5_table.to(dev) if inp.t5_table is not None else None
    slopes = inp.alibi_slopes.to(dev) if inp.alibi_slopes is not None else None
    kw = dict(mask_kw(c), bias=bias, t5_table=table, alibi_slopes=slopes)
    o, lse = sdpa_fwd(q, k, v, **kw)
    out = {"o": o, "lse": lse}
    if backward:
        dq, dk, dv = sdpa_bwd(q, k, v, o, do, lse, **kw)
        out.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    return {n: t.float().cpu().numpy() for n, t in out.items()}


def run_oracle(c, inp, backward=True, batches=None, kv_heads=None):
    kw = dict(mask_kw(c), bias=inp.bias, t5_table=inp.t5_table,
              alibi_slopes=inp.alibi_slopes, batches=batches, kv_heads=kv_heads)
    O, LSE = attention_forward(inp.q, inp.k, inp.v, **kw)
    out = {"o": O, "lse": LSE}
    if backward:
        dq, dk, dv = attention_backward(inp.q, inp.k, inp.v, inp.do, **kw)
        out.update(dq=dq, dk=dk, dv=dv)
    return out


def assert_close(got: dict, ref: dict, names=("o", "lse", "dq", "dk", "dv")):
    """Element-wise check wherever the oracle computed a value (NaN = not sampled)."""
    report = {}
    for n in names:
        if n not in ref:
            continue
        r = ref[n]
        g = got[n]
        sel = ~np.isnan(r)
        assert sel.any(), n
        rs, gs = r[sel], g[sel]
        both_inf = np.isinf(rs) & (rs == gs)
        with np.errstate(invalid="ignore"):  # inf - inf where both agree: masked below
            err = np.where(both_inf, 0.0, np.abs(gs.astype(np.float64) - rs))
        if n == "lse":
            tol = np.full_like(rs, LSE_ATOL)
        else:
            tol = ATOL + RTOL * np.abs(rs)
        bad = ~(err <= tol)
        report[n] = float(np.nanmax(err)) if err.size else 0.0
        assert not bad.any(), (f"{n}: {int(bad.sum())} of {bad.size} outside tolerance, "
                               f"max err {np.nanmax(err):.3e}; first bad ref "
                               f"{rs[bad][:4]} got {gs[bad][:4]}")
    return report
