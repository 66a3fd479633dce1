"""GPU parity at the full sizes of the benchmark workloads, in the launch
configuration the bench times, checked against the float64 oracle on sampled
(batch, KV-head group) units -- and, where a whole head is too large for the
oracle, on sampled query rows -- plus bitwise repeatability at full size.

Workloads (seeded N(0,1) inputs, bf16; see scaled_dot_product_bwd_b200.inputs):
  mistral4k  B4 Hq32 Hkv8 L4096 d128, causal, window_left 4096 (== causal)
  mistral8k  B2 Hq32 Hkv8 L8192 d128, causal, window_left 4096
  t5rpe      B16 H12 L1024 d64, bidirectional, T5 table [32, 12], max_distance 128
  t5dense    same shape, dense fp32 bias [16, 12, 1024, 1024]
  sweep      forward only, Hq32 d128 causal, Hkv in {32, 8, 1}, B * L = 32768
"""
import numpy as np
import pytest
import torch

from gpu_helpers import assert_close, case_inputs, run_cuda
from oracle import attention_backward, attention_forward

pytestmark = pytest.mark.gpu

FULL = {
    "mistral4k": dict(B=4, Hq=32, Hkv=8, L=4096, d=128, causal=True, wl=4096,
                      sample=dict(batches=[3], kv_heads=[5])),
    "mistral8k": dict(B=2, Hq=32, Hkv=8, L=8192, d=128, causal=True, wl=4096,
                      sample=dict(batches=[1], kv_heads=[0])),
    "t5rpe": dict(B=16, Hq=12, Hkv=12, L=1024, d=64, bias="t5",
                  sample=dict(batches=[0, 15], kv_heads=[0, 11])),
    "t5dense": dict(B=16, Hq=12, Hkv=12, L=1024, d=64, bias="dense",
                    sample=dict(batches=[7], kv_heads=[3, 10])),
}


def _oracle(c, inp, sample, backward=True, query_rows=None):
    kw = dict(causal=c.get("causal", False), window_left=c.get("wl", -1),
              window_right=c.get("wr", -1), bias=inp.bias, t5_table=inp.t5_table, **sample)
    O, LSE = attention_forward(inp.q, inp.k, inp.v, query_rows=query_rows, **kw)
    out = {"o": O, "lse": LSE}
    if backward:
        dq, dk, dv = attention_backward(inp.q, inp.k, inp.v, inp.do, **kw)
        out.update(dq=dq, dk=dk, dv=dv)
    return out


@pytest.mark.parametrize("name", list(FULL))
def test_full_size_parity_and_repeatability(name):
    c = FULL[name]
    inp = case_inputs(c)
    got = run_cuda(c, inp)
    again = run_cuda(c, inp)
    for n in got:
        assert np.array_equal(got[n], again[n]), f"{n} not bitwise repeatable"
    ref = _oracle(c, inp, c["sample"])
    assert_close(got, ref)


SWEEP = [(hkv, L) for hkv in (32, 8, 1) for L in (512, 2048, 8192, 16384)]


@pytest.mark.parametrize("hkv,L", SWEEP)
def test_forward_sweep_parity_and_repeatability(hkv, L):
    c = dict(B=32768 // L, Hq=32, Hkv=hkv, L=L, d=128, causal=True)
    inp = case_inputs(c)
    got = run_cuda(c, inp, backward=False)
    again = run_cuda(c, inp, backward=False)
    for n in got:
        assert np.array_equal(got[n], again[n]), f"{n} not bitwise repeatable"
    # one (batch, KV group) unit; for long sequences a spread of query rows
    rows = None if L <= 2048 else np.unique(np.r_[0:64, L // 2 - 64:L // 2 + 64,
                                                  L - 200:L, np.linspace(0, L - 1, 97).astype(int)])
    sample = dict(batches=[c["B"] - 1], kv_heads=[hkv - 1])
    ref = _oracle(c, inp, sample, backward=False, query_rows=rows)
    assert_close(got, ref, names=("o", "lse"))
