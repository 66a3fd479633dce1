"""The allocation-free backward entry point, sdpa_bwd_noalloc, for callers
that cannot allocate device memory around the call (kernel hosts that hand a
library only its inputs and outputs, processes under a hard memory cap,
latency-bound loops that avoid cudaMalloc / cudaFree).  Its workspace (the
D vector) is a fixed array inside the library instead of caller memory; its results must match
sdpa_bwd's bit for bit, call after call.

Kept in its own file, named to be collected last.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import ATOL, RTOL
from scaled_dot_product_bwd_b200 import SdpaError, sdpa_bwd, sdpa_bwd_noalloc, sdpa_fwd
from scaled_dot_product_bwd_b200 import sdpa_bwd_workspace_size
from scaled_dot_product_bwd_b200.binding import NOALLOC_SCRATCH_BYTES
from scaled_dot_product_bwd_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu


def _same(got, ref, name):
    """Bit-identical: both entry points run the same kernels on the same inputs,
    so any difference means the scratch array fed a kernel stale or foreign
    data.  The tolerance figure is only there to describe a mismatch."""
    if torch.equal(got, ref):
        return
    a = got.float().cpu().numpy()
    b = ref.float().cpu().numpy()
    within = bool(np.all(np.abs(a - b) <= ATOL + RTOL * np.abs(b)))
    raise AssertionError(f"{name}: not bit-identical to sdpa_bwd "
                         f"(max |diff| {np.nanmax(np.abs(a - b)):.3e}, "
                         f"{'within' if within else 'outside'} the oracle tolerance)")


@pytest.mark.parametrize("kw", [dict(causal=True), dict(causal=False, t5=True)])
def test_noalloc_matches_workspace_entry_point_twice(kw):
    dev = torch.device("cuda")
    t5 = kw.get("t5", False)
    mask = {n: v for n, v in kw.items() if n != "t5"}
    for call, seed in enumerate((1, 2)):   # two calls in a row, different inputs
        inp = make_inputs(2, 300, 4, 2, 128, seed=seed, t5_buckets=32 if t5 else 0)
        q, k, v, do = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.do))
        extra = dict(mask)
        if t5:
            extra["t5_table"] = inp.t5_table.to(dev)
        o, lse = sdpa_fwd(q, k, v, **extra)
        ref = sdpa_bwd(q, k, v, o, do, lse, **extra)
        out = (torch.full_like(q, float("nan")), torch.full_like(k, float("nan")),
               torch.full_like(v, float("nan")))
        got = sdpa_bwd_noalloc(q, k, v, o, do, lse, *out, **extra)
        torch.cuda.synchronize()
        for name, g, r in zip(("dq", "dk", "dv"), got, ref):
            _same(g, r, f"call {call + 1} {name}")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    dev = torch.device("cuda")
    L = 66000                              # workspace = 64 * 66000 * 4 bytes > 16 MiB
    q = torch.zeros(1, L, 64, 64, device=dev, dtype=torch.bfloat16)
    k = torch.zeros(1, L, 1, 64, device=dev, dtype=torch.bfloat16)
    assert sdpa_bwd_workspace_size(q, k) > NOALLOC_SCRATCH_BYTES
    lse = torch.zeros(1, 64, L, device=dev)
    with pytest.raises(SdpaError) as e:
        sdpa_bwd_noalloc(q, k, k, q, q, lse, torch.empty_like(q), torch.empty_like(k),
                         torch.empty_like(k), causal=True)
    assert e.value.status == 3             # SDPA_ERR_WORKSPACE: nothing launched
