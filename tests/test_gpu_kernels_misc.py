"""GPU checks of the T5 bucket device function (bit-exact against the oracle)
and of the bounded-wait timeout path (no fault, no hang)."""
import numpy as np
import pytest
import torch

from oracle import t5_relative_bucket
from scaled_dot_product_bwd_b200 import (sdpa_debug_wait_timeout, sdpa_exp2_fma,
                                         sdpa_read_device_status,
                                         sdpa_set_wait_limit_ns, sdpa_t5_bucket)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("nb,md,bidir", [(32, 128, True), (32, 128, False), (64, 256, True),
                                         (16, 40, True), (128, 1000, False), (8, 20, True),
                                         (16, 24, True), (8, 20, False), (32, 4096, True),
                                         (128, 20000, True), (64, 40, False), (128, 65, True)])
def test_t5_buckets_bit_exact(nb, md, bidir):
    rel = np.arange(-20000, 20001, dtype=np.int32)
    got = sdpa_t5_bucket(torch.from_numpy(rel).cuda(), nb, md, bidir).cpu().numpy()
    want = t5_relative_bucket(rel, nb, md, bidir)
    assert np.array_equal(got, want), np.nonzero(got != want)[0][:10]


def test_wait_timeout_reports_status_and_context_survives():
    assert sdpa_read_device_status() == 0
    sdpa_set_wait_limit_ns(2_000_000)          # 2 ms
    try:
        sdpa_debug_wait_timeout()
        assert sdpa_read_device_status() == 5  # SDPA_ERR_TIMEOUT, read once then cleared
        assert sdpa_read_device_status() == 0
    finally:
        sdpa_set_wait_limit_ns(2_000_000_000)
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0            # the context is still usable


def test_exp2_fma_within_its_bound():
    # The FMA-pipe exponential against float64 exp2 (and CUDA's exp2f) over the
    # range the kernels feed it: relative error below the stated 1.2e-4.
    x = torch.cat([torch.linspace(-125, 125, 1_000_001), torch.linspace(-0.5, 0.5, 100_001),
                   torch.tensor([-200.0, float("-inf")])]).cuda()
    y = sdpa_exp2_fma(x).double().cpu()
    xs = x.double().cpu()
    ref = torch.exp2(xs)
    rel = ((y[:-2] / ref[:-2]) - 1).abs().max().item()
    assert rel < 1.2e-4, rel
    cuda_rel = ((y[:-2] / torch.exp2(x[:-2]).double().cpu()) - 1).abs().max().item()
    assert cuda_rel < 1.3e-4, cuda_rel
    # inputs below -125 clamp to 2^-125, never wrap into large values
    assert 0 < y[-2].item() < 1e-37 and 0 < y[-1].item() < 1e-37
