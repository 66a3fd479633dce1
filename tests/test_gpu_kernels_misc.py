"""GPU checks of the T5 bucket device function (bit-exact against the oracle)
and of the bounded-wait timeout path (no fault, no hang)."""
import numpy as np
import pytest
import torch

from oracle import t5_relative_bucket
from scaled_dot_product_bwd_b200 import (sdpa_debug_wait_timeout, sdpa_read_device_status,
                                         sdpa_set_wait_limit_ns, sdpa_t5_bucket)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("nb,md,bidir", [(32, 128, True), (32, 128, False), (64, 256, True),
                                         (16, 40, True), (128, 1000, False), (8, 20, True)])
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
