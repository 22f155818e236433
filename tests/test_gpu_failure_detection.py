"""Failure detection on the GPU without a fault: a bounded device wait that can never be
satisfied gives up after its limit, the host reads PF_ERR_TIMEOUT from the status word, and
the context stays usable afterwards."""
import time

import numpy as np
import pytest
import torch

import oracle
import patch_attention_b200 as pa

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_the_device_stays_usable():
    t0 = time.time()
    assert pa.pf_selftest_bounded_wait(20_000_000) == pa.PF_ERR_TIMEOUT  # 20 ms
    assert time.time() - t0 < 5.0
    # the status word was cleared by the read
    assert pa.pf_selftest_bounded_wait(1_000_000) == pa.PF_ERR_TIMEOUT
    # and the device still computes: one guidance combine checked against the oracle
    g = torch.Generator(device="cuda").manual_seed(0)
    u = torch.randn(2, 4096, device="cuda", generator=g)
    c = u + 0.5 * torch.randn(2, 4096, device="cuda", generator=g)
    _, _, rel = pa.cfg_combine_relmae(c, u, 7.0)
    torch.cuda.synchronize()
    _, _, ref_rel = oracle.rel_mae(c.double().cpu().numpy(), u.double().cpu().numpy())
    np.testing.assert_allclose(rel.double().cpu().numpy(), ref_rel, rtol=1e-5)
