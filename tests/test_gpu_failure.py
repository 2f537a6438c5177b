"""Failure detection on the GPU without a fault: a bounded wait that nothing
completes must come back as DSA_ERR_TIMEOUT through dsa_check, and the
context must stay usable for the next call."""
import time

import pytest
import torch

import sparse_attention_long_fp8_b200 as dsa

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    dsa.dsa_check()                                  # start from a clean error word
    t0 = time.perf_counter()
    dsa.dsa_selftest_wait_timeout(100)
    with pytest.raises(dsa.DsaError) as err:
        dsa.dsa_check()
    elapsed = time.perf_counter() - t0
    assert err.value.status == dsa.DSA_ERR_TIMEOUT
    assert 0.09 < elapsed < 5.0                      # the wait gave up after its limit
    dsa.dsa_check()                                  # the word was cleared
    # the context still runs real work
    cfg = dsa.CONFIGS["tiny"]
    inp = dsa.make_inputs(cfg, seed=0, device="cuda")
    res = dsa.forward(inp, cfg)
    dsa.dsa_check()
    assert torch.isfinite(res["out"]).all()
