"""GPU parity of the per-row FP8 quantiser against the oracle: codes and
scales are integer-valued outputs of fp32 decisions, so they must match bit
for bit."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_long_fp8_b200 as dsa
from sparse_attention_long_fp8_b200 import inputs as dsa_inputs

pytestmark = pytest.mark.gpu


def _rows(n, dim, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(n, dim, generator=g) * torch.exp(torch.randn(n, 1, generator=g) * 3)
    if n >= 4:
        x[0] = 0.0                               # all-zero row: scale 1
        x[1] = -0.0 * x[1].abs()                 # negative zeros keep their sign
        x[2] = 0.0
        x[2, 5] = -3.0                           # one non-zero value: it maps to -448
        x[3] = torch.linspace(-1, 1, dim)        # many values near rounding ties
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("n,dim", [(1, 128), (1003, 128), (777, 64), (517, 32)])
def test_quantiser_bit_exact_against_oracle(n, dim):
    x = _rows(n, dim, seed=n + dim)
    xd = x.cuda()
    codes = torch.empty(n, dim, dtype=torch.uint8, device="cuda")
    scales = torch.empty(n, device="cuda")
    dsa.dsa_quantize_e4m3(xd, codes, scales)
    dsa.dsa_check()
    want_c, want_s = oracle.quantize_rows(x)
    got_c, got_s = codes.cpu().numpy(), scales.cpu().numpy()
    assert np.array_equal(got_s.view(np.uint32), want_s.view(np.uint32))
    bad = np.argwhere(got_c != want_c)
    assert len(bad) == 0, f"{len(bad)} codes differ, first {bad[:4].tolist()}"


def test_quantiser_on_indexer_shaped_queries_matches_generator():
    """q rows of [T, H^I, d^I] = [256, 64, 128]: the same bytes the input
    generator (torch's cast) produces."""
    g = torch.Generator().manual_seed(11)
    x = torch.randn(256, 64, 128, generator=g).to(torch.bfloat16)
    codes = torch.empty(256, 64, 128, dtype=torch.uint8, device="cuda")
    scales = torch.empty(256, 64, device="cuda")
    dsa.dsa_quantize_e4m3(x.cuda(), codes, scales)
    dsa.dsa_check()
    tc, ts = dsa_inputs.quantize_e4m3_rows(x)
    assert torch.equal(codes.cpu(), tc) and torch.equal(scales.cpu(), ts)
