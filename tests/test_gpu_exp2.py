"""The sparse kernel's FMA-pipe exponential run on the GPU (through
vsa_selftest_exp2) against float64 2^x and against the float32 model of its
steps in exp2_fit."""
import numpy as np
import pytest
import torch

from block_sparse_attention_15_b200 import binding as vsa
from block_sparse_attention_15_b200 import exp2_fit as E

pytestmark = pytest.mark.gpu
BOUND = 7.5e-5


def test_device_exp2_within_bound_and_matches_model():
    rng = np.random.default_rng(11)
    x = np.concatenate([
        np.linspace(-130.0, 33.0, 2_000_001),
        rng.uniform(-120.0, 32.0, 500_000),
        np.arange(-120, 33) + 0.5,
        np.nextafter(np.arange(-120, 33) + 0.5, -np.inf),
        np.nextafter(np.arange(-120, 33) + 0.5, np.inf),
    ]).astype(np.float32)
    y, mismatch = vsa.selftest_exp2(torch.from_numpy(x).cuda())
    y = y.cpu().numpy()
    assert mismatch == 0, "the two halves of the packed evaluation disagree"
    inside = x >= -120.0
    rel = np.abs(y[inside].astype(np.float64) / np.exp2(x[inside].astype(np.float64)) - 1.0)
    assert rel.max() <= BOUND, rel.max()
    assert np.all(y[~inside] <= 2.0 ** -119)
    # the model's float64-then-float32 rounding may differ from a fused
    # multiply-add by one float32 ulp at most
    model = E.exp2_model(x)
    ulps = np.abs(y.view(np.int32).astype(np.int64) - model.view(np.int32).astype(np.int64))
    assert ulps.max() <= 1, ulps.max()
