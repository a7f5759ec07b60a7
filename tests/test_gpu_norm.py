"""GPU parity of the RMS normalisation between stacked layers against the oracle."""

import numpy as np
import pytest
import torch

import workloads as W
from oracle import formats as F
from oracle import moe as M

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def S():
    import bit_quantized_moe_stq1_b200 as S
    return S


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _check(S, x, eps, inplace=False):
    xb = _bits(x)
    ref = M.rms_norm(F.bf16_decode(xb), eps)
    y = S.rmsnorm_bf16(x, eps, y=x if inplace else None)
    got = F.bf16_decode(_bits(y))
    # FP64 arithmetic on the GPU, then FP32 and bf16 rounding: at most half a bf16 step
    # from the exact value plus the FP32 step of the intermediate
    bound = (2.0 ** -8 + 2.0 ** -23) * np.abs(ref) + 1e-38
    assert np.all(np.abs(got - ref) <= bound), float(np.max(np.abs(got - ref) / bound))
    # and almost always the correctly rounded bf16 value itself
    assert np.mean(got == F.bf16_decode(F.bf16_encode_rne(ref))) > 0.999
    return got


@pytest.mark.parametrize("T,H", [(1, 8), (3, 72), (5, 2056), (32, 6144), (300, 512)])
def test_rmsnorm_matches_oracle(S, T, H):
    x = W.bf16_normal((T, H), 1.0, DEV, 0, "rms", T, H)
    _check(S, x, 1e-6)


def test_rmsnorm_wide_range_inplace_and_zero_rows(S):
    T, H = 6, 6144
    x = W.bf16_normal((T, H), 1.0, DEV, 0, "rmsw")
    x[1] *= 1e30          # squares beyond the FP32 range
    x[2] *= 1e-30
    x[3] = 0              # eps keeps a zero row at zero
    x[4, ::7] = 0
    got = _check(S, x.clone(), 1e-6, inplace=True)
    assert np.all(got[3] == 0)
    _check(S, x, 0.5)


def test_rmsnorm_empty_and_bad_args(S):
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device=DEV)
    assert S.rmsnorm_bf16(x).shape == (0, 64)
    with pytest.raises(RuntimeError):
        S.rmsnorm_bf16(torch.zeros((2, 12), dtype=torch.bfloat16, device=DEV))
