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


def _bits16(t):
    return t.contiguous().view(torch.int16).cpu().numpy()


@pytest.mark.parametrize("T,H,I,E,k", [(32, 6144, 256, 16, 4), (5, 768, 256, 8, 2), (3, 24576, 256, 4, 2)])
def test_norm_out_matches_the_separate_normalisation(S, T, H, I, E, k):
    """moe_desc.norm_out: the combine with the RMS normalisation fused (or, past the fused
    kernel's row width, the two launches) gives the bits of the unnormalised layer output
    followed by stq_rmsnorm_bf16, with the residual read from x and with y aliasing x."""
    tag = ("normout", T, H, I, E, k)
    gw = [W.stq_grid_weights(E * I, H, DEV, 0, *tag, "g"), W.stq_grid_weights(E * I, H, DEV, 0, *tag, "u"),
          W.stq_grid_weights(E * H, I, DEV, 0, *tag, "d")]
    packs = [S.stq1_pack(m) for m in gw]
    sh = [W.bf16_normal((I, H), 0.02, DEV, 0, *tag, "sg"), W.bf16_normal((I, H), 0.02, DEV, 0, *tag, "su"),
          W.bf16_normal((H, I), 0.02, DEV, 0, *tag, "sd")]
    ew = S.ExpertWeights(S.FMT_STQ1_0, *packs, None, None, None, *sh)
    x = W.bf16_normal((T, H), 1.0, DEV, 0, *tag, "x")
    ids, tw = W.uniform_routing(T, E, k, DEV, 0, *tag, "ids")
    plain = S.make_desc(T, H, I, E, k, add_residual=True)
    fused = S.make_desc(T, H, I, E, k, add_residual=True, norm_eps=W.STACK_RMS_EPS)
    ws = torch.zeros(S.moe_workspace_bytes(plain), dtype=torch.uint8, device=DEV)
    assert S.moe_workspace_bytes(fused) == S.moe_workspace_bytes(plain)
    ref = torch.empty((T, H), dtype=torch.bfloat16, device=DEV)
    S.moe_expert_forward(plain, x, ids, tw, ew, ref, ws)
    S.rmsnorm_bf16(ref, W.STACK_RMS_EPS, y=ref)
    got = torch.empty_like(ref)
    S.moe_expert_forward(fused, x, ids, tw, ew, got, ws)
    assert S.moe_get_device_error(ws) == 0
    assert np.array_equal(_bits16(got), _bits16(ref))
    inplace = x.clone()
    S.moe_expert_forward(fused, inplace, ids, tw, ew, inplace, ws)
    assert np.array_equal(_bits16(inplace), _bits16(ref))
