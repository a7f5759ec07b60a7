"""GPU parity of the STQ1_0 GEMV (single matrix) against the oracle:
|y - y_ref| <= 1e-3 * sum |w x| + 1e-5 per element."""

import numpy as np
import pytest
import torch

import workloads as W
from oracle import formats as F
from oracle import moe as M

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_REL, TOL_ABS = 1e-3, 1e-5


@pytest.fixture(scope="module")
def S():
    import bit_quantized_moe_stq1_b200 as S
    return S


def _check(y, yr, sr):
    err = np.abs(y - yr)
    bound = TOL_REL * sr + TOL_ABS
    assert np.all(err <= bound), float(np.max(err / bound))


@pytest.mark.parametrize("rows,K,n", [(16, 256, 1), (16, 512, 3), (48, 768, 9), (64, 1024, 17), (2048, 6144, 1),
                                      (6144, 2048, 8)])
def test_stq1_gemv_vs_oracle(S, rows, K, n):
    w = W.stq_grid_weights(rows, K, DEV, 0, "gw", rows, K)
    x = W.bf16_normal((n, K), 1.0, DEV, 0, "gx", n, K)
    packed = S.stq1_pack(w)
    y = S.stq1_gemv(packed, rows, K, x).cpu().double().numpy()
    # the oracle reads the generator's weights through its own pack/unpack
    wp = F.stq1_pack(w.cpu().numpy())
    xb = x.view(torch.int16).cpu().numpy().view(np.uint16)
    yr, sr = M.stq1_gemv(wp, rows, K, xb)
    _check(y, yr, sr)


def test_stq1_gemv_special_cases(S):
    rows, K = 32, 512
    # d = 1, all lanes positive with zero lane 3: y = sum of x over lanes 0..2
    code = np.full((rows, K // 256, 64), 24, dtype=np.int64)
    dbits = np.full((rows, K // 256), F.fp16_encode_rne(1.0), np.uint16)
    packed = torch.from_numpy(F.stq1_layout(code, dbits)).to(DEV)
    x = W.bf16_normal((2, K), 1.0, DEV, 0, "sp")
    y = S.stq1_gemv(packed, rows, K, x).cpu().double().numpy()
    xd = x.float().double().cpu().numpy()
    ref = np.array([[sum(xd[t, k] for k in range(K) if k % 4 != 3)] * rows for t in range(2)])
    _check(y, ref, np.abs(xd).sum(1, keepdims=True).repeat(rows, 1))
    # one-hot activations pick out one weight column exactly
    w = W.stq_grid_weights(rows, K, DEV, 0, "oh")
    pk = S.stq1_pack(w)
    eye = torch.zeros((8, K), device=DEV)
    cols = [0, 1, 63, 64, 255, 256, 300, 511]
    for i, c in enumerate(cols):
        eye[i, c] = 1.0
    y = S.stq1_gemv(pk, rows, K, eye.to(torch.bfloat16)).cpu().numpy()
    assert np.array_equal(y, w[:, cols].t().cpu().numpy())
    # all-zero weights and empty token batch
    z = S.stq1_pack(torch.zeros((16, 256), device=DEV))
    assert torch.all(S.stq1_gemv(z, 16, 256, x[:, :256].contiguous()) == 0)
    assert S.stq1_gemv(pk, rows, K, x[:0]).numel() == 0


def test_bounded_wait_reports_timeout_and_context_survives(S):
    """A wait that nothing satisfies runs out (about two seconds), records STQ_ERR_TIMEOUT
    and returns; the context then runs a GEMV as before."""
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    S.wait_selftest(err)
    assert S.read_error(err) == -8
    w = W.stq_grid_weights(32, 256, DEV, 0, "wait")
    x = W.bf16_normal((1, 256), 1.0, DEV, 0, "waitx")
    packed = S.stq1_pack(w)
    y = S.stq1_gemv(packed, 32, 256, x).cpu().double().numpy()
    yr, sr = M.stq1_gemv(packed.cpu().numpy(), 32, 256, x.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))
    assert np.all(np.abs(y - yr) <= 1e-3 * sr + 1e-5)
