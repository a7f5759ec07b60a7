"""GPU parity of the format kernels against the oracle: bit-exact, via the C ABI."""

import numpy as np
import pytest
import torch

import workloads as W
from oracle import formats as F

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    import bit_quantized_moe_stq1_b200 as S
    return S


DEV = "cuda"


@pytest.mark.parametrize("rows,K", [(16, 256), (48, 768), (2048, 6144), (6144, 2048)])
def test_stq1_pack_grid_bitexact(S, rows, K):
    w = W.stq_grid_weights(rows, K, DEV, 0, "pk", rows, K)
    got = S.stq1_pack(w).cpu().numpy()
    ref = F.stq1_pack(w.cpu().numpy())
    assert got.size == rows * K // 256 * 42
    assert np.array_equal(got, ref)
    back = S.stq1_unpack(torch.from_numpy(ref).to(DEV), rows, K).cpu().numpy()
    assert np.array_equal(back.view(np.uint32), w.cpu().numpy().view(np.uint32))


def test_stq1_pack_off_grid_and_ties(S):
    rows, K = 32, 512
    w = W.float_normal((rows, K), 0.05, DEV, 0, "offgrid")
    w[0, 0:4] = torch.tensor([0.1, -0.1, 0.1, 0.1])
    w[1, 4:8] = torch.tensor([0.3, 0.2, -0.2, 0.2])
    w[2, 8:12] = torch.tensor([-0.0, 0.0, 1.0, -1.0])
    w[3, 256:512] = 0.0                      # d = 0 block
    w[4, 0:256] = 1e-7                       # subnormal FP16 d
    got = S.stq1_pack(w).cpu().numpy()
    assert np.array_equal(got, F.stq1_pack(w.cpu().numpy()))


def test_stq1_unpack_canonical_all_codes(S):
    rows, K = 32, 512
    codes = (np.arange(rows * 2 * 64).reshape(rows, 2, 64) * 7 + 3) % 32
    dvals = np.array([0.0, 2.0 ** -24, 1.0, 65504.0] * 16)[:rows * 2].reshape(rows, 2)
    dbits = F.fp16_encode_rne(dvals)
    codes = np.where((dvals == 0)[:, :, None], 0, codes)
    b = F.stq1_layout(codes, dbits)
    got = S.stq1_unpack(torch.from_numpy(b).to(DEV), rows, K).cpu().numpy()
    ref = F.stq1_unpack(b, rows, K).astype(np.float32)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    again = S.stq1_pack(torch.from_numpy(got).to(DEV)).cpu().numpy()
    assert np.array_equal(again, b)


def test_stq1_pack_nonfinite_sets_error(S):
    w = torch.zeros((16, 256), device=DEV)
    w[3, 5] = float("nan")
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    S.stq1_pack(w, err=err)
    assert S.read_error(err) == -4
    assert S.read_error(err) == 0
    w[3, 5] = 7.0e4
    S.stq1_pack(w, err=err)
    assert S.read_error(err) == -4


@pytest.mark.parametrize("rows,K", [(4, 64), (64, 6144), (2048, 2048)])
def test_mxfp4_pack_unpack_bitexact(S, rows, K):
    w = W.float_normal((rows, K), 1.0, DEV, 0, "mx", rows, K)
    w = w * torch.exp2(torch.randint(-30, 30, (rows, 1), device=DEV).float())
    w[0, :32] = 0.0
    w[0, 1] = -0.0
    w[0, 32:64] = torch.tensor([6.0, -0.1, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -5.0] + [0.0] * 22)
    c, s = S.mxfp4_pack(w)
    rc, rs = F.mxfp4_pack(w.cpu().numpy())
    assert np.array_equal(c.cpu().numpy(), rc) and np.array_equal(s.cpu().numpy(), rs)
    u = S.mxfp4_unpack(c, s, rows, K).cpu().numpy()
    ru = F.mxfp4_unpack_f32(rc, rs, rows, K)
    assert np.array_equal(u.view(np.uint32), ru.view(np.uint32))


def test_mxfp4_unpack_edge_scales(S):
    rows, K = 2, 64
    codes = (np.arange(64).reshape(2, 32) * 9 % 256).astype(np.uint8)
    scales = np.array([[0, 254], [127, 255]], dtype=np.uint8)
    got = S.mxfp4_unpack(torch.from_numpy(codes.copy()).to(DEV), torch.from_numpy(scales).to(DEV), rows, K).cpu().numpy()
    ref = F.mxfp4_unpack_f32(codes, scales, rows, K)
    fin = ~np.isnan(ref)
    assert np.array_equal(np.isnan(got), ~fin)
    assert np.array_equal(got[fin].view(np.uint32), ref[fin].view(np.uint32))


def test_mxfp4_random_workload_roundtrip(S):
    c, s = W.mxfp4_random(256, 6144, DEV, 0, "w4")
    u = S.mxfp4_unpack(c, s, 256, 6144).cpu().numpy()
    ru = F.mxfp4_unpack_f32(c.cpu().numpy(), s.cpu().numpy(), 256, 6144)
    assert np.array_equal(u.view(np.uint32), ru.view(np.uint32))


def _all_bf16_groups():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    x = np.zeros((65536, 64), dtype=np.uint16)
    x[:, 0] = bits                                # own group max (or NaN/Inf group)
    x[:, 32] = bits
    x[:, 33] = F.bf16_encode_rne(np.array([1.0]))[0]   # companion amax 1.0
    return x


def test_mxfp8_quant_exhaustive_bitexact(S):
    xb = _all_bf16_groups()
    xt = torch.from_numpy(xb.view(np.int16)).to(DEV).view(torch.bfloat16)
    c, s = S.mxfp8_quantize_bf16(xt)
    rc, rs = F.mxfp8_quantize(F.bf16_decode(xb))
    c, s = c.cpu().numpy(), s.cpu().numpy()
    bad = np.flatnonzero(~np.all(c == rc, axis=1) | ~np.all(s == rs, axis=1))
    assert bad.size == 0, [(hex(int(xb[i, 0])), c[i, :2], rc[i, :2], s[i], rs[i]) for i in bad[:8]]


def test_mxfp8_quant_activation_workload(S):
    x = W.bf16_normal((4096, 6144), 1.0, DEV, 0, "act")
    c, s = S.mxfp8_quantize_bf16(x)
    xb = x.view(torch.int16).cpu().numpy().view(np.uint16)
    rc, rs = F.mxfp8_quantize(F.bf16_decode(xb[:512]))
    assert np.array_equal(c[:512].cpu().numpy(), rc) and np.array_equal(s[:512].cpu().numpy(), rs)
    rc2, rs2 = F.mxfp8_quantize(F.bf16_decode(xb[-7:]))
    assert np.array_equal(c[-7:].cpu().numpy(), rc2) and np.array_equal(s[-7:].cpu().numpy(), rs2)


def test_mxfp8_quant_many_rows_ragged(S):
    """4099 rows: CTAs of 8 rows with a 3-row tail, every row checked."""
    x = W.bf16_normal((4099, 512), 1.0, DEV, 0, "act-ragged")
    c, s = S.mxfp8_quantize_bf16(x)
    rc, rs = F.mxfp8_quantize(F.bf16_decode(x.view(torch.int16).cpu().numpy().view(np.uint16)))
    assert np.array_equal(c.cpu().numpy(), rc) and np.array_equal(s.cpu().numpy(), rs)


def _imp(K, tag):
    return torch.exp(W.float_normal((K,), 1.0, DEV, 0, "imp", tag)).contiguous()


@pytest.mark.parametrize("rows,K,dist,imp", [(16, 256, "normal", False), (32, 768, "normal", True),
                                             (48, 512, "laplace", True), (16, 6144, "outlier", True),
                                             (2048, 6144, "normal", True)])
def test_stq1_pack_ls_bitexact(S, rows, K, dist, imp):
    """The least-squares encoder's bytes equal the oracle's (FP64 decisions on both sides)."""
    w = W.float_normal((rows, K), 0.02, DEV, 0, "ls", rows, K, dist)
    if dist == "laplace":
        w = w * torch.log(1.0 / W.float_normal((rows, K), 1.0, DEV, 0, "lsu", rows).abs().clamp_min(1e-3))
    elif dist == "outlier":
        w[:, ::97] *= 40.0
    v = _imp(K, (rows, K)) if imp else None
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    got = S.stq1_pack_ls(w.contiguous(), v, err=err).cpu().numpy()
    assert S.read_error(err) == 0
    ref = F.stq1_pack_ls(w.cpu().numpy(), None if v is None else v.cpu().numpy())
    assert np.array_equal(got, ref), int(np.count_nonzero(got != ref))


def test_stq1_pack_ls_errors(S):
    w = W.float_normal((16, 256), 0.02, DEV, 0, "lserr")
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    S.stq1_pack_ls(w, -torch.ones(256, device=DEV), err=err)
    assert S.read_error(err) == -1
    w[2, 7] = float("inf")
    S.stq1_pack_ls(w, err=err)
    assert S.read_error(err) == -4
    assert S.stq1_pack_ls(w[:0]).numel() == 0
