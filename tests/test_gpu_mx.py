"""GPU parity of the W4A8 path (tcgen05 block-scaled GEMM) against the oracle."""

import numpy as np
import pytest
import torch

import workloads as W
from oracle import formats as F
from oracle import moe as M
from mx_checks import check_mxfp8_layer

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def S():
    import bit_quantized_moe_stq1_b200 as S
    return S


def np_bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _gemm_case(S, N, K, Mtok, tag):
    wc, ws = W.mxfp4_random(N, K, DEV, 0, "wc", tag)
    x = W.bf16_normal((Mtok, K), 1.0, DEV, 0, "wx", tag)
    ac, asc = S.mxfp8_quantize_bf16(x)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    y = S.w4a8_gemm(wc, ws, N, K, ac, asc, err=err).cpu().double().numpy()
    assert S.read_error(err) == 0
    rac, ras = F.mxfp8_quantize(F.bf16_decode(np_bits(x)))
    yr, sr = M.w4a8_gemm(wc.cpu().numpy(), ws.cpu().numpy(), rac, ras, N, K)
    err_abs = np.abs(y - yr)
    bound = 1e-3 * sr + 1e-5
    assert np.all(err_abs <= bound), (float(np.max(err_abs / bound)), np.argwhere(err_abs > bound)[:5])


@pytest.mark.parametrize("N,K,Mtok", [(128, 128, 1), (128, 256, 16), (128, 512, 17), (256, 384, 33), (128, 128, 64),
                                      (384, 256, 100), (128, 1024, 200)])
def test_w4a8_gemm_small(S, N, K, Mtok):
    _gemm_case(S, N, K, Mtok, (N, K, Mtok))


def test_w4a8_gemm_single_expert_config(S):
    """128 tokens x K = 6144 -> N = 2048, MXFP4 codes uniform, scales in [118, 127]."""
    _gemm_case(S, 2048, 6144, 128, "cfg1")


def test_w4a8_gemm_zero_and_empty(S):
    N, K, Mtok = 128, 256, 8
    wc = torch.zeros((N, K // 2), dtype=torch.uint8, device=DEV)
    ws = torch.full((N, K // 32), 127, dtype=torch.uint8, device=DEV)
    ac = torch.full((Mtok, K), 0x38, dtype=torch.uint8, device=DEV)
    asc = torch.full((Mtok, K // 32), 127, dtype=torch.uint8, device=DEV)
    y = S.w4a8_gemm(wc, ws, N, K, ac, asc)
    assert torch.all(y == 0)
    # all-ones: e2m1 code 2 (1.0) times e4m3 0x38 (1.0) -> y = K
    wc.fill_(0x22)
    y = S.w4a8_gemm(wc, ws, N, K, ac, asc)
    assert torch.all(y == float(K))
    assert S.w4a8_gemm(wc, ws, N, K, ac[:0], asc[:0]).numel() == 0


# --------------------------------------------------------------------------- MXFP4 MoE layer

def _mx_layer(S, T, H, I, E, k, shared, tag, routing="router", shared_fmt="bf16"):
    g = [W.mxfp4_random(E * I, H, DEV, 0, tag, "g"), W.mxfp4_random(E * I, H, DEV, 0, tag, "u"),
         W.mxfp4_random(E * H, I, DEV, 0, tag, "d")]
    sh = None
    if shared:
        sh = [W.bf16_normal((I, H), 0.02, DEV, 0, tag, "sg"), W.bf16_normal((I, H), 0.02, DEV, 0, tag, "su"),
              W.bf16_normal((H, I), 0.02, DEV, 0, tag, "sd")]
    x = W.bf16_normal((T, H), 1.0, DEV, 0, tag, "x")
    if routing == "router":
        wr = W.bf16_normal((E, H), 0.02, DEV, 0, tag, "r")
        ids, tw, _ = S.moe_router_topk(x, wr, k)
    else:
        ids, tw = W.zipf_routing(T, E, k, DEV, 0, tag, "z")
    desc = S.make_desc(T, H, I, E, k, out_fp32=True)
    ws = torch.zeros(S.moe_workspace_bytes(desc), dtype=torch.uint8, device=DEV)
    y = torch.empty((T, H), dtype=torch.float32, device=DEV)
    sh_mx8 = None
    if sh and shared_fmt == "mx8":
        sh_mx8 = [S.mxfp8_quantize_bf16(m) for m in sh]
        ew = S.ExpertWeights(S.FMT_MXFP4, g[0][0], g[1][0], g[2][0], g[0][1], g[1][1], g[2][1],
                             *(c for c, _ in sh_mx8), sh_fmt=S.SHARED_MXFP8, sh_gate_sc=sh_mx8[0][1],
                             sh_up_sc=sh_mx8[1][1], sh_down_sc=sh_mx8[2][1])
    else:
        ew = S.ExpertWeights(S.FMT_MXFP4, g[0][0], g[1][0], g[2][0], g[0][1], g[1][1], g[2][1],
                             *(sh if sh else (None, None, None)))
    S.moe_expert_forward(desc, x, ids, tw, ew, y, ws)
    assert S.moe_get_device_error(ws) == 0
    P = T * k
    v = lambda r, dt, shp: S.moe_workspace_view(desc, ws, r, dt, shp).cpu().numpy()
    return dict(g=[(a.cpu().numpy(), b.cpu().numpy()) for a, b in g], sh=sh, x=x, ids=ids.cpu().numpy(),
                tw=tw.cpu().double().numpy(), y=y.cpu().double().numpy(),
                xq=v("xq", torch.uint8, (P + T, H)), xs=v("xs", torch.uint8, (P + T, H // 32)),
                hq=v("hq", torch.uint8, (P + T, I)), hs=v("hs", torch.uint8, (P + T, I // 32)),
                sh_mx8=None if sh_mx8 is None else [(c.cpu().numpy(), s_.cpu().numpy()) for c, s_ in sh_mx8],
                h=S.moe_workspace_view(desc, ws, "h", torch.bfloat16, (P + T, I)).float().cpu().double().numpy(),
                Y=v("Y", torch.float32, (P + T, H)).astype(np.float64),
                perm=v("perm", torch.int32, (P,)), inv=v("inv", torch.int32, (P,)))


def _rows(pair, e, R, K):
    c, s = pair
    return c[e * R:(e + 1) * R], s[e * R:(e + 1) * R]


def _check_mx_layer(r, T, H, I, E, k, experts=None):
    def weights(e):
        return (F.mxfp4_unpack(*_rows(r["g"][0], e, I, H), I, H), F.mxfp4_unpack(*_rows(r["g"][1], e, I, H), I, H),
                F.mxfp4_unpack(*_rows(r["g"][2], e, H, I), H, I))
    check_mxfp8_layer(r, T, H, I, E, k, weights, experts)


@pytest.mark.parametrize("T,H,I,E,k,shared", [(5, 512, 256, 8, 2, True), (3, 256, 128 * 2, 4, 4, False),
                                               (40, 512, 256, 4, 4, False), (1000, 512, 256, 2, 1, True),
                                               (481, 256, 256, 1, 1, False)])
def test_moe_mx_small_full_check(S, T, H, I, E, k, shared):
    """Every N tile width: 16 (decode) up to 240 (128 or more tokens per expert; 481 tokens
    on one expert give tiles of 240, 240 and 1)."""
    r = _mx_layer(S, T, H, I, E, k, shared, ("mxs", T, H, I, E, k))
    _check_mx_layer(r, T, H, I, E, k)


@pytest.mark.parametrize("T,H,I,E,k", [(5, 512, 256, 8, 2), (40, 512, 256, 4, 4), (300, 768, 512, 8, 2)])
def test_moe_mx_mxfp8_shared_full_check(S, T, H, I, E, k):
    """MXFP4 layer with the MXFP8 shared expert (N tiles of 16 to 128 tokens)."""
    r = _mx_layer(S, T, H, I, E, k, True, ("mxsh8", T, H, I, E, k), shared_fmt="mx8")
    _check_mx_layer(r, T, H, I, E, k)


def test_moe_mx_decode_shape_sampled(S):
    T, H, I, E, k = 32, 6144, 2048, 256, 8
    r = _mx_layer(S, T, H, I, E, k, True, "mxdec")
    counts = np.bincount(r["ids"].reshape(-1), minlength=E)
    touched = np.flatnonzero(counts)
    sample = np.unique(np.concatenate([touched[np.argsort(-counts[touched], kind="stable")[:2]], touched[::40]]))
    _check_mx_layer(r, T, H, I, E, k, experts=sample)


def test_moe_mx_prefill_shape_sampled(S):
    """4096 tokens, Zipf(1.1) routing over 256 experts, weights Dirichlet(1)."""
    T, H, I, E, k = 4096, 6144, 2048, 256, 8
    r = _mx_layer(S, T, H, I, E, k, False, "mxpre", routing="zipf")
    counts = np.bincount(r["ids"].reshape(-1), minlength=E)
    order = np.argsort(counts, kind="stable")
    sample = [order[-1], order[len(order) // 2], order[np.flatnonzero(counts[order])[0]]]
    _check_mx_layer(r, T, H, I, E, k, experts=sample)
