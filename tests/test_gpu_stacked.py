"""GPU parity of the stacked decode (eight MoE layers of hidden 6144, 256 experts of
intermediate 2048, top-8, 32 tokens; layers 1, 3, 5, 7 STQ1_0 and 2, 4, 6, 8
MXFP4-W/MXFP8-A; a BF16 router and a BF16 shared expert per layer; residual add and
RMS normalisation between layers), built by the benchmark's own workload class and
checked layer by layer against the oracle, each layer fed the GPU's own layer input:

* router: top-8 set and weights against the oracle's softmax/top-k (near-ties skipped);
* grouping: exact;
* STQ1_0 layers (decode regime, T = 32): gate/up + SwiGLU (propagated bound plus one
  BF16 step) and down (1e-3 S + 1e-5 on the GPU's own h) for sampled experts and the
  shared expert;
* MXFP4 layers: activation quantisation in sorted pair order (bit-exact), SwiGLU + MXFP8
  h, down, for sampled experts; the shared expert;
* combine with the residual, rounded to BF16: the FP32 sum bound plus half a BF16 step;
* RMS normalisation of the GPU's layer output: half a BF16 step plus one FP32 step.

Finally the benchmark's own step function must give the same bits as the layer-by-layer
chain (every kernel on the path is deterministic)."""

import numpy as np
import pytest
import torch

import workloads as W
from oracle import formats as F
from oracle import moe as M
from mx_checks import check_bf16_gate_up, check_down, check_mxfp8_layer

pytestmark = pytest.mark.gpu
DEV = "cuda"
T, H, I, E, K = 32, W.HIDDEN, W.INTER, W.EXPERTS, W.TOPK


@pytest.fixture(scope="module")
def S():
    import bit_quantized_moe_stq1_b200 as S
    return S


@pytest.fixture(scope="module")
def stack(S):
    import bench

    wl = bench.MoeLayers(S, torch.device(DEV), "stacked_decode", T, ("stq", "mx") * 4, True, True, True, E)
    yield wl
    del wl
    torch.cuda.empty_cache()


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _stq_expert(wl, l, e):
    """Float64 gate [I, H], up [I, H], down [H, I] of expert e of STQ1_0 layer l, drawn
    again from the seeded generator the workload packed them from (16 experts per draw)."""
    e0 = 16 * (e // 16)
    out = []
    for which, rows, cols in (("g", I, H), ("u", I, H), ("d", H, I)):
        wf = W.stq_grid_weights(16 * rows, cols, DEV, 0, wl.name, l, which, e0)
        out.append(wf[(e - e0) * rows:(e - e0 + 1) * rows].double().cpu().numpy())
        del wf
    return out


def _mx_expert(Lw, e):
    def rows(codes, scales, R, Kd):
        return F.mxfp4_unpack(codes[e * R:(e + 1) * R].cpu().numpy(), scales[e * R:(e + 1) * R].cpu().numpy(), R, Kd)
    return (rows(Lw.gate, Lw.gate_sc, I, H), rows(Lw.up, Lw.up_sc, I, H), rows(Lw.down, Lw.down_sc, H, I))


def _sample(ids):
    counts = np.bincount(ids.reshape(-1), minlength=E)
    touched = np.flatnonzero(counts)
    busiest = touched[np.argsort(-counts[touched], kind="stable")[:2]]
    return np.unique(np.concatenate([busiest, touched[:: max(1, touched.size // 3)]]))


def _check_router(x_bits, wr, ids, tw):
    ri, rw, p = M.router_topk(x_bits, _bits(wr), K)
    for t in range(T):
        ps = np.sort(p[t])[::-1]
        if ps[K - 1] - ps[K] < 1e-6 * ps[0]:
            continue
        assert set(ids[t]) == set(ri[t]), t
        for j, e in enumerate(ids[t]):
            assert abs(tw[t, j] - rw[t, list(ri[t]).index(e)]) <= 1e-5


def _check_combine_bf16_residual(y_bf16, Y, inv, tw, xd):
    """y = bf16(sum_s w Y[inv] + Y_shared + x) in FP32: the FP32 sum bound plus half a
    BF16 step of the result."""
    P = T * K
    yc = np.zeros((T, H))
    mag = np.zeros((T, H))
    for t in range(T):
        for s in range(K):
            term = tw[t, s] * Y[inv[t * K + s]]
            yc[t] += term
            mag[t] += np.abs(term)
        yc[t] += Y[P + t] + xd[t]
        mag[t] += np.abs(Y[P + t]) + np.abs(xd[t])
    err = np.abs(y_bf16 - yc)
    bound = 1e-6 * mag + 2.0 ** -8 * (np.abs(yc) + 1e-6 * mag) + 1e-30
    assert np.all(err <= bound), float(np.max(err / bound))


def _check_rmsnorm(pre_bits, post_bits):
    ref = M.rms_norm(F.bf16_decode(pre_bits), W.STACK_RMS_EPS)
    got = F.bf16_decode(post_bits)
    bound = (2.0 ** -8 + 2.0 ** -23) * np.abs(ref) + 1e-38
    assert np.all(np.abs(got - ref) <= bound), float(np.max(np.abs(got - ref) / bound))


def test_stacked_decode_layer_by_layer(S, stack):
    wl = stack
    P = T * K
    ws, desc = wl.ws, wl.desc
    assert desc.T == T and desc.add_residual == 1 and desc.out_fp32 == 0
    cur = wl.x[0].clone()
    x0 = cur.clone()
    view = lambda r, dt, shp: S.moe_workspace_view(desc, ws, r, dt, shp)
    for l, L in enumerate(wl.layers):
        xin_bits = _bits(cur)
        xd = F.bf16_decode(xin_bits)
        ids, tw, _ = S.moe_router_topk(cur, L["wr"], K)
        y = torch.empty((T, H), dtype=torch.bfloat16, device=DEV)
        S.moe_expert_forward(desc, cur, ids, tw, L["w"], y, ws)
        assert S.moe_get_device_error(ws) == 0, l
        ids_n, tw_n = ids.cpu().numpy(), tw.cpu().double().numpy()
        _check_router(xin_bits, L["wr"], ids_n, tw_n)
        counts, offsets, perm, inv = M.permute(ids_n, E)
        assert np.array_equal(view("perm", torch.int32, (P,)).cpu().numpy(), perm)
        assert np.array_equal(view("inv", torch.int32, (P,)).cpu().numpy(), inv)
        h = view("h", torch.bfloat16, (P + T, I)).float().cpu().double().numpy()
        Y = view("Y", torch.float32, (P + T, H)).cpu().double().numpy()
        sample = _sample(ids_n)
        if L["fmt"] == "stq":
            for e in sample:
                pos = np.arange(offsets[e], offsets[e + 1])
                Wg, Wu, Wd = _stq_expert(wl, l, int(e))
                check_bf16_gate_up(Wg, Wu, xd[perm[pos] // K], h[pos])
                check_down(Wd, h[pos], Y[pos], (l, int(e)))
            sg, su, sd = (m.float().double().cpu().numpy() for m in L["sh_bf16"])
            check_bf16_gate_up(sg, su, xd, h[P:P + T])
            check_down(sd, h[P:P + T], Y[P:P + T], (l, "shared"))
        else:
            r = dict(ids=ids_n, tw=tw_n, x=cur, sh=L["sh_bf16"], sh_mx8=None, y=None, h=h, Y=Y,
                     perm=perm, inv=inv,
                     xq=view("xq", torch.uint8, (P + T, H)).cpu().numpy(),
                     xs=view("xs", torch.uint8, (P + T, H // 32)).cpu().numpy(),
                     hq=view("hq", torch.uint8, (P + T, I)).cpu().numpy(),
                     hs=view("hs", torch.uint8, (P + T, I // 32)).cpu().numpy())
            check_mxfp8_layer(r, T, H, I, E, K, lambda e: _mx_expert(L["w"], int(e)), sample)
        _check_combine_bf16_residual(F.bf16_decode(_bits(y)), Y, inv, tw_n, xd)
        pre = _bits(y)
        S.rmsnorm_bf16(y, W.STACK_RMS_EPS, y=y)
        _check_rmsnorm(pre, _bits(y))
        cur = y
    # the benchmark's step (the timed chain, with its own scratch buffers) gives the same bits
    out = wl.step(0, x=x0)
    torch.cuda.synchronize()
    assert torch.equal(out, cur)
