"""GPU parity of the MoE layer steps against the oracle, stage by stage:
grouping (exact), router (top-k set exact away from near-ties), gate/up + SwiGLU
(propagated bound), down and shared expert (1e-3 * S + 1e-5 on the GPU's own h),
combine (FP32 sum of the GPU's own expert outputs)."""

import numpy as np
import pytest
import torch

import workloads as W
from oracle import formats as F
from oracle import moe as M
from mx_checks import check_mx8_shared, check_mxfp8_layer

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def S():
    import bit_quantized_moe_stq1_b200 as S
    return S


def np_bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


# --------------------------------------------------------------------------- grouping


@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (8, 8, 256), (32, 8, 256), (4096, 8, 256), (5, 3, 7), (300, 8, 1024)])
def test_permute_exact(S, T, k, E):
    if T * k >= 4096 * 8:
        ids, _ = W.zipf_routing(T, E, k, DEV, 0, "pz")
    else:
        g = W.generator(DEV, 0, "pu", T, k, E)
        ids = torch.randint(0, E, (T, k), generator=g, device=DEV, dtype=torch.int32)
    out = S.moe_permute(ids, E)
    counts, offsets, perm, inv = M.permute(ids.cpu().numpy(), E)
    assert np.array_equal(out["counts"].cpu().numpy(), counts)
    assert np.array_equal(out["offsets"].cpu().numpy(), offsets)
    assert np.array_equal(out["perm"].cpu().numpy(), perm)
    assert np.array_equal(out["inv"].cpu().numpy(), inv)
    touched = np.flatnonzero(counts)
    assert int(out["ntouched"].item()) == touched.size
    assert np.array_equal(out["tlist"].cpu().numpy()[:touched.size], touched)


def test_permute_bad_ids_and_empty(S):
    ids = torch.tensor([[0, 300], [-1, 2]], dtype=torch.int32, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = S.moe_permute(ids, 256, err=err)
    assert S.read_error(err) == -6
    assert out["inv"].cpu().tolist() == [0, -1, -1, 1]
    assert out["counts"].sum().item() == 2
    out = S.moe_permute(torch.zeros((0, 8), dtype=torch.int32, device=DEV), 256)
    assert int(out["ntouched"].item()) == 0 and int(out["offsets"][-1].item()) == 0


# --------------------------------------------------------------------------- router


@pytest.mark.parametrize("T,H,E,k", [(8, 6144, 256, 8), (32, 6144, 256, 8), (3, 512, 20, 4)])
def test_router_topk(S, T, H, E, k):
    x = W.bf16_normal((T, H), 1.0, DEV, 0, "rx", T)
    wr = W.bf16_normal((E, H), 0.02, DEV, 0, "rw", E)
    ids, w, logits = S.moe_router_topk(x, wr, k)
    ri, rw, p = M.router_topk(np_bits(x), np_bits(wr), k)
    _, lr = M.router_probs(np_bits(x), np_bits(wr))
    sl = np.abs(F.bf16_decode(np_bits(x))) @ np.abs(F.bf16_decode(np_bits(wr))).T
    assert np.all(np.abs(logits.cpu().double().numpy() - lr) <= 1e-3 * sl + 1e-5)
    ids, w = ids.cpu().numpy(), w.cpu().double().numpy()
    for t in range(T):
        ps = np.sort(p[t])[::-1]
        if ps[k - 1] - ps[k] < 1e-6 * ps[0]:
            continue                      # near-tie at the k-th place: any valid choice
        assert set(ids[t]) == set(ri[t])
        for j, e in enumerate(ids[t]):
            assert abs(w[t, j] - rw[t, list(ri[t]).index(e)]) <= 1e-5
        assert abs(w[t].sum() - 1.0) < 1e-5


def test_router_nonfinite_inputs_give_valid_ids(S):
    T, H, E, k = 4, 512, 64, 8
    x = W.bf16_normal((T, H), 1.0, DEV, 0, "rnf")
    x[1, 7] = float("nan")
    x[2, 3] = float("inf")
    x[3, :] = float("nan")
    wr = W.bf16_normal((E, H), 0.02, DEV, 0, "rnfw")
    ids, w, _ = S.moe_router_topk(x, wr, k)
    ids, w = ids.cpu().numpy(), w.cpu().numpy()
    assert ids.min() >= 0 and ids.max() < E
    for t in range(T):
        assert len(set(ids[t])) == k
    assert np.all(np.isfinite(w)) and np.allclose(w.sum(1), 1.0, atol=1e-5)


# --------------------------------------------------------------------------- STQ1_0 MoE layer


def _make_layer(S, T, H, I, E, k, shared, tag):
    gw = [W.stq_grid_weights(E * I, H, DEV, 0, tag, "g"), W.stq_grid_weights(E * I, H, DEV, 0, tag, "u"),
          W.stq_grid_weights(E * H, I, DEV, 0, tag, "d")]
    packs = [S.stq1_pack(m) for m in gw]
    sh = None
    if shared:
        sh = [W.bf16_normal((I, H), 0.02, DEV, 0, tag, "sg"), W.bf16_normal((I, H), 0.02, DEV, 0, tag, "su"),
              W.bf16_normal((H, I), 0.02, DEV, 0, tag, "sd")]
    wr = W.bf16_normal((E, H), 0.02, DEV, 0, tag, "r")
    x = W.bf16_normal((T, H), 1.0, DEV, 0, tag, "x")
    return gw, packs, sh, wr, x


def _run_layer(S, T, H, I, E, k, shared, tag, residual=False, ids=None, tw=None, x=None, regime=None,
               shared_fmt="bf16"):
    gw, packs, sh, wr, x0 = _make_layer(S, T, H, I, E, k, shared, tag)
    x = x0 if x is None else x
    if ids is None:
        ids, tw, _ = S.moe_router_topk(x, wr, k)
    regime = S.REGIME_DECODE if regime is None else regime
    desc = S.make_desc(T, H, I, E, k, out_fp32=True, add_residual=residual, regime=regime)
    ws = torch.zeros(S.moe_workspace_bytes(desc), dtype=torch.uint8, device=DEV)
    y = torch.empty((T, H), dtype=torch.float32, device=DEV)
    sh_mx8 = None
    if sh and shared_fmt == "mx8":
        sh_mx8 = [S.mxfp8_quantize_bf16(m) for m in sh]
        ew = S.ExpertWeights(S.FMT_STQ1_0, *packs, None, None, None, *(c for c, _ in sh_mx8),
                             sh_fmt=S.SHARED_MXFP8, sh_gate_sc=sh_mx8[0][1], sh_up_sc=sh_mx8[1][1],
                             sh_down_sc=sh_mx8[2][1])
    else:
        ew = S.ExpertWeights(S.FMT_STQ1_0, *packs, *(None, None, None),
                             *(sh if sh else (None, None, None)))
    S.moe_expert_forward(desc, x, ids, tw, ew, y, ws)
    assert S.moe_get_device_error(ws) == 0
    P = T * k
    st = dict(
        h=S.moe_workspace_view(desc, ws, "h", torch.bfloat16, (P + T, I)).float().cpu().double().numpy(),
        Y=S.moe_workspace_view(desc, ws, "Y", torch.float32, (P + T, H)).cpu().double().numpy(),
        perm=S.moe_workspace_view(desc, ws, "perm", torch.int32, (P,)).cpu().numpy(),
        inv=S.moe_workspace_view(desc, ws, "inv", torch.int32, (P,)).cpu().numpy(),
        offsets=S.moe_workspace_view(desc, ws, "offsets", torch.int32, (E + 1,)).cpu().numpy(),
        xq=S.moe_workspace_view(desc, ws, "xq", torch.uint8, (P + T, H)).cpu().numpy(),
        xs=S.moe_workspace_view(desc, ws, "xs", torch.uint8, (P + T, H // 32)).cpu().numpy(),
        hq=S.moe_workspace_view(desc, ws, "hq", torch.uint8, (P + T, I)).cpu().numpy(),
        hs=S.moe_workspace_view(desc, ws, "hs", torch.uint8, (P + T, I // 32)).cpu().numpy(),
        sh_mx8=None if sh_mx8 is None else [(c.cpu().numpy(), s_.cpu().numpy()) for c, s_ in sh_mx8],
    )
    return dict(gw=gw, sh=sh, x=x, ids=ids.cpu().numpy(), tw=tw.cpu().double().numpy(), y=y.cpu().double().numpy(),
                **st)


SILU_DMAX = 1.1  # max |silu'(g)| (about 1.0998)


def _check_gate_up(Wg, Wu, X, h_gpu):
    """h = bf16(silu(g) u): bound from the GEMV tolerance of g and u, plus one bf16 ulp."""
    g, sg = M.matvec_with_scale(Wg, X)
    u, su = M.matvec_with_scale(Wu, X)
    tg, tu = 1e-3 * sg + 1e-5, 1e-3 * su + 1e-5
    h = M.silu(g) * u
    bound = SILU_DMAX * tg * (np.abs(u) + tu) + np.abs(M.silu(g)) * tu + 2.0 ** -7 * (np.abs(h) + SILU_DMAX * tg * (np.abs(u) + tu) + np.abs(M.silu(g)) * tu) + 1e-6
    err = np.abs(h_gpu - h)
    assert np.all(err <= bound), float(np.max(err / bound))


def _check_down(Wd, h_rows, Y_rows):
    y, sy = M.matvec_with_scale(Wd, h_rows)
    assert np.all(np.abs(Y_rows - y) <= 1e-3 * sy + 1e-5), float(np.max(np.abs(Y_rows - y) / (1e-3 * sy + 1e-5)))


def _check_layer(r, T, H, I, E, k, experts=None):
    P = T * k
    counts, offsets, perm, inv = M.permute(r["ids"], E)
    assert np.array_equal(r["perm"], perm) and np.array_equal(r["inv"], inv)
    xd = r["x"].float().double().cpu().numpy()
    touched = np.flatnonzero(counts)
    if experts is None:
        experts = touched
    gw = r["gw"]
    for e in experts:
        pos = np.arange(offsets[e], offsets[e + 1])
        toks = perm[pos] // k
        Wg = gw[0][e * I:(e + 1) * I].double().cpu().numpy()
        Wu = gw[1][e * I:(e + 1) * I].double().cpu().numpy()
        Wd = gw[2][e * H:(e + 1) * H].double().cpu().numpy()
        _check_gate_up(Wg, Wu, xd[toks], r["h"][pos])
        _check_down(Wd, r["h"][pos], r["Y"][pos])
    if r["sh_mx8"] is not None:
        check_mx8_shared(r, T, H, I, P)
    elif r["sh"] is not None:
        sg, su, sd = (m.float().double().cpu().numpy() for m in r["sh"])
        _check_gate_up(sg, su, xd, r["h"][P:P + T])
        _check_down(sd, r["h"][P:P + T], r["Y"][P:P + T])
    # combine of the GPU's own expert outputs
    yc = np.zeros((T, H))
    mag = np.zeros((T, H))
    for t in range(T):
        for s in range(k):
            yc[t] += r["tw"][t, s] * r["Y"][inv[t * k + s]]
            mag[t] += np.abs(r["tw"][t, s] * r["Y"][inv[t * k + s]])
        if r["sh"] is not None:
            yc[t] += r["Y"][P + t]
            mag[t] += np.abs(r["Y"][P + t])
    assert np.all(np.abs(r["y"] - yc) <= 1e-6 * mag + 1e-6)


@pytest.mark.parametrize("T,H,I,E,k,shared", [(1, 256, 256, 1, 1, False), (5, 512, 256, 8, 2, True),
                                               (13, 768, 512, 16, 4, True), (40, 512, 256, 4, 4, False)])
def test_moe_stq_small_full_check(S, T, H, I, E, k, shared):
    r = _run_layer(S, T, H, I, E, k, shared, ("small", T, H, I, E, k))
    _check_layer(r, T, H, I, E, k)


@pytest.mark.parametrize("T,H,I,E,k,shared", [(40, 512, 256, 8, 4, False), (256, 512, 256, 8, 2, True),
                                               (97, 1024, 512, 2, 2, False)])
def test_moe_stq_decode_many_tokens_full_check(S, T, H, I, E, k, shared):
    """Decode kernels with several 8-token chunks per expert (up to 97 tokens)."""
    r = _run_layer(S, T, H, I, E, k, shared, ("many", T, H, I, E, k))
    _check_layer(r, T, H, I, E, k)


# --------------------------------------------------------------------------- STQ1_0 prefill regime


def _stq_weights(r, H, I):
    gw = r["gw"]

    def weights(e):
        return (gw[0][e * I:(e + 1) * I].double().cpu().numpy(), gw[1][e * I:(e + 1) * I].double().cpu().numpy(),
                gw[2][e * H:(e + 1) * H].double().cpu().numpy())
    return weights


def _check_prefill(r, T, H, I, E, k, experts=None):
    check_mxfp8_layer(r, T, H, I, E, k, _stq_weights(r, H, I), experts)


@pytest.mark.parametrize("T,H,I,E,k,shared", [(5, 512, 256, 8, 2, True), (256, 512, 256, 8, 2, True),
                                               (200, 768, 512, 4, 3, True), (97, 1024, 512, 2, 2, False),
                                               (300, 256, 256, 3, 1, False)])
def test_moe_stq_prefill_full_check(S, T, H, I, E, k, shared):
    """Tensor-core STQ1_0 GEMM: 1 to 300 tokens per expert (several 112-token tiles with
    ragged tails), K from one 256-block up, gate/up item groups of 64 features."""
    r = _run_layer(S, T, H, I, E, k, shared, ("pf", T, H, I, E, k), regime=S.REGIME_PREFILL)
    _check_prefill(r, T, H, I, E, k)


@pytest.mark.parametrize("split", [(112, 113, 1), (300, 0, 0), (111, 1, 224)])
def test_moe_stq_prefill_tile_edges(S, split):
    """Expert loads at the 112-token tile edges and one expert taking every token."""
    E, k, H, I = 3, 1, 512, 256
    T = sum(split)
    ids = torch.tensor(np.repeat(np.arange(E), split).reshape(T, 1), dtype=torch.int32, device=DEV)
    tw = torch.ones((T, 1), dtype=torch.float32, device=DEV)
    r = _run_layer(S, T, H, I, E, k, True, ("edges",) + split, ids=ids, tw=tw, regime=S.REGIME_PREFILL)
    _check_prefill(r, T, H, I, E, k)


def test_moe_stq_prefill_wide_range_activations(S):
    """Activations spanning 2^-30 .. 2^30 and a zero row through the MXFP8 prefill path."""
    T, H, I, E, k = 160, 512, 256, 2, 2
    g = W.generator(DEV, 0, "wide-pf", "mag")
    mag = torch.exp2(torch.randint(-30, 31, (T, H), generator=g, device=DEV).float())
    x = (W.bf16_normal((T, H), 1.0, DEV, 0, "wide-pf", "x").float() * mag).to(torch.bfloat16)
    x[7] = 0
    ids, tw = W.uniform_routing(T, E, k, DEV, 0, "wide-pf", "ids")
    r = _run_layer(S, T, H, I, E, k, True, "wide-pf", ids=ids, tw=tw, x=x, regime=S.REGIME_PREFILL)
    _check_prefill(r, T, H, I, E, k)


@pytest.mark.parametrize("T,H,I,E,k,regime", [(5, 512, 256, 8, 2, "decode"), (8, 6144, 2048, 256, 8, "decode"),
                                               (200, 768, 512, 4, 3, "prefill"), (17, 512, 512, 2, 2, "decode")])
def test_moe_stq_mxfp8_shared(S, T, H, I, E, k, regime):
    """STQ1_0 layers with the MXFP8 shared expert, decode and prefill regimes (the
    decode config's shape included; routed experts sampled there)."""
    reg = S.REGIME_DECODE if regime == "decode" else S.REGIME_PREFILL
    r = _run_layer(S, T, H, I, E, k, True, ("sh8", T, H, I, E, k), regime=reg, shared_fmt="mx8")
    counts = np.bincount(r["ids"].reshape(-1), minlength=E)
    touched = np.flatnonzero(counts)
    sample = touched if touched.size <= 8 else touched[:: touched.size // 4]
    if regime == "decode":
        _check_layer(r, T, H, I, E, k, experts=sample)
    else:
        _check_prefill(r, T, H, I, E, k, experts=sample)


def test_moe_stq_auto_regime_threshold(S):
    """STQ_REGIME_AUTO takes the prefill kernels from 32 routed tokens per expert on
    average: its output equals the forced regime's, bit for bit, on either side."""
    H, I, E, k = 512, 256, 4, 2
    for T, pick in ((63, "decode"), (64, "prefill")):
        ys = {}
        for name, reg in (("auto", S.REGIME_AUTO), ("decode", S.REGIME_DECODE), ("prefill", S.REGIME_PREFILL)):
            ys[name] = _run_layer(S, T, H, I, E, k, True, ("auto", T), regime=reg)["y"]
        assert np.array_equal(ys["auto"], ys[pick])
        assert not np.array_equal(ys["decode"], ys["prefill"])


def test_moe_stq_prefill_config_sampled(S):
    """Prefill MoE layer, STQ1_0: 256 experts, 6144/2048, 1024 tokens, top-8, shared
    (32 routed tokens per expert on average: the automatic regime picks the GEMM)."""
    T, H, I, E, k = 1024, 6144, 2048, 256, 8
    r = _run_layer(S, T, H, I, E, k, True, "prefill", regime=S.REGIME_AUTO)
    counts = np.bincount(r["ids"].reshape(-1), minlength=E)
    touched = np.flatnonzero(counts)
    busiest = touched[np.argsort(-counts[touched], kind="stable")[:2]]
    sample = np.unique(np.concatenate([busiest, touched[:: max(1, touched.size // 3)]]))
    _check_prefill(r, T, H, I, E, k, experts=sample)


def test_moe_stq_prefill_bench_shape_sampled(S):
    """The STQ1_0 prefill workload as timed: 4096 tokens, Zipf(1.1) routing over 256
    experts, top-8, 6144/2048, no shared expert; busiest, median and lightest experts."""
    T, H, I, E, k = 4096, 6144, 2048, 256, 8
    ids, tw = W.zipf_routing(T, E, k, DEV, 0, "stqpre", "z")
    r = _run_layer(S, T, H, I, E, k, False, "stqpre", ids=ids, tw=tw, regime=S.REGIME_AUTO)
    counts = np.bincount(r["ids"].reshape(-1), minlength=E)
    order = np.argsort(counts, kind="stable")
    sample = [order[-1], order[len(order) // 2], order[np.flatnonzero(counts[order])[0]]]
    _check_prefill(r, T, H, I, E, k, experts=sample)


def test_moe_stq_decode_config_sampled(S):
    """Decode MoE layer, STQ1_0: 256 experts, 6144/2048, 8 tokens, top-8, shared."""
    T, H, I, E, k = 8, 6144, 2048, 256, 8
    r = _run_layer(S, T, H, I, E, k, True, "decode")
    counts = np.bincount(r["ids"].reshape(-1), minlength=E)
    touched = np.flatnonzero(counts)
    busiest = touched[np.argsort(-counts[touched], kind="stable")[:2]]
    sample = np.unique(np.concatenate([busiest, touched[:: max(1, touched.size // 3)]]))
    _check_layer(r, T, H, I, E, k, experts=sample)


def test_moe_stq_residual_and_bf16_output(S):
    T, H, I, E, k = 6, 512, 256, 8, 2
    gw, packs, sh, wr, x = _make_layer(S, T, H, I, E, k, True, "res")
    ids, tw, _ = S.moe_router_topk(x, wr, k)
    ew = S.ExpertWeights(S.FMT_STQ1_0, *packs, None, None, None, *sh)
    out = {}
    for fp32, res in [(True, False), (True, True), (False, True)]:
        desc = S.make_desc(T, H, I, E, k, out_fp32=fp32, add_residual=res)
        ws = torch.zeros(S.moe_workspace_bytes(desc), dtype=torch.uint8, device=DEV)
        y = torch.empty((T, H), dtype=torch.float32 if fp32 else torch.bfloat16, device=DEV)
        S.moe_expert_forward(desc, x, ids, tw, ew, y, ws)
        out[(fp32, res)] = y.float().cpu().double().numpy()
    xd = x.float().double().cpu().numpy()
    assert np.allclose(out[(True, True)], out[(True, False)] + xd, rtol=1e-6, atol=1e-6)
    ref_b = F.bf16_decode(F.bf16_encode_rne(out[(True, True)]))
    assert np.array_equal(out[(False, True)], ref_b)


def test_moe_stq_wide_range_activations(S):
    """Activations spanning 2^-30 .. 2^30 within each row, and a zero row."""
    T, H, I, E, k = 6, 512, 256, 8, 2
    g = W.generator(DEV, 0, "wide", "mag")
    mag = torch.exp2(torch.randint(-30, 31, (T, H), generator=g, device=DEV).float())
    x = (W.bf16_normal((T, H), 1.0, DEV, 0, "wide", "x").float() * mag).to(torch.bfloat16)
    x[3] = 0
    ids, tw = W.uniform_routing(T, E, k, DEV, 0, "wide", "ids")
    r = _run_layer(S, T, H, I, E, k, True, "wide", ids=ids, tw=tw, x=x)
    _check_layer(r, T, H, I, E, k)


@pytest.mark.parametrize("T,H,I,E,k", [(8, 512, 256, 16, 2), (6, 1024, 512, 8, 2), (6, 768, 512, 8, 2)])
def test_moe_stq_decode_integer_path_exactness(S, T, H, I, E, k):
    """Experts with one or two routed tokens (a layer averaging at most two per expert)
    run the integer GEMV: activations as a 22-bit fixed point per 256-k block, exact
    integer sums per block.  With every block's elements within 2^14 of its largest
    magnitude the down projection of the GPU's own h then matches the float64 product to a
    few FP32 roundings, far inside the layer tolerance (1e-3 S); experts with more tokens
    keep that tolerance.  An activation row spanning 2^-20 .. 2^0 inside each block checks
    the rounded elements against their bound, 2^-22 of the block's largest magnitude per
    element."""
    r = _run_layer(S, T, H, I, E, k, True, ("exact", T, H, I, E, k))
    counts, offsets, perm, _ = M.permute(r["ids"], E)
    gw = r["gw"]
    small = [e for e in np.flatnonzero(counts) if counts[e] <= 2]
    assert small, "no expert with one or two tokens"
    for e in small:
        pos = np.arange(offsets[e], offsets[e + 1])
        Wd = gw[2][e * H:(e + 1) * H].double().cpu().numpy()
        h = r["h"][pos]
        # every 256-block of h within 2^14 of its largest magnitude: the fixed point is exact
        hb = np.abs(h).reshape(len(pos), -1, 256)
        nz = np.where(hb > 0, hb, np.inf).min(axis=2)
        if np.all(hb.max(axis=2) <= nz * 2.0 ** 14):
            y, sy = M.matvec_with_scale(Wd, h)
            err = np.abs(r["Y"][pos] - y)
            assert np.all(err <= 1e-6 * sy + 1e-12), float(np.max(err / (1e-6 * sy + 1e-12)))
    _check_layer(r, T, H, I, E, k)

    # wide range inside each block: rounded elements stay within their bound
    g = W.generator(DEV, 0, "exact-wide", "mag")
    mag = torch.exp2(-torch.randint(0, 21, (T, H), generator=g, device=DEV).float())
    x = (W.bf16_normal((T, H), 1.0, DEV, 0, "exact-wide", "x").float() * mag).to(torch.bfloat16)
    r = _run_layer(S, T, H, I, E, k, True, ("exact", T, H, I, E, k), x=x)
    _check_layer(r, T, H, I, E, k)


def test_moe_stq_decode_large_h_takes_the_bf16_path(S):
    """H = 8192: the integer path's activation stage (six limb rows of H + 64 bytes) would pass
    the 47 KB shared-memory limit, so the layer runs the BF16 GEMV for every expert; results stay
    within the layer tolerance."""
    T, H, I, E, k = 4, 8192, 256, 8, 2
    r = _run_layer(S, T, H, I, E, k, True, ("largeh", T, H, I, E, k))
    _check_layer(r, T, H, I, E, k)


def test_moe_bad_expert_id_reports_and_skips(S):
    T, H, I, E, k = 2, 256, 256, 4, 2
    gw, packs, sh, wr, x = _make_layer(S, T, H, I, E, k, False, "bad")
    ids = torch.tensor([[0, 9], [1, 2]], dtype=torch.int32, device=DEV)
    tw = torch.full((T, k), 0.5, device=DEV)
    desc = S.make_desc(T, H, I, E, k, out_fp32=True)
    ws = torch.zeros(S.moe_workspace_bytes(desc), dtype=torch.uint8, device=DEV)
    y = torch.empty((T, H), dtype=torch.float32, device=DEV)
    S.moe_expert_forward(desc, x, ids, tw, S.ExpertWeights(S.FMT_STQ1_0, *packs), y, ws)
    assert S.moe_get_device_error(ws) == -6
    assert torch.isfinite(y).all()

