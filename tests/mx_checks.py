"""Stage-by-stage check of a MoE layer whose routed experts take MXFP8 activations
(MXFP4 experts, and STQ1_0 experts in the prefill regime) against the oracle:
grouping (exact), activation quantisation in sorted pair order (bit-exact), gate/up +
SwiGLU + MXFP8 h (propagated bound plus one E4M3 step), down on the GPU's own h
(1e-3 * S + 1e-5), the BF16 shared expert, and the combine of the GPU's own outputs."""

import numpy as np
import torch

from oracle import formats as F
from oracle import moe as M

SILU_DMAX = 1.1  # max |silu'(g)| (about 1.0998)


def np_bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def check_bf16_gate_up(Wg, Wu, X, h_gpu):
    """h = bf16(silu(g) u): bound from the GEMV tolerance of g and u, plus one bf16 ulp."""
    g, sg = M.matvec_with_scale(Wg, X)
    u, su = M.matvec_with_scale(Wu, X)
    tg, tu = 1e-3 * sg + 1e-5, 1e-3 * su + 1e-5
    h = M.silu(g) * u
    prop = SILU_DMAX * tg * (np.abs(u) + tu) + np.abs(M.silu(g)) * tu
    bound = prop + 2.0 ** -7 * (np.abs(h) + prop) + 1e-6
    err = np.abs(h_gpu - h)
    assert np.all(err <= bound), float(np.max(err / bound))


def check_down(Wd, h_rows, Y_rows, tag=None):
    """Y = Wd h on the GPU's own h rows: |Y - y| <= 1e-3 S + 1e-5."""
    y, sy = M.matvec_with_scale(Wd, h_rows)
    tol = 1e-3 * sy + 1e-5
    assert np.all(np.abs(Y_rows - y) <= tol), (tag, float(np.max(np.abs(Y_rows - y) / tol)))


def shared_mx8_weights(r):
    """Dequantised MXFP8 shared expert (Wg, Wu, Wd) from the codes and scales the GPU
    used; the codes themselves are checked against the oracle's quantiser."""
    out = []
    for bf, (codes, scales) in zip(r["sh"], r["sh_mx8"]):
        c, sc = F.mxfp8_quantize(F.bf16_decode(np_bits(bf)))
        assert np.array_equal(codes, c) and np.array_equal(scales, sc)
        out.append(F.mxfp8_dequantize(codes, scales))
    return out


def check_mx8_shared(r, T, H, I, P):
    """MXFP8 shared expert: x quantised into rows P.. (bit-exact), gate/up + SwiGLU into
    MXFP8 h rows P.. (propagated bound plus one E4M3 step), down on the GPU's own h."""
    Wg, Wu, Wd = shared_mx8_weights(r)
    xq, xs = F.mxfp8_quantize(F.bf16_decode(np_bits(r["x"])))
    assert np.array_equal(r["xq"][P:P + T], xq) and np.array_equal(r["xs"][P:P + T], xs)
    check_mx_expert(Wg, Wu, Wd, F.mxfp8_dequantize(xq, xs), r["hq"][P:P + T], r["hs"][P:P + T], r["Y"][P:P + T])


def check_mx_expert(Wg, Wu, Wd, A, hq, hs, Y, tag=None):
    """One expert on MXFP8 activations A: SwiGLU and MXFP8 h (bound), down (1e-3 S + 1e-5)."""
    g, sg = M.matvec_with_scale(Wg, A)
    u, su = M.matvec_with_scale(Wu, A)
    tg, tu = 1e-3 * sg + 1e-5, 1e-3 * su + 1e-5
    h = M.swiglu(g, u)
    prop = SILU_DMAX * tg * (np.abs(u) + tu) + np.abs(M.silu(g)) * tu
    _, href_s = F.mxfp8_quantize(h.astype(np.float32).astype(np.float64))
    sc = np.maximum(np.repeat(F.ue8m0_decode(href_s), 32, axis=1), np.repeat(F.ue8m0_decode(hs), 32, axis=1))
    bound = prop * (1 + 2.0 ** -4) + 2.0 ** -4 * np.abs(h) + sc * 2.0 ** -9 + 1e-6
    hdeq = F.mxfp8_dequantize(hq, hs)
    assert np.all(np.abs(hdeq - h) <= bound), (tag, float(np.max(np.abs(hdeq - h) / bound)))
    y, sy = M.matvec_with_scale(Wd, hdeq)
    tol = 1e-3 * sy + 1e-5
    assert np.all(np.abs(Y - y) <= tol), (tag, float(np.max(np.abs(Y - y) / tol)))


def check_mxfp8_layer(r, T, H, I, E, k, weights, experts=None):
    """r: the GPU layer's outputs and workspace views (ids, tw, x, xq, xs, hq, hs, h, Y,
    perm, inv, y, sh); weights(e) -> decoded (Wg [I, H], Wu [I, H], Wd [H, I]) float64."""
    P = T * k
    counts, offsets, perm, inv = M.permute(r["ids"], E)
    assert np.array_equal(r["perm"], perm) and np.array_equal(r["inv"], inv)
    xb = np_bits(r["x"])
    # stage 1: activations quantised in sorted pair order, bit-exact
    rxq, rxs = F.mxfp8_quantize(F.bf16_decode(xb[perm // k]))
    assert np.array_equal(r["xq"][:P], rxq) and np.array_equal(r["xs"][:P], rxs)
    A = F.mxfp8_dequantize(rxq, rxs)
    touched = np.flatnonzero(counts)
    for e in (touched if experts is None else experts):
        pos = np.arange(offsets[e], offsets[e + 1])
        Wg, Wu, Wd = weights(e)
        # stages 2 and 3: SwiGLU + MXFP8 h, then down on the GPU's own h
        check_mx_expert(Wg, Wu, Wd, A[pos], r["hq"][pos], r["hs"][pos], r["Y"][pos], int(e))
    if r.get("sh_mx8") is not None:
        check_mx8_shared(r, T, H, I, P)
    elif r["sh"] is not None:
        X = F.bf16_decode(xb)
        sg_, su_, sd_ = (m.float().double().cpu().numpy() for m in r["sh"])
        check_bf16_gate_up(sg_, su_, X, r["h"][P:P + T])
        y, sy = M.matvec_with_scale(sd_, r["h"][P:P + T])
        assert np.all(np.abs(r["Y"][P:P + T] - y) <= 1e-3 * sy + 1e-5)
    if r.get("y") is None:
        return      # the caller checks its own combine (e.g. BF16 output with a residual)
    # combine of the GPU's own expert outputs: FP32 sum of k (+1) terms
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
