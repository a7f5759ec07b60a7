"""Routed-expert FFN of one MoE layer, computed the plain way in float64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Shapes ("Hy4-preview-FlashMoE-STQ1_0", "Package details"): hidden H = 6144,
MoE intermediate I = 2048, E = 256 routed experts, k = 8 selected per token,
one shared expert.  Steps, in order: router (softmax over the E logits, top-k,
renormalised), token-to-expert grouping, per expert gate/up projections, SwiGLU,
down projection, weighted top-k combine plus the shared expert; between stacked
layers, an RMS normalisation of the residual stream (a reading, see rms_norm).

Every matrix product is a float64 numpy matmul of decoded values (a library
primitive); every reduction bound S = sum |w * x| is returned beside the result
so tests can apply |y - y_ref| <= 1e-3 * S + 1e-5.
"""

import numpy as np

from . import formats as F

# ----------------------------------------------------------------------------
# Products with their error scale
# ----------------------------------------------------------------------------


def matvec_with_scale(W, X):
    """W [rows, K] float64, X [n, K] float64 -> (Y [n, rows], S [n, rows]) with
    Y = X @ W^T and S = |X| @ |W|^T."""
    W = np.asarray(W, dtype=np.float64)
    X = np.asarray(X, dtype=np.float64)
    return X @ W.T, np.abs(X) @ np.abs(W).T


def stq1_gemv(packed, rows, K, x_bf16):
    """y = W x for STQ1_0 W [rows, K] and BF16 activations [n, K] -> float64
    (y [n, rows], S [n, rows])."""
    W = F.stq1_unpack(packed, rows, K)
    return matvec_with_scale(W, F.bf16_decode(x_bf16))


def w4a8_gemm(w_codes, w_scales, a_codes, a_scales, N, K):
    """Y[m, n] = sum_k a[m, k] w[n, k] with MXFP4 weights [N, K] and MXFP8
    activations [M, K] -> float64 (Y [M, N], S [M, N])."""
    W = F.mxfp4_unpack(w_codes, w_scales, N, K)
    A = F.mxfp8_dequantize(a_codes, a_scales)
    return matvec_with_scale(W, A)


# ----------------------------------------------------------------------------
# Router
# ----------------------------------------------------------------------------


def router_probs(x_bf16, wr_bf16):
    """logits[t, e] = sum_h x[t, h] wr[e, h]; probabilities = softmax over e."""
    logits = F.bf16_decode(x_bf16) @ F.bf16_decode(wr_bf16).T
    z = logits - logits.max(axis=1, keepdims=True)
    p = np.exp(z)
    return p / p.sum(axis=1, keepdims=True), logits


def router_topk(x_bf16, wr_bf16, k):
    """Top-k experts by probability (equal probabilities: lower expert id first),
    weights renormalised over the k chosen.  Returns (ids [T, k] int32, w [T, k]
    float64, p [T, E])."""
    p, _ = router_probs(x_bf16, wr_bf16)
    order = np.argsort(-p, axis=1, kind="stable")[:, :k]
    pk = np.take_along_axis(p, order, axis=1)
    return order.astype(np.int32), pk / pk.sum(axis=1, keepdims=True), p


# ----------------------------------------------------------------------------
# Token-to-expert grouping
# ----------------------------------------------------------------------------


def permute(topk_ids, E):
    """Pairs p = t*k + slot, sorted by expert and, within an expert, by p.
    Returns counts [E], offsets [E+1] (exclusive scan), perm [P] (pair at each
    sorted position), inv [P] (sorted position of each pair)."""
    flat = np.asarray(topk_ids, dtype=np.int64).reshape(-1)
    if flat.size and (flat.min() < 0 or flat.max() >= E):
        raise ValueError("expert id out of range")
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    perm = np.argsort(flat, kind="stable").astype(np.int64)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size)
    return counts, offsets, perm, inv


# ----------------------------------------------------------------------------
# SwiGLU
# ----------------------------------------------------------------------------


def silu(v):
    """silu(v) = v / (1 + exp(-v)), float64."""
    v = np.asarray(v, dtype=np.float64)
    with np.errstate(over="ignore"):
        return v / (1.0 + np.exp(-v))


def swiglu(g, u):
    """h = silu(g) * u, where g and u are first rounded to float32 (the
    accumulator type of the projections) and the product is then formed in
    float64."""
    g32 = np.asarray(g, dtype=np.float64).astype(np.float32).astype(np.float64)
    u32 = np.asarray(u, dtype=np.float64).astype(np.float32).astype(np.float64)
    return silu(g32) * u32


# ----------------------------------------------------------------------------
# One expert
# ----------------------------------------------------------------------------


def expert_gate_up(Wg, Wu, X):
    """(g, Sg, u, Su) for decoded gate/up [I, H] and activations X [n, H]."""
    g, sg = matvec_with_scale(Wg, X)
    u, su = matvec_with_scale(Wu, X)
    return g, sg, u, su


def expert_ffn_bf16h(Wg, Wu, Wd, X):
    """Expert on the STQ1_0 / BF16 path: h rounded to BF16 before the down
    projection.  Returns dict with g, u, h (float64 of the BF16 h), h_bits, y, Sy."""
    g, sg, u, su = expert_gate_up(Wg, Wu, X)
    hb = F.bf16_encode_rne(swiglu(g, u))
    h = F.bf16_decode(hb)
    y, sy = matvec_with_scale(Wd, h)
    return dict(g=g, sg=sg, u=u, su=su, h=h, h_bits=hb, y=y, sy=sy)


def expert_ffn_mx(Wg, Wu, Wd, A):
    """Expert on the W4A8 path: A are the dequantised MXFP8 activations; h is
    re-quantised to MXFP8 (per 32 along I) before the down projection."""
    g, sg, u, su = expert_gate_up(Wg, Wu, A)
    hv = swiglu(g, u).astype(np.float32).astype(np.float64)
    hc, hs = F.mxfp8_quantize(hv)
    h = F.mxfp8_dequantize(hc, hs)
    y, sy = matvec_with_scale(Wd, h)
    return dict(g=g, sg=sg, u=u, su=su, h_codes=hc, h_scales=hs, h=h, y=y, sy=sy)


# ----------------------------------------------------------------------------
# Combine
# ----------------------------------------------------------------------------


def combine(Y_pairs, S_pairs, topk_w, shared=None, shared_S=None, residual=None):
    """y[t] = sum_s w[t, s] * Y[t*k + s] (+ shared[t]) (+ residual[t]), in slot
    order s = 0..k-1.  Y_pairs [P, H] is indexed by pair p = t*k + s.  Returns
    (y [T, H], S [T, H]) with S the matching sum of |terms|."""
    w = np.asarray(topk_w, dtype=np.float64)
    T, k = w.shape
    Y = np.asarray(Y_pairs, dtype=np.float64).reshape(T, k, -1)
    S = np.asarray(S_pairs, dtype=np.float64).reshape(T, k, -1)
    y = np.einsum("ts,tsh->th", w, Y)
    s = np.einsum("ts,tsh->th", np.abs(w), S)
    if shared is not None:
        y = y + shared
        s = s + (shared_S if shared_S is not None else np.abs(shared))
    if residual is not None:
        y = y + residual
        s = s + np.abs(residual)
    return y, s


# ----------------------------------------------------------------------------
# Between stacked layers
# ----------------------------------------------------------------------------


def rms_norm(x, eps):
    """y[t, :] = x[t, :] / sqrt(mean_j x[t, j]^2 + eps), float64, unit gain.

    The stacked decode of "Hy4-preview-FlashMoE-STQ1_0" ("Package details") chains
    MoE layers with a residual add and names no normalisation; the reading used
    here applies this normalisation to each layer's output (residual included)
    before it becomes the next layer's input, which keeps eight random layers
    finite.  Callers round the result to BF16 to compare with a BF16 output."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps)
