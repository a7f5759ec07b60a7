"""Pins of the oracle's MoE steps: brute-force loops on tiny inputs, closed
forms and invariants.  CPU only."""

import itertools

import numpy as np
import pytest

from oracle import formats as F
from oracle import moe as M

from test_oracle_formats import grid_weights


def _bf16(rng, shape, std=1.0):
    return F.bf16_encode_rne(rng.normal(0, std, shape))


# --------------------------------------------------------------------------- GEMV / GEMM


@pytest.mark.parametrize("rows,K,n", [(16, 256, 1), (16, 512, 3), (32, 256, 2)])
def test_stq_gemv_brute_force_from_structure(rows, K, n):
    # y[t, r] = sum over groups, over non-zero lanes, of sign * d * x, built
    # directly from (zero lane, sign, d) without the byte layout.
    rng = np.random.default_rng(rows + K + n)
    w, z, s, d = grid_weights(rng, rows, K)
    xb = _bf16(rng, (n, K))
    x = F.bf16_decode(xb)
    y, S = M.stq1_gemv(F.stq1_pack(w), rows, K, xb)
    for t in range(n):
        for r in range(rows):
            acc = 0.0
            sabs = 0.0
            for j in range(K // 4):
                for l in range(4):
                    if l == z[r, j]:
                        continue
                    term = s[r, j, l] * d[r, (4 * j) // 256] * x[t, 4 * j + l]
                    acc += term
                    sabs += abs(term)
            assert abs(y[t, r] - acc) <= 1e-12 * (sabs + 1)
            assert abs(S[t, r] - sabs) <= 1e-12 * (sabs + 1)


def test_stq_gemv_one_hot_and_all_positive():
    rows, K = 16, 512
    # d = 1, all-positive rows with zero lane 3: y = sum of x over lanes 0..2 of every group
    code = np.full((rows, K // 256, 64), 8 * 3, dtype=np.int64)
    dbits = np.full((rows, K // 256), F.fp16_encode_rne(1.0), np.uint16)
    packed = F.stq1_layout(code, dbits)
    rng = np.random.default_rng(11)
    xb = _bf16(rng, (1, K))
    x = F.bf16_decode(xb)[0]
    y, _ = M.stq1_gemv(packed, rows, K, xb)
    ref = sum(x[k] for k in range(K) if k % 4 != 3)
    assert np.allclose(y[0], ref, rtol=0, atol=1e-12)
    # one-hot x picks one weight column exactly
    w, *_ = grid_weights(rng, rows, K)
    b = F.stq1_pack(w)
    for k in [0, 1, 255, 256, 511]:
        e = np.zeros((1, K))
        e[0, k] = 1.0
        yk, _ = M.stq1_gemv(b, rows, K, F.bf16_encode_rne(e))
        assert np.array_equal(yk[0], w[:, k].astype(np.float64))


def test_w4a8_gemm_brute_force():
    rng = np.random.default_rng(12)
    N, K, Mt = 4, 64, 3
    wc = rng.integers(0, 256, (N, K // 2)).astype(np.uint8)
    ws = rng.integers(118, 128, (N, K // 32)).astype(np.uint8)
    ac, asc = F.mxfp8_quantize(F.bf16_decode(_bf16(rng, (Mt, K))))
    Y, S = M.w4a8_gemm(wc, ws, ac, asc, N, K)
    for m in range(Mt):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                byte = wc[n, k // 2]
                nib = (byte >> (4 * (k % 2))) & 15
                wv = F.e2m1_decode(np.uint8(nib)) * 2.0 ** (int(ws[n, k // 32]) - 127)
                av = F.e4m3_decode(ac[m, k]) * 2.0 ** (int(asc[m, k // 32]) - 127)
                acc += wv * av
            assert abs(Y[m, n] - acc) <= 1e-12 * (abs(acc) + 1)


# --------------------------------------------------------------------------- router


def test_router_softmax_topk_properties():
    rng = np.random.default_rng(13)
    T, H, E, k = 5, 64, 32, 8
    xb = _bf16(rng, (T, H))
    wr = _bf16(rng, (E, H), 0.5)
    ids, w, p = M.router_topk(xb, wr, k)
    assert np.allclose(p.sum(axis=1), 1.0, atol=1e-12)
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-12)
    for t in range(T):
        # brute force: sort (prob desc, id asc)
        order = sorted(range(E), key=lambda e: (-p[t, e], e))[:k]
        assert list(ids[t]) == order
        logits = F.bf16_decode(xb[t]) @ F.bf16_decode(wr).T
        q = np.exp(logits - logits.max())
        assert np.allclose(p[t], q / q.sum(), rtol=1e-12)
    # relabelling the experts relabels the choice
    perm = rng.permutation(E)
    ids2, w2, _ = M.router_topk(xb, wr[perm], k)
    assert np.array_equal(perm[ids2], ids) and np.allclose(w2, w)


def test_router_ties_go_to_lower_id():
    T, H, E = 1, 32, 16
    xb = F.bf16_encode_rne(np.ones((T, H)))
    wr = F.bf16_encode_rne(np.zeros((E, H)))
    ids, w, _ = M.router_topk(xb, wr, 8)
    assert list(ids[0]) == list(range(8)) and np.allclose(w, 1 / 8)


# --------------------------------------------------------------------------- permute


def test_permute_matches_stable_sort_by_loops():
    rng = np.random.default_rng(14)
    for T, E, k in [(1, 4, 2), (7, 16, 8), (33, 256, 8)]:
        ids = rng.integers(0, E, (T, k))
        counts, offsets, perm, inv = M.permute(ids, E)
        flat = ids.reshape(-1)
        ref = sorted(range(T * k), key=lambda p: (flat[p], p))
        assert list(perm) == ref
        assert counts.sum() == T * k and offsets[0] == 0 and offsets[-1] == T * k
        assert np.all(np.diff(offsets) == counts)
        for e in range(E):
            assert counts[e] == sum(1 for v in flat if v == e)
            assert all(flat[perm[i]] == e for i in range(offsets[e], offsets[e + 1]))
        assert np.array_equal(perm[inv], np.arange(T * k))


def test_permute_rejects_bad_ids():
    with pytest.raises(ValueError):
        M.permute(np.array([[0, 256]]), 256)


# --------------------------------------------------------------------------- SwiGLU and combine


def test_silu_closed_forms():
    v = np.linspace(-30, 30, 601)
    # silu(v) - silu(-v) = v(sigmoid(v) + sigmoid(-v)) = v
    assert np.allclose(M.silu(v) - M.silu(-v), v, atol=1e-12)
    assert M.silu(0.0) == 0.0
    assert abs(M.silu(1.0) - 1.0 / (1.0 + np.exp(-1.0))) < 1e-15
    assert abs(M.silu(40.0) - 40.0) < 1e-12 and abs(M.silu(-800.0)) == 0.0


def test_swiglu_rounds_inputs_to_f32():
    g = np.array([1.0 + 2.0 ** -30])
    u = np.array([2.0])
    assert M.swiglu(g, u)[0] == M.silu(1.0) * 2.0


def test_combine_brute_force():
    rng = np.random.default_rng(15)
    T, k, H = 3, 4, 5
    Y = rng.normal(size=(T * k, H))
    S = np.abs(Y)
    w = rng.random((T, k))
    sh = rng.normal(size=(T, H))
    res = rng.normal(size=(T, H))
    y, s = M.combine(Y, S, w, sh, None, res)
    for t, h in itertools.product(range(T), range(H)):
        ref = sum(w[t, j] * Y[t * k + j, h] for j in range(k)) + sh[t, h] + res[t, h]
        assert abs(y[t, h] - ref) < 1e-12
        assert s[t, h] >= abs(y[t, h]) - 1e-12


def test_expert_ffn_stage_consistency():
    rng = np.random.default_rng(16)
    I, H, n = 16, 256, 2
    wg, *_ = grid_weights(rng, I, H)
    wu, *_ = grid_weights(rng, I, H)
    wd, *_ = grid_weights(rng, H, I * 16)
    wd = wd[:, :I]
    X = F.bf16_decode(_bf16(rng, (n, H)))
    out = M.expert_ffn_bf16h(wg, wu, wd, X)
    g = X @ wg.astype(np.float64).T
    u = X @ wu.astype(np.float64).T
    h = F.bf16_decode(F.bf16_encode_rne(M.silu(g.astype(np.float32).astype(np.float64)) * u.astype(np.float32)))
    assert np.array_equal(out["h"], h)
    assert np.allclose(out["y"], h @ wd.astype(np.float64).T, rtol=1e-13, atol=1e-15)


def test_expert_ffn_bf16h_rounds_h_to_nearest_even_bf16():
    """Worked by hand: activation e_0, gate rows 64 h*, up rows 1/64, so g >= 37 and
    silu(g) = g exactly (exp(-g) vanishes next to 1), and h = h* exactly.  h* = 1 + 2^-8 is
    a BF16 tie that goes down to the even 1.0; 1 + 3 * 2^-8 a tie that goes up to the even
    1.015625; 1 + 2^-8 + 2^-10 lies above a tie and goes up to 1.0078125.  The down
    projection (identity rows and one row of ones) must see the rounded h."""
    H, I = 4, 3
    hstar = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 1 + 2.0 ** -8 + 2.0 ** -10])
    X = np.zeros((1, H))
    X[0, 0] = 1.0
    Wg = np.zeros((I, H))
    Wg[:, 0] = 64.0 * hstar
    Wu = np.zeros((I, H))
    Wu[:, 0] = 1.0 / 64.0
    Wd = np.vstack([np.eye(I), np.ones((1, I))])
    out = M.expert_ffn_bf16h(Wg, Wu, Wd, X)
    expect_h = np.array([1.0, 1.015625, 1.0078125])
    assert np.array_equal(out["h"][0], expect_h)
    assert np.array_equal(out["h_bits"][0], np.array([0x3F80, 0x3F82, 0x3F81]))
    assert np.array_equal(out["y"][0], np.append(expect_h, expect_h.sum()))


def _ffn_mx_tie_case():
    """One token through a 32-feature expert whose h is decided by hand.  a = e_0, every
    gate row 40 e_0 and every up row u e_0 with u = FP32 0x3cd9999a (0.0265625 rounded up),
    the down projection the identity.  g = 40 and silu(40) = 40 exactly in float64 and in
    FP32 (exp(-40) vanishes next to 1), so h = 40 u: 1.0625 + 2.98e-8 in float64 but
    exactly 1.0625 once rounded to FP32, as the GPU's FP32 epilogue holds it.  The
    smallest power of two 2^k with 1.0625 <= 448 * 2^k is 2^-8 (448 * 2^-9 = 0.875 is too
    small), so the MXFP8 scale is 2^-8 (UE8M0 119) and h / scale = 272 lies halfway between
    the E4M3 values 256 (0x78) and 288 (0x79): it rounds to the even 256."""
    I = H = 32
    u = np.array([0x3CD9999A], dtype=np.uint32).view(np.float32)[0]
    A = np.zeros((1, H))
    A[0, 0] = 1.0
    Wg = np.zeros((I, H))
    Wg[:, 0] = 40.0
    Wu = np.zeros((I, H))
    Wu[:, 0] = float(u)
    return Wg, Wu, np.eye(H, I), A


def test_expert_ffn_mx_rounds_h_to_f32_before_quantising():
    """Worked by hand (see _ffn_mx_tie_case): codes 0x78, scale 119, h = y = 1.0.  Without the
    FP32 rounding of h the tie breaks upward (0x79, 1.125)."""
    Wg, Wu, Wd, A = _ffn_mx_tie_case()
    out = M.expert_ffn_mx(Wg, Wu, Wd, A)
    assert np.all(out["h_codes"] == 0x78) and np.all(out["h_scales"] == 119)
    assert np.all(out["h"] == 1.0) and np.all(out["y"] == 1.0)
    # the case has teeth: the same steps without the FP32 rounding give the other code
    g, _, u, _ = M.expert_gate_up(Wg, Wu, A)
    hc, hs = F.mxfp8_quantize(M.silu(g) * u)
    assert np.all(hc == 0x79) and np.all(hs == 119)


def test_rms_norm_closed_forms():
    """Constant rows: a / sqrt(a^2 + eps) (eps = 3, a = 1 gives exactly 1/2; eps = 0
    gives sign(a)); a 3-4 row: mean square 12.5, so y = (3, 4) / sqrt(12.5)."""
    y = M.rms_norm(np.array([[1.0] * 8, [-2.5] * 8]), 3.0)
    assert np.all(y[0] == 0.5) and np.allclose(y[1], -2.5 / np.sqrt(6.25 + 3.0), rtol=0, atol=1e-15)
    assert np.all(M.rms_norm(np.full((1, 16), -7.0), 0.0) == -1.0)
    y = M.rms_norm(np.array([[3.0, 4.0]]), 0.0)
    assert abs(y[0, 0] - 0.848528137423857) < 1e-14 and abs(y[0, 1] - 1.131370849898476) < 1e-14


def test_rms_norm_invariants():
    """With eps = 0 every output row has mean square 1 and the map ignores a positive
    scale of its row; rows are independent of one another."""
    rng = np.random.default_rng(5)
    x = rng.standard_normal((6, 96)) * np.array([[1e-3], [1.0], [7.0], [1e4], [0.5], [3.0]])
    y = M.rms_norm(x, 0.0)
    assert np.allclose(np.mean(y * y, axis=1), 1.0, rtol=0, atol=1e-13)
    assert np.allclose(M.rms_norm(x * 2.0 ** 11, 0.0), y, rtol=1e-15, atol=0)
    assert np.array_equal(M.rms_norm(x[2:3], 0.0), y[2:3])
    # eps only lowers the output: |y_eps| < |y_0| elementwise where x != 0
    ye = M.rms_norm(x, 1e-2)
    assert np.all(np.abs(ye) <= np.abs(y))
