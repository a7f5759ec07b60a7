"""Pins of the oracle's least-squares STQ1_0 encoder ("Hy4-preview-GGUF", section 3,
"Our encoder"): closed forms, the uniform-importance reduction, a hand-worked
importance case, and the descent property against the upstream amax rule."""

import numpy as np
import pytest

from oracle import formats as F


def _block(groups):
    """One row of one 256-block from 64 groups of four values."""
    return np.asarray(groups, dtype=np.float32).reshape(1, 256)


def test_equal_magnitudes_keep_amax_and_lane0():
    """All |w| = c: the incremental costs tie, so the zero goes to lane 0, and the
    least-squares scale of the kept lanes is c itself (= the upstream amax)."""
    rng = np.random.default_rng(3)
    c = np.float32(0.0371)
    w = (np.where(rng.random((4, 256)) < 0.5, -1.0, 1.0) * c).astype(np.float32)
    code, dbits = F.stq1_codes_ls(w)
    assert np.all(dbits == F.fp16_encode_rne(np.float64(c)))
    assert np.all(code >> 3 == 0)
    up_code, up_d = F.stq1_codes_from_float(w)
    assert np.array_equal(code, up_code) and np.array_equal(dbits, up_d)


def test_uniform_importance_is_argmin_and_mean_of_kept():
    """With v = 1 the cost v (w^2 - (|w| - d)^2) = 2 d |w| - d^2 grows with |w|, so the
    zero is the upstream argmin |w|, and d is the plain mean of the 192 kept |w| —
    checked by loops over a small matrix."""
    rng = np.random.default_rng(4)
    w = (rng.standard_normal((16, 512)) * 0.02).astype(np.float32)
    code, dbits = F.stq1_codes_ls(w)
    for r in range(16):
        for b in range(2):
            kept = []
            for gi in range(64):
                grp = [float(v) for v in w[r, 256 * b + 4 * gi: 256 * b + 4 * gi + 4]]
                z = min(range(4), key=lambda j: (abs(grp[j]), j))
                assert code[r, b, gi] >> 3 == z
                kept += [abs(grp[j]) for j in range(4) if j != z]
            mean = sum(kept) / len(kept)
            assert dbits[r, b] == F.fp16_encode_rne(np.float64(mean))


def test_importance_moves_the_zero_hand_example():
    """Group 0 = (0.1, 0.3, 1, 1) with importance (1, 100, 1, 1); the other 63 groups
    are (0, 1, 1, 1) with importance 1.  Upstream zeroes lane 0 (smallest |w|); the
    incremental cost at d ~ 1 is 1*(0.01 - 0.81) = -0.8 for lane 0 but
    100*(0.09 - 0.49) = -40 for lane 1, so the encoder zeroes lane 1 (code 8: zero
    lane 1, all kept lanes positive).  d = (0.1 + 1 + 1 + 189) / 192."""
    groups = [[0.1, 0.3, 1.0, 1.0]] + [[0.0, 1.0, 1.0, 1.0]] * 63
    v = np.ones(256, dtype=np.float32)
    v[1] = 100.0
    w = _block(groups)
    code, dbits = F.stq1_codes_ls(w, v)
    assert code[0, 0, 0] == 8 and np.all(code[0, 0, 1:] == 0)
    d_exact = (np.float64(np.float32(0.1)) + 2.0 + 189.0) / 192.0
    assert dbits[0, 0] == F.fp16_encode_rne(d_exact)
    up_code, _ = F.stq1_codes_from_float(w)
    assert up_code[0, 0, 0] == 0


@pytest.mark.parametrize("dist", ["normal", "laplace", "outlier"])
def test_never_worse_than_amax_rule(dist):
    """Each round minimises the weighted squared error over one decision with the
    other fixed, starting from the upstream scale, so the weighted SSD of every row
    is at most that of the upstream amax rule (on these inputs by a wide margin)."""
    rng = np.random.default_rng({"normal": 5, "laplace": 6, "outlier": 7}[dist])
    if dist == "normal":
        w = rng.standard_normal((32, 768))
    elif dist == "laplace":
        w = rng.laplace(size=(32, 768))
    else:
        w = rng.standard_normal((32, 768))
        w[:, ::97] *= 40.0
    w = (w * 0.02).astype(np.float32)
    v = np.exp(rng.standard_normal(768)).astype(np.float32)
    for imp in (None, v):
        p_ls = F.stq1_pack_ls(w, imp)
        p_up = F.stq1_pack(w)
        for r in range(0, 32, 16):
            sl = slice(r, r + 16)
            a = F.stq1_weighted_ssd(w[sl], p_ls.reshape(2, -1)[r // 16], imp)
            b = F.stq1_weighted_ssd(w[sl], p_up.reshape(2, -1)[r // 16], imp)
            assert a <= b


def test_zero_block_and_zero_importance():
    """An all-zero block, or importance zero on every lane, gives d = 0 and all codes 0."""
    w = np.zeros((16, 256), dtype=np.float32)
    code, dbits = F.stq1_codes_ls(w)
    assert np.all(code == 0) and np.all(dbits == 0)
    rng = np.random.default_rng(8)
    w = rng.standard_normal((16, 256)).astype(np.float32)
    code, dbits = F.stq1_codes_ls(w, np.zeros(256, dtype=np.float32))
    assert np.all(code == 0) and np.all(dbits == 0)


def test_rejects_bad_inputs():
    w = np.zeros((16, 256), dtype=np.float32)
    with pytest.raises(ValueError):
        F.stq1_codes_ls(w, -np.ones(256, dtype=np.float32))
    w[3, 5] = np.inf
    with pytest.raises(F.NonFiniteError):
        F.stq1_codes_ls(w)


def test_importance_weights_the_scale_hand_example():
    """Group 0 = (0, 0.5, 1, 1) with importance 1000 on the 0.5; the other 63 groups
    are (0, 1, 1, 1), importance 1.  Every zero stays on lane 0 and
    d = (1000 * 0.5 + 1 + 1 + 189) / (1000 + 1 + 1 + 189) = 691 / 1191."""
    groups = [[0.0, 0.5, 1.0, 1.0]] + [[0.0, 1.0, 1.0, 1.0]] * 63
    v = np.ones(256, dtype=np.float32)
    v[1] = 1000.0
    code, dbits = F.stq1_codes_ls(_block(groups), v)
    assert np.all(code == 0)
    assert dbits[0, 0] == F.fp16_encode_rne(np.float64(691.0) / 1191.0)
