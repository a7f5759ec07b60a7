"""Plant plausible mistakes in the oracle (on the CPU, via monkeypatch) and check
that the pins catch each one.  This shows the pins constrain the oracle rather
than restate it."""

import numpy as np
import pytest

from oracle import formats as F
from oracle import moe as M

import test_oracle_formats as TF
import test_oracle_moe as TM


def _fails(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


def test_reversed_sign_order_is_caught(monkeypatch):
    monkeypatch.setattr(F, "_NZ_LANES", F._NZ_LANES[:, ::-1].copy())
    _fails(TF.test_codebook_is_zero_lane_and_ordered_signs)
    _fails(TF.test_stq_layout_second_reading)


def test_wrong_scale_boundary_is_caught(monkeypatch):
    orig = F.mxfp8_scale_exponent

    def off_by_one(amax):
        fm, E = np.frexp(np.asarray(amax, np.float64))
        m, e = 2.0 * fm, E - 1
        k = np.where(m < 1.75, e - 8, e - 7)          # '<' instead of '<='
        return np.where(np.asarray(amax) == 0, 127, np.clip(k + 127, 0, 254)).astype(np.int64)

    monkeypatch.setattr(F, "mxfp8_scale_exponent", off_by_one)
    _fails(TF.test_mxfp8_quant_exhaustive_bf16_own_amax)
    monkeypatch.setattr(F, "mxfp8_scale_exponent", orig)


def test_round_half_away_is_caught(monkeypatch):
    def rta(v, frac_bits, emin):
        v = np.asarray(v, np.float64)
        a = np.abs(v)
        _, E = np.frexp(a)
        q = np.ldexp(1.0, np.maximum(E - 1, emin) - frac_bits)
        return np.copysign(np.floor(a / q + 0.5) * q, v)

    monkeypatch.setattr(F, "round_to_binary", rta)
    _fails(TF.test_e2m1_rounding_brute_force)
    _fails(TF.test_bf16_rne_matches_library_cast)


def test_transposed_gemv_is_caught(monkeypatch):
    def transposed(W, X):
        W = np.asarray(W, np.float64)
        X = np.asarray(X, np.float64)
        Wt = W.reshape(W.shape[1], W.shape[0]) if W.shape[0] != W.shape[1] else W.T
        return X @ Wt.T.reshape(W.shape).T, np.abs(X) @ np.abs(W).T

    monkeypatch.setattr(M, "matvec_with_scale", transposed)
    _fails(TM.test_stq_gemv_brute_force_from_structure, 16, 256, 1)


def test_dropped_slot_in_combine_is_caught(monkeypatch):
    orig = M.combine

    def drop_last(Y, S, w, shared=None, shared_S=None, residual=None):
        w = np.array(w, np.float64)
        w[:, -1] = 0.0
        return orig(Y, S, w, shared, shared_S, residual)

    monkeypatch.setattr(M, "combine", drop_last)
    _fails(TM.test_combine_brute_force)


def test_unstable_permute_is_caught(monkeypatch):
    def unstable(ids, E):
        flat = np.asarray(ids, np.int64).reshape(-1)
        counts = np.bincount(flat, minlength=E)
        offsets = np.concatenate([[0], np.cumsum(counts)])
        perm = np.argsort(-np.arange(flat.size))[np.argsort(flat[::-1], kind="stable")]
        inv = np.empty_like(perm)
        inv[perm] = np.arange(perm.size)
        return counts, offsets, perm, inv

    monkeypatch.setattr(M, "permute", unstable)
    _fails(TM.test_permute_matches_stable_sort_by_loops)


@pytest.mark.parametrize("mistake", ["sum", "eps_outside", "no_sqrt"])
def test_rms_norm_mistakes_are_caught(monkeypatch, mistake):
    def wrong(x, eps):
        x = np.asarray(x, np.float64)
        if mistake == "sum":
            return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)
        ms = np.mean(x * x, axis=-1, keepdims=True)
        if mistake == "eps_outside":
            return x / (np.sqrt(ms) + eps)
        return x / (ms + eps)

    monkeypatch.setattr(M, "rms_norm", wrong)
    _fails(TM.test_rms_norm_closed_forms)


@pytest.mark.parametrize("mistake", ["argmax", "unweighted_scale", "magnitude_zero"])
def test_ls_encoder_mistakes_are_caught(monkeypatch, mistake):
    import test_oracle_encoder as TE
    orig_argmin, orig_sum = np.argmin, np.sum

    def codes(w, importance=None, rounds=F.STQ_LS_ROUNDS):
        w = np.asarray(w, dtype=np.float32).astype(np.float64)
        rows, K = w.shape
        v = np.ones(K) if importance is None else np.asarray(importance, np.float32).astype(np.float64)
        nb = K // 256
        x = w.reshape(rows, nb, 64, 4)
        vg = np.broadcast_to(v.reshape(nb, 64, 4), x.shape)
        ax = np.abs(x)
        d = np.max(ax.reshape(rows, nb, 256), axis=2)
        for _ in range(rounds):
            e = ax - d[:, :, None, None]
            cost = vg * (x * x - e * e)
            if mistake == "argmax":
                z = np.argmax(cost, axis=3)
            elif mistake == "magnitude_zero":
                z = np.argmin(ax, axis=3)
            else:
                z = np.argmin(cost, axis=3)
            keep = np.ones(x.shape, dtype=bool)
            np.put_along_axis(keep, z[..., None], False, axis=3)
            wt = np.ones_like(vg) if mistake == "unweighted_scale" else vg
            num = np.sum(np.where(keep, wt * ax, 0.0), axis=(2, 3))
            den = np.sum(np.where(keep, wt, 0.0), axis=(2, 3))
            d = np.where(den > 0, num / np.where(den > 0, den, 1.0), 0.0)
        dbits = F.fp16_encode_rne(d)
        neg = np.signbit(x).astype(np.int64)
        sb = np.take_along_axis(neg, F._NZ_LANES[z], axis=3)
        code = 8 * z + sb[..., 0] + 2 * sb[..., 1] + 4 * sb[..., 2]
        code = np.where((F.fp16_decode(dbits) == 0)[:, :, None], 0, code)
        return code.astype(np.int64), dbits

    monkeypatch.setattr(F, "stq1_codes_ls", codes)
    with pytest.raises(AssertionError):
        TE.test_importance_moves_the_zero_hand_example()
        TE.test_importance_weights_the_scale_hand_example()
        TE.test_uniform_importance_is_argmin_and_mean_of_kept()
