"""Pins of the oracle's format code against what the pages and the mathematics fix.

None of these tests needs a GPU.  Each one checks the oracle against something
other than itself: numbers printed on the pages (``tests/golden``), closed forms,
brute-force searches over every code, library IEEE conversions, or a second,
loop-based reading of the byte layout.
"""

import itertools
import math
import os

import numpy as np
import pytest
import torch

from oracle import formats as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _constants():
    out = {}
    for line in open(os.path.join(GOLDEN, "page_constants.txt")):
        line = line.split("#")[0].strip()
        if line:
            k, v = (s.strip() for s in line.split("="))
            out[k] = float(v)
    return out


C = _constants()


def grid_weights(rng, rows, K, d=None):
    """Ternary 3:4 grid weights built directly from (zero lane, signs, d)."""
    z = rng.integers(0, 4, (rows, K // 4))
    s = rng.integers(0, 2, (rows, K // 4, 4)) * 2 - 1
    if d is None:
        d = np.abs(rng.normal(0, 0.02, (rows, K // 256))).astype(np.float16).astype(np.float64)
    pat = np.where(np.arange(4)[None, None, :] == z[..., None], 0.0, s)
    return (pat.reshape(rows, K // 256, 256) * d[:, :, None]).reshape(rows, K).astype(np.float32), z, s, d


# --------------------------------------------------------------------------- byte counts


def test_stq_bytes_per_block_from_pages():
    assert C["stq_block_bytes"] == 2 + C["stq_code_bytes_per_block"]
    assert C["stq_code_bytes_per_block"] * 8 == C["stq_groups_per_block"] * C["stq_bits_per_group"]
    assert C["stq_block_bytes"] * 8 / C["stq_block_weights"] == C["stq_bpw"]
    rng = np.random.default_rng(1)
    for rows, K in [(16, 256), (32, 512), (48, 1024)]:
        w, *_ = grid_weights(rng, rows, K)
        b = F.stq1_pack(w)
        assert b.size == rows * K // 256 * 42 == F.stq1_packed_bytes(rows, K)


def test_expert_matrix_bytes_and_mixed_bpw():
    # One routed gate (or up) matrix of the real shape packs to 2048*6144/256*42 bytes.
    assert F.stq1_packed_bytes(int(C["moe_intermediate"]), int(C["hidden"])) == 2_064_384
    # The 1.78 bpw routed average of the review page is the gate/up mix of 29
    # STQ1_0 layers and 48 IQ2_XXS layers, which pins 1.3125 bpw for STQ1_0.
    mix = (C["stq_layers"] * C["stq_bpw"] + C["iq2_layers"] * C["iq2_xxs_bpw"]) / (C["stq_layers"] + C["iq2_layers"])
    assert round(mix, 2) == C["routed_bpw_mix"]


def test_full_matrix_pack_size():
    rng = np.random.default_rng(2)
    rows, K = 64, int(C["hidden"])
    w, *_ = grid_weights(rng, rows, K)
    assert F.stq1_pack(w).size == rows * 24 * 42


# --------------------------------------------------------------------------- STQ1_0 codebook


def test_codebook_has_32_distinct_three_nonzero_patterns():
    pats = F.stq1_pattern(np.arange(32))
    assert pats.shape == (32, 4)
    assert len({tuple(p) for p in pats}) == C["stq_patterns"] == 32
    for p in pats:
        assert (p == 0).sum() == 1 and set(np.abs(p[p != 0])) == {1.0}


def test_codebook_is_zero_lane_and_ordered_signs():
    # Every (zero lane, sign triple) pair appears exactly once, and the sign bit n
    # belongs to the n-th non-zero lane counted upward.
    seen = {}
    for c in range(32):
        p = F.stq1_pattern(np.array(c))
        z = int(np.flatnonzero(p == 0)[0])
        nz = [l for l in range(4) if l != z]
        signs = tuple(int(p[l] < 0) for l in nz)
        seen[(z, signs)] = c
    assert len(seen) == 32
    for z, signs in itertools.product(range(4), itertools.product((0, 1), repeat=3)):
        assert seen[(z, signs)] == 8 * z + signs[0] + 2 * signs[1] + 4 * signs[2]


# --------------------------------------------------------------------------- STQ1_0 pack / unpack


def test_stq_roundtrip_grid_inputs():
    rng = np.random.default_rng(3)
    for rows, K in [(16, 256), (32, 768), (64, 2048)]:
        w, *_ = grid_weights(rng, rows, K)
        b = F.stq1_pack(w)
        u = F.stq1_unpack(b, rows, K)
        assert np.array_equal(u.astype(np.float32), w)
        assert np.array_equal(np.signbit(u), np.signbit(w))
        assert np.array_equal(F.stq1_pack(u.astype(np.float32)), b)


@pytest.mark.parametrize("dval", [0.0, 2.0 ** -24, 1.0, 65504.0, 6.1e-5])
def test_stq_canonical_bytes_roundtrip_all_codes(dval):
    # Every one of the 32 codes in every lane position, with edge scales.
    rows, K = 16, 256
    codes = (np.arange(rows * 64).reshape(rows, 1, 64) + np.arange(rows)[:, None, None]) % 32
    dbits = np.full((rows, 1), F.fp16_encode_rne(dval), dtype=np.uint16)
    if dval == 0.0:
        codes = np.zeros_like(codes)  # canonical form of a zero block
    b = F.stq1_layout(codes, dbits)
    u = F.stq1_unpack(b, rows, K).astype(np.float32)
    assert np.array_equal(F.stq1_pack(u), b)


def _read_code_by_loops(packed, rows, K, r, j):
    """Second reading of the byte layout, element by element, with plain loops."""
    nb = K // 256
    tile, rr = divmod(r, 16)
    b, jj = divmod(j, 64)
    base = (tile * nb + b) * 672
    g, h = rr % 8, rr // 8
    t, s = jj // 16, jj % 16
    lane = 4 * g + t
    i = 2 * s + h
    words = [int.from_bytes(bytes(packed[base + 32 + 16 * lane + 4 * w: base + 36 + 16 * lane + 4 * w]), "little") for w in range(4)]
    words.append(int.from_bytes(bytes(packed[base + 544 + 4 * lane: base + 548 + 4 * lane]), "little"))
    stream = sum(wd << (32 * n) for n, wd in enumerate(words))
    code = (stream >> (5 * i)) & 31
    dword = int.from_bytes(bytes(packed[base + 4 * g: base + 4 * g + 4]), "little")
    dbits = (dword >> (16 * h)) & 0xFFFF
    return code, dbits


def test_stq_layout_second_reading():
    rng = np.random.default_rng(4)
    rows, K = 32, 512
    w, z, s, d = grid_weights(rng, rows, K)
    b = F.stq1_pack(w)
    for r in range(rows):
        for j in range(K // 4):
            code, dbits = _read_code_by_loops(b, rows, K, r, j)
            assert code >> 3 == z[r, j]
            nz = [l for l in range(4) if l != z[r, j]]
            for n, l in enumerate(nz):
                assert ((code >> n) & 1) == (s[r, j, l] < 0)
            assert F.fp16_decode(np.uint16(dbits)) == d[r, j // 64]


def test_stq_pack_rule_off_grid():
    # Upstream rule: d = fp16(amax); zero at argmin |w| (first lane on ties);
    # remaining lanes keep their sign.  Checked group by group with loops.
    rng = np.random.default_rng(5)
    rows, K = 16, 512
    w = rng.normal(0, 0.05, (rows, K)).astype(np.float32)
    w[0, 0:4] = [0.1, -0.1, 0.1, 0.1]        # tie -> lane 0
    w[1, 4:8] = [0.3, 0.2, -0.2, 0.2]        # tie on |.| -> lane 1
    w[2, 8:12] = [-0.0, 0.0, 1.0, -1.0]      # tie between +-0 -> lane 0
    code, dbits = F.stq1_codes_from_float(w)
    d = F.fp16_decode(dbits)
    for r in range(rows):
        for b in range(K // 256):
            amax = np.max(np.abs(w[r, 256 * b: 256 * b + 256]).astype(np.float64))
            assert d[r, b] == np.float64(np.float16(amax))
            for j in range(64):
                grp = w[r, 256 * b + 4 * j: 256 * b + 4 * j + 4].astype(np.float64)
                zref = min(range(4), key=lambda l: (abs(grp[l]), l))
                c = code[r, b, j]
                assert c >> 3 == zref
                nz = [l for l in range(4) if l != zref]
                for n, l in enumerate(nz):
                    assert ((c >> n) & 1) == int(math.copysign(1.0, grp[l]) < 0)


def test_stq_pack_rejects_nonfinite_and_overrange():
    w = np.zeros((16, 256), np.float32)
    w[3, 7] = np.nan
    with pytest.raises(F.NonFiniteError):
        F.stq1_pack(w)
    w[3, 7] = 70000.0
    with pytest.raises(F.NonFiniteError):
        F.stq1_pack(w)


# --------------------------------------------------------------------------- scalar formats


def test_e2m1_value_set_golden():
    vals = [float(v) for v in open(os.path.join(GOLDEN, "e2m1_values.txt")).read().split("\n")[-2].split()]
    got = F.e2m1_decode(np.arange(16))
    assert np.array_equal(got, np.array(vals))
    assert np.array_equal(np.signbit(got[8:]), np.ones(8, bool))


def test_ue8m0_is_power_of_two():
    e = np.arange(256, dtype=np.uint8)
    v = F.ue8m0_decode(e)
    for i in range(255):
        assert v[i] == 2.0 ** (i - 127)
    assert np.isnan(v[255])


def test_e4m3_code_table():
    v = F.e4m3_decode(np.arange(256, dtype=np.uint8))
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF])
    assert np.sum(~np.isnan(v)) == 254
    assert v[0x7E] == 448.0 and np.nanmax(v) == 448.0
    assert v[0x01] == 2.0 ** -9 and v[0x08] == 2.0 ** -6 and v[0x38] == 1.0
    pos = v[0:0x7F]
    assert np.all(np.diff(pos) > 0)
    assert np.array_equal(v[0x80:0xFF], -pos) and np.signbit(v[0x80])


def test_fp16_and_bf16_decode_match_library():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    a = F.fp16_decode(bits)
    b = torch.from_numpy(bits.view(np.int16)).view(torch.float16).double().numpy()
    assert np.array_equal(np.nan_to_num(a, nan=7.0), np.nan_to_num(b, nan=7.0))
    c = F.bf16_decode(bits)
    d = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.array_equal(np.nan_to_num(c, nan=7.0), np.nan_to_num(d, nan=7.0))


def test_bf16_rne_matches_library_cast():
    rng = np.random.default_rng(6)
    x = np.concatenate([
        rng.normal(0, 1, 100000), rng.normal(0, 1e-38, 1000), rng.normal(0, 1e38, 1000),
        [0.0, -0.0, 3.4e38, -3.4e38, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 2 ** -133, 2 ** -134],
    ]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(F.bf16_encode_rne(x.astype(np.float64)), ref)


def _nearest_even(values, table):
    """Brute-force nearest grid value; ties -> the code with even last bit."""
    out = []
    for v in values:
        best = None
        for code, t in table:
            dist = abs(abs(v) - t)
            key = (dist, code & 1)
            if best is None or key < best[0]:
                best = (key, code, t)
        out.append(best[1])
    return np.array(out)


def test_e4m3_rounding_brute_force():
    table = [(c, F.e4m3_decode(np.uint8(c))) for c in range(0x7F)]
    rng = np.random.default_rng(7)
    v = np.concatenate([rng.uniform(0, 448, 3000), rng.uniform(0, 2 ** -5, 3000),
                        [(table[i][1] + table[i + 1][1]) / 2 for i in range(126)]])
    got = F.e4m3_encode_grid(F.round_to_binary(v, 3, -6)) & 0x7F
    assert np.array_equal(got, _nearest_even(v, table))


def test_e2m1_rounding_brute_force():
    table = [(c, F.e2m1_decode(np.uint8(c))) for c in range(8)]
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    rng = np.random.default_rng(8)
    v = np.concatenate([rng.uniform(0, 6, 4000), mids])
    got = F.e2m1_encode_grid(F.round_to_binary(v, 1, 0)) & 7
    assert np.array_equal(got, _nearest_even(v, table))
    assert list(F.e2m1_decode(_nearest_even(mids, table))) == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]


# --------------------------------------------------------------------------- MXFP8 activation quant


def _check_group_quant(vals, codes, sc):
    vals = np.asarray(vals, np.float64)
    amax = np.max(np.abs(vals))
    if amax == 0:
        assert sc == 127
    else:
        k = int(sc) - 127
        assert amax * 2.0 ** -k <= 448.0
        if sc > 0:
            assert amax * 2.0 ** -(k - 1) > 448.0      # smallest such power of two
    deq = F.e4m3_decode(codes) * 2.0 ** (int(sc) - 127)
    # each code is the nearest E4M3 grid point of v * 2**-k (ties even)
    table = [(c, F.e4m3_decode(np.uint8(c))) for c in range(0x7F)]
    ref = _nearest_even(np.abs(vals) * 2.0 ** -(int(sc) - 127), table)
    assert np.array_equal(codes & 0x7F, ref)
    assert np.array_equal(codes >> 7, np.signbit(vals).astype(np.uint8))
    return deq


def test_mxfp8_quant_exhaustive_bf16_fixed_companion():
    # Every BF16 pattern, in a group whose amax is fixed at 1.0 by a companion
    # element (so the scale is 2^-8 unless the pattern itself is larger).
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    v = F.bf16_decode(bits)
    fin = np.isfinite(v)
    x = np.zeros((65536, 32))
    x[:, 0] = np.where(fin, v, 0.0)
    x[:, 1] = 1.0
    codes, sc = F.mxfp8_quantize(x)
    a = np.abs(x[:, 0])
    exp_sc = np.where(a <= 1.0, 119, F.mxfp8_scale_exponent(np.maximum(a, 1.0)))
    assert np.array_equal(sc[:, 0], exp_sc)
    # brute-force rounding of every pattern (vectorised nearest over the table)
    vals = F.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    y = a * np.ldexp(1.0, -(sc[:, 0].astype(np.int64) - 127))
    dist = np.abs(y[:, None] - vals[None, :])
    dmin = dist.min(axis=1, keepdims=True)
    cand = dist == dmin
    even = cand & (np.arange(0x7F)[None, :] % 2 == 0)
    pick = np.where(even.any(axis=1), np.argmax(even, axis=1), np.argmax(cand, axis=1))
    assert np.array_equal(codes[:, 0] & 0x7F, pick)
    assert np.array_equal(codes[:, 0] >> 7, np.signbit(x[:, 0]).astype(np.uint8))


def test_mxfp8_quant_exhaustive_bf16_own_amax():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    v = F.bf16_decode(bits)
    fin = np.isfinite(v)
    x = np.zeros((65536, 32))
    x[:, 5] = np.where(fin, v, 0.0)
    codes, sc = F.mxfp8_quantize(x)
    a = np.abs(x[:, 5])
    nz = a > 0
    k = sc[:, 0].astype(np.int64) - 127
    assert np.all(a[nz] * np.ldexp(1.0, -k[nz]) <= 448.0)
    big = nz & (sc[:, 0] > 0)
    assert np.all(a[big] * np.ldexp(1.0, -(k[big] - 1)) > 448.0)
    assert np.all(sc[~nz, 0] == 127)
    # the group maximum is represented to within half an E4M3 ulp of its binade
    deq = F.e4m3_decode(codes[:, 5]) * np.ldexp(1.0, k)
    rel = np.abs(deq[nz] - x[nz, 5]) / np.abs(x[nz, 5])
    assert np.all(rel <= 2.0 ** -4 + 1e-15)
    for i in np.random.default_rng(9).integers(0, 65536, 300):
        if fin[i]:
            _check_group_quant(x[i], codes[i, :], sc[i, 0])


def test_mxfp8_quant_nonfinite_and_zero_groups():
    x = np.zeros((3, 64))
    x[0, 3] = np.inf
    x[1, 40] = np.nan
    x[2, :32] = -0.0
    codes, sc = F.mxfp8_quantize(x)
    assert sc[0, 0] == 255 and np.all(codes[0, :32] == 0x7F) and sc[0, 1] == 127
    assert sc[1, 1] == 255 and np.all(codes[1, 32:] == 0x7F)
    assert sc[2, 0] == 127 and np.all(codes[2, :32] == 0x80) and np.all(codes[2, 32:] == 0)


def test_mxfp8_negative_underflow_keeps_sign():
    x = np.zeros((1, 32))
    x[0, 0] = 448.0
    x[0, 1] = -2.0 ** -12      # rounds to zero at scale 2^0
    codes, sc = F.mxfp8_quantize(x)
    assert sc[0, 0] == 127 and codes[0, 1] == 0x80 and codes[0, 0] == 0x7E


# --------------------------------------------------------------------------- MXFP4 weights


def test_mxfp4_roundtrip_and_rule():
    rng = np.random.default_rng(10)
    rows, K = 8, 256
    w = (rng.normal(0, 1, (rows, K)) * np.exp2(rng.integers(-20, 20, (rows, 1)))).astype(np.float32)
    codes, sc = F.mxfp4_pack(w)
    assert codes.shape == (rows, K // 2) and sc.shape == (rows, K // 32)
    table = [(c, F.e2m1_decode(np.uint8(c))) for c in range(8)]
    nib = np.empty((rows, K), np.uint8)
    nib[:, 0::2], nib[:, 1::2] = codes & 15, codes >> 4
    for r in range(rows):
        for b in range(K // 32):
            g = w[r, 32 * b: 32 * b + 32].astype(np.float64)
            k = int(sc[r, b]) - 127
            amax = np.abs(g).max()
            assert amax <= 6 * 2.0 ** k and amax > 6 * 2.0 ** (k - 1)
            ref = _nearest_even(np.abs(g) * 2.0 ** -k, table)
            assert np.array_equal(nib[r, 32 * b: 32 * b + 32] & 7, ref)
            assert np.array_equal(nib[r, 32 * b: 32 * b + 32] >> 3, np.signbit(g).astype(np.uint8))
    # pack(unpack(.)) is the identity on packed weights whose group maximum uses the top binade
    u = F.mxfp4_unpack(codes, sc, rows, K).astype(np.float32)
    c2, s2 = F.mxfp4_pack(u)
    deq2 = F.mxfp4_unpack(c2, s2, rows, K)
    assert np.array_equal(deq2, u.astype(np.float64))


def test_mxfp4_zero_group_and_negative_zero():
    w = np.zeros((1, 64), np.float32)
    w[0, 1] = -0.0
    w[0, 32] = 6.0
    w[0, 33] = -0.1          # rounds to -0 at scale 2^0
    codes, sc = F.mxfp4_pack(w)
    assert sc[0, 0] == 127 and sc[0, 1] == 127
    assert codes[0, 0] == 0x80 and codes[0, 16] == (0x7 | (0x8 << 4))
