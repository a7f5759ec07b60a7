"""Bit-level formats: IEEE half / bfloat16, OCP-MX E4M3 / E2M1 / UE8M0, and the
STQ1_0 3:4 sparse-ternary block in this library's own byte layout.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  Plain numpy, float64.

Every encoder rounds with ``round_to_binary`` (round to nearest, ties to even,
on the exact float64 value) and every decoder evaluates the format's defining
formula.  Nothing here is shared with the CUDA library.
"""

import numpy as np

# ----------------------------------------------------------------------------
# Generic round-to-nearest-even onto a binary floating-point grid
# ----------------------------------------------------------------------------


def round_to_binary(v, frac_bits, emin):
    """Round float64 ``v`` to the nearest value of a binary floating format with
    ``frac_bits`` fraction bits and smallest normal exponent ``emin``; values
    below 2**emin use the subnormal quantum 2**(emin - frac_bits).  Ties go to
    the value whose last fraction bit is 0.  Overflow is not handled here: the
    callers guarantee the range.  The sign (including -0) is kept."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    _, E = np.frexp(a)               # a = m * 2**E, m in [0.5, 1)
    e = np.maximum(E - 1, emin)      # binade exponent, clamped into the subnormal range
    q = np.ldexp(1.0, e - frac_bits)  # grid spacing in that binade (power of two)
    with np.errstate(invalid="ignore"):
        r = np.rint(a / q) * q       # a / q is exact; rint rounds half to even
    return np.copysign(r, v)


# ----------------------------------------------------------------------------
# IEEE binary16 and bfloat16
# ----------------------------------------------------------------------------


def fp16_decode(bits):
    """IEEE binary16 bit patterns (uint16) -> float64."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def fp16_encode_rne(v):
    """float64 -> IEEE binary16 bits, round to nearest even (numpy's IEEE cast)."""
    return np.asarray(v, dtype=np.float64).astype(np.float16).view(np.uint16)


def bf16_decode(bits):
    """bfloat16 = the top 16 bits of an IEEE binary32 -> float64."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    with np.errstate(invalid="ignore"):  # signalling-NaN patterns widen to a quiet NaN
        return b.view(np.float32).astype(np.float64)


def bf16_encode_rne(v):
    """float64 -> bfloat16 bits (8 significant bits, exponent range of binary32),
    round to nearest even on the exact value; overflow -> +-inf, NaN -> 0x7FC0."""
    v = np.asarray(v, dtype=np.float64)
    r = round_to_binary(v, 7, -126)
    with np.errstate(over="ignore"):
        f = r.astype(np.float32)     # exact for every grid value; 2**128 -> inf
    bits = (f.view(np.uint32) >> 16).astype(np.uint16)
    return np.where(np.isnan(v), np.uint16(0x7FC0), bits).astype(np.uint16)


# ----------------------------------------------------------------------------
# OCP-MX element and scale types
# ----------------------------------------------------------------------------

E4M3_MAX = 448.0
E2M1_MAX = 6.0


def e4m3_decode(codes):
    """E4M3 ("FN" variant): sign, 4 exponent bits (bias 7), 3 mantissa bits;
    exponent field 0 is subnormal (m/8 * 2**-6); S.1111.111 is NaN; no infinity."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s, ef, m = c >> 7, (c >> 3) & 15, c & 7
    val = np.where(ef == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.ldexp(1.0, ef - 7))
    val = np.where((c & 0x7F) == 0x7F, np.nan, val)
    return np.where(s == 1, -val, val)


def e4m3_encode_grid(r):
    """Exact E4M3 value (|r| <= 448, already on the grid) -> code; sign bit from
    signbit(r) so that -0 encodes as 0x80."""
    r = np.asarray(r, dtype=np.float64)
    a = np.abs(r)
    if np.any(a > E4M3_MAX):
        raise ValueError("value above the E4M3 range")
    _, E = np.frexp(a)
    e = E - 1
    with np.errstate(invalid="ignore", divide="ignore"):
        mant_norm = np.rint((a / np.ldexp(1.0, e) - 1.0) * 8.0)
    mant_sub = np.rint(a * 2.0 ** 9)
    sub = a < 2.0 ** -6
    code = np.where(sub, mant_sub, (e + 7) * 8 + mant_norm)
    code = np.where(a == 0, 0, code).astype(np.int64)
    code = code | (np.signbit(r).astype(np.int64) << 7)
    return code.astype(np.uint8)


def e2m1_decode(codes):
    """E2M1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0; exponent
    field 0 is subnormal (m * 0.5).  Values {0, 0.5, 1, 1.5, 2, 3, 4, 6} x +-1."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64) & 15
    s, ef, m = c >> 3, (c >> 1) & 3, c & 1
    val = np.where(ef == 0, m * 0.5, (1.0 + m / 2.0) * np.ldexp(1.0, ef - 1))
    return np.where(s == 1, -val, val)


def e2m1_encode_grid(r):
    """Exact E2M1 value (|r| <= 6, on the grid) -> 4-bit code, sign from signbit."""
    r = np.asarray(r, dtype=np.float64)
    a = np.abs(r)
    if np.any(a > E2M1_MAX):
        raise ValueError("value above the E2M1 range")
    _, E = np.frexp(a)
    e = E - 1
    with np.errstate(invalid="ignore", divide="ignore"):
        mant = np.rint((a / np.ldexp(1.0, e) - 1.0) * 2.0)
    code = np.where(a < 1.0, np.rint(a * 2.0), (e + 1) * 2 + mant)
    code = np.where(a == 0, 0, code).astype(np.int64)
    code = code | (np.signbit(r).astype(np.int64) << 3)
    return code.astype(np.uint8)


def ue8m0_decode(e):
    """UE8M0 scale: 2**(e - 127) for e in 0..254; e = 255 is NaN."""
    e = np.asarray(e, dtype=np.uint8).astype(np.int64)
    return np.where(e == 255, np.nan, np.ldexp(1.0, e - 127))


# ----------------------------------------------------------------------------
# MXFP8 activation quantisation (E4M3 elements, UE8M0 scale per 32 along K)
# ----------------------------------------------------------------------------


def mxfp8_scale_exponent(amax):
    """Per group: k = the smallest integer with amax <= 448 * 2**k (448 = 1.75 *
    2**8).  With amax = m * 2**E, m in [1, 2): k = E - 8 if m <= 1.75, else E - 7.
    Returned as the biased UE8M0 field e = clamp(k + 127, 0, 254); amax == 0 gives
    e = 127.  Non-finite groups are handled by the caller."""
    amax = np.asarray(amax, dtype=np.float64)
    fm, E = np.frexp(amax)
    m, e = 2.0 * fm, E - 1
    k = np.where(m <= 1.75, e - 8, e - 7)
    sc = np.clip(k + 127, 0, 254)
    return np.where(amax == 0, 127, sc).astype(np.int64)


def mxfp8_quantize(v):
    """Quantise rows of float64 values (exact BF16 or FP32 inputs) [rows, K],
    K % 32 == 0, to MXFP8: codes [rows, K] uint8 and scales [rows, K/32] uint8.

    Scale: smallest power of two putting the group's amax <= 448 (the config text
    of the single-expert W4A8 GEMM: "UE8M0 scale = smallest power of two putting
    the group's amax <= 448").  Codes: E4M3 round-to-nearest-even of v * 2**-k,
    subnormals included, sign kept.  A group holding NaN or Inf gets e = 255 and
    all codes 0x7F."""
    v = np.asarray(v, dtype=np.float64)
    rows, K = v.shape
    if K % 32:
        raise ValueError("K must be a multiple of 32")
    g = v.reshape(rows, K // 32, 32)
    bad = ~np.all(np.isfinite(g), axis=2)
    amax = np.max(np.abs(np.where(np.isfinite(g), g, 0.0)), axis=2)
    sc = mxfp8_scale_exponent(amax)
    sc = np.where(bad, 255, sc)
    k = np.where(bad, 0, sc - 127)
    scaled = np.ldexp(np.where(np.isfinite(g), g, 0.0), -k[:, :, None])
    r = round_to_binary(scaled, 3, -6)
    codes = e4m3_encode_grid(r)
    codes = np.where(bad[:, :, None], np.uint8(0x7F), codes)
    return codes.reshape(rows, K).astype(np.uint8), sc.astype(np.uint8)


def mxfp8_dequantize(codes, scales):
    """MXFP8 codes [rows, K] and scales [rows, K/32] -> float64 values."""
    codes = np.asarray(codes, dtype=np.uint8)
    rows, K = codes.shape
    s = ue8m0_decode(scales).reshape(rows, K // 32, 1)
    return (e4m3_decode(codes).reshape(rows, K // 32, 32) * s).reshape(rows, K)


# ----------------------------------------------------------------------------
# MXFP4 weights (E2M1 elements, UE8M0 scale per 32 along K)
# ----------------------------------------------------------------------------


class NonFiniteError(ValueError):
    pass


def mxfp4_scale_exponent(amax):
    """Per group: k = the smallest integer with amax <= 6 * 2**k (6 = 1.5 * 2**2).
    With amax = m * 2**E, m in [1, 2): k = E - 2 if m <= 1.5, else E - 1.
    Biased e = clamp(k + 127, 0, 254); amax == 0 gives e = 127.  (The pages fix
    only "FP4 E2M1 g32 + UE8M0"; this mirrors the activation rule with 6 in place
    of 448.)"""
    amax = np.asarray(amax, dtype=np.float64)
    fm, E = np.frexp(amax)
    m, e = 2.0 * fm, E - 1
    k = np.where(m <= 1.5, e - 2, e - 1)
    sc = np.clip(k + 127, 0, 254)
    return np.where(amax == 0, 127, sc).astype(np.int64)


def mxfp4_pack(w):
    """float32 weights [rows, K] -> (codes [rows, K/2] uint8 with element 2i in the
    low nibble, scales [rows, K/32] uint8).  Codes are E2M1 round-to-nearest-even
    of w * 2**-k with the sign bit of w kept.  Non-finite weights are an error."""
    w = np.asarray(w, dtype=np.float32).astype(np.float64)
    rows, K = w.shape
    if K % 32:
        raise ValueError("K must be a multiple of 32")
    if not np.all(np.isfinite(w)):
        raise NonFiniteError("non-finite weight")
    g = w.reshape(rows, K // 32, 32)
    sc = mxfp4_scale_exponent(np.max(np.abs(g), axis=2))
    r = round_to_binary(np.ldexp(g, -(sc - 127)[:, :, None]), 1, 0)
    code = e2m1_encode_grid(r).reshape(rows, K).astype(np.uint8)
    packed = (code[:, 0::2] | (code[:, 1::2] << 4)).astype(np.uint8)
    return packed, sc.astype(np.uint8)


def mxfp4_unpack(codes, scales, rows, K):
    """(codes, scales) -> float64 weights [rows, K] = e2m1(code) * 2**(e - 127)."""
    codes = np.asarray(codes, dtype=np.uint8).reshape(rows, K // 2)
    nib = np.empty((rows, K), dtype=np.uint8)
    nib[:, 0::2] = codes & 15
    nib[:, 1::2] = codes >> 4
    s = ue8m0_decode(np.asarray(scales, dtype=np.uint8).reshape(rows, K // 32))
    return (e2m1_decode(nib).reshape(rows, K // 32, 32) * s[:, :, None]).reshape(rows, K)


def mxfp4_unpack_f32(codes, scales, rows, K):
    """The float32 result the unpack entry point returns: the exact value rounded
    to binary32 (only overflow to +-inf can change it)."""
    with np.errstate(over="ignore"):
        return mxfp4_unpack(codes, scales, rows, K).astype(np.float32)


# ----------------------------------------------------------------------------
# STQ1_0: 3:4 sparse ternary, 256-weight blocks, one FP16 scale, 42 bytes/block
# ----------------------------------------------------------------------------
#
# Pattern of one four-weight group (5 bits, 32 values): c = 8*z + s, where z is
# the zero lane (0..3) and bit n of s (n = 0, 1, 2) is 1 when the n-th non-zero
# lane, counting lanes upward, is negative.  Weight = d * (0 if lane == z else
# +-1).  Group j of block b of a row covers k = 256*b + 4*j + lane.
#
# Byte layout of a matrix [rows, K] (rows % 16 == 0, K % 256 == 0): tiles of 16
# consecutive rows, each tile stored as its K/256 "tile-blocks" in block order;
# a tile-block (16 rows x 256 k, 672 bytes = 16 x 42) is
#   [0, 32)     8 little-endian words; word g = d(row g) | d(row g+8) << 16
#   [32, 544)   lane L (0..31) owns 16 bytes at 32 + 16*L: words 0..3 of its stream
#   [544, 672)  lane L's word 4 at 544 + 4*L
# Lane L = 4*g + t owns the 32 codes of rows g and g+8 whose group index j lies
# in [16*t, 16*t + 16) (k in [64*t, 64*t + 64) of the block); code number
# i = 2*s + h belongs to row g + 8*h and group j = 16*t + s, and occupies bits
# [5*i, 5*i + 5) of the lane's 160-bit stream (words 0..4, little-endian).  Tile
# rows are relative to the tile.

STQ_BLOCK = 256
STQ_TILE_ROWS = 16
STQ_BLOCK_BYTES = 42
STQ_TILE_BLOCK_BYTES = STQ_TILE_ROWS * STQ_BLOCK_BYTES  # 672

# non-zero lanes, in ascending order, for each zero lane z
_NZ_LANES = np.array([[1, 2, 3], [0, 2, 3], [0, 1, 3], [0, 1, 2]], dtype=np.int64)


def stq1_packed_bytes(rows, K):
    return rows * (K // STQ_BLOCK) * STQ_BLOCK_BYTES


def stq1_pattern(code):
    """5-bit code -> the four lane values in {-1, 0, +1} (float64 [..., 4])."""
    c = np.asarray(code, dtype=np.int64)
    z, s = c >> 3, c & 7
    out = np.ones(c.shape + (4,), dtype=np.float64)
    lanes = _NZ_LANES[z]                                  # [..., 3]
    for n in range(3):
        neg = (s >> n) & 1
        np.put_along_axis(out, lanes[..., n:n + 1], np.where(neg == 1, -1.0, 1.0)[..., None], axis=-1)
    np.put_along_axis(out, z[..., None], 0.0, axis=-1)
    return out


def _lane_maps():
    """For lane L and code number i: (tile row, group index within the block)."""
    L = np.arange(32)[:, None]
    i = np.arange(32)[None, :]
    g, t = L // 4, L % 4
    s, h = i // 2, i % 2
    return g + 8 * h, 16 * t + s


def stq1_codes_from_float(w):
    """Upstream quantiser rule ("Hy4-preview-GGUF", section 3, "Our encoder"
    paragraph, describing upstream): per 256-block d = amax rounded to FP16; per
    group the zero goes to argmin |w| (first lane on ties); the other three lanes
    keep their sign.  Returns (codes [rows, K/256, 64] int64, d bits [rows, K/256]
    uint16).  Exact on inputs already on the ternary grid."""
    w = np.asarray(w, dtype=np.float32).astype(np.float64)
    rows, K = w.shape
    if K % STQ_BLOCK:
        raise ValueError("K must be a multiple of 256")
    if not np.all(np.isfinite(w)):
        raise NonFiniteError("non-finite weight")
    nb = K // STQ_BLOCK
    amax = np.max(np.abs(w.reshape(rows, nb, STQ_BLOCK)), axis=2)
    if np.any(amax > 65504.0):
        raise NonFiniteError("block amax above the FP16 range")
    dbits = fp16_encode_rne(amax)
    grp = w.reshape(rows, nb, 64, 4)
    z = np.argmin(np.abs(grp), axis=3)                    # first minimum
    neg = np.signbit(grp).astype(np.int64)
    sbits = np.take_along_axis(neg, _NZ_LANES[z], axis=3)  # signs of the non-zero lanes
    code = 8 * z + sbits[..., 0] + 2 * sbits[..., 1] + 4 * sbits[..., 2]
    code = np.where((fp16_decode(dbits) == 0)[:, :, None], 0, code)
    return code.astype(np.int64), dbits


STQ_LS_ROUNDS = 3


def stq1_codes_ls(w, importance=None, rounds=STQ_LS_ROUNDS):
    """Least-squares STQ1_0 encoder ("Hy4-preview-GGUF", section 3, "Our encoder"):
    the byte format is unchanged, two decisions differ from the upstream rule.

    Per 256-block of a row, with importance v_k >= 0 per column (None: all 1):
      start from the upstream scale d = amax |w|; then, `rounds` times,
      1. per group of four, the zero goes to the lane j minimising the incremental
         cost v_j * (w_j^2 - (|w_j| - d)^2) (first lane on ties), with the current d;
      2. d = sum(v * sel * w) / sum(v * sel^2) over the block, sel = sign(w) on the
         three kept lanes and 0 on the zero lane (0 when the denominator is 0).
    Reading: "alternating for 3 rounds" is taken as three (placement, scale) rounds
    after the upstream start; the stored d is the last scale rounded to FP16, the
    codes are the last placement with the kept lanes' signs.  All arithmetic is
    float64, each cost evaluated as v * (w*w - (|w|-d)*(|w|-d)) in that order.
    Returns (codes [rows, K/256, 64] int64, d bits [rows, K/256] uint16)."""
    w = np.asarray(w, dtype=np.float32).astype(np.float64)
    rows, K = w.shape
    if K % STQ_BLOCK:
        raise ValueError("K must be a multiple of 256")
    if not np.all(np.isfinite(w)):
        raise NonFiniteError("non-finite weight")
    v = np.ones(K) if importance is None else np.asarray(importance, dtype=np.float32).astype(np.float64)
    if v.shape != (K,) or not np.all(np.isfinite(v)) or np.any(v < 0):
        raise ValueError("importance must be K finite non-negative values")
    nb = K // STQ_BLOCK
    x = w.reshape(rows, nb, 64, 4)
    vg = np.broadcast_to(v.reshape(nb, 64, 4), x.shape)
    ax = np.abs(x)
    d = np.max(ax.reshape(rows, nb, STQ_BLOCK), axis=2)
    if np.any(d > 65504.0):
        raise NonFiniteError("block amax above the FP16 range")
    z = np.zeros(x.shape[:3], dtype=np.int64)
    for _ in range(rounds):
        e = ax - d[:, :, None, None]
        cost = vg * (x * x - e * e)
        z = np.argmin(cost, axis=3)                         # first minimum
        keep = np.ones(x.shape, dtype=bool)
        np.put_along_axis(keep, z[..., None], False, axis=3)
        num = np.sum(np.where(keep, vg * ax, 0.0), axis=(2, 3))
        den = np.sum(np.where(keep, vg, 0.0), axis=(2, 3))
        d = np.where(den > 0, num / np.where(den > 0, den, 1.0), 0.0)
    dbits = fp16_encode_rne(d)
    neg = np.signbit(x).astype(np.int64)
    sbits = np.take_along_axis(neg, _NZ_LANES[z], axis=3)
    code = 8 * z + sbits[..., 0] + 2 * sbits[..., 1] + 4 * sbits[..., 2]
    code = np.where((fp16_decode(dbits) == 0)[:, :, None], 0, code)
    return code.astype(np.int64), dbits


def stq1_pack_ls(w, importance=None):
    """float32 weights [rows, K] -> STQ1_0 bytes with the least-squares encoder."""
    code, dbits = stq1_codes_ls(w, importance)
    return stq1_layout(code, dbits)


def stq1_weighted_ssd(w, packed, importance=None):
    """sum_k v_k (w_k - w_hat_k)^2 of a packed matrix against its float source."""
    w = np.asarray(w, dtype=np.float32).astype(np.float64)
    rows, K = w.shape
    v = np.ones(K) if importance is None else np.asarray(importance, dtype=np.float32).astype(np.float64)
    return float(np.sum(v[None, :] * (w - stq1_unpack(packed, rows, K)) ** 2))


def stq1_layout(code, dbits):
    """Codes [rows, K/256, 64] and d bits [rows, K/256] -> packed bytes."""
    rows, nb = dbits.shape
    if rows % STQ_TILE_ROWS:
        raise ValueError("rows must be a multiple of 16")
    nt = rows // STQ_TILE_ROWS
    out = np.zeros((nt, nb, STQ_TILE_BLOCK_BYTES), dtype=np.uint8)
    d = dbits.astype(np.uint32).reshape(nt, 16, nb)
    dw = (d[:, 0:8, :] | (d[:, 8:16, :] << 16)).transpose(0, 2, 1)        # [nt, nb, 8]
    out[:, :, 0:32] = np.ascontiguousarray(dw.astype("<u4")).view(np.uint8).reshape(nt, nb, 32)
    ct = code.reshape(nt, 16, nb, 64)
    trow, tgrp = _lane_maps()                                             # [32 lanes, 32 codes]
    lane_codes = ct[:, trow, :, tgrp].transpose(2, 3, 0, 1).astype(np.uint64)  # [nt, nb, L, i]
    words = np.zeros((nt, nb, 32, 5), dtype=np.uint64)
    for i in range(32):
        sh = 5 * i
        w0, off = sh // 32, sh % 32
        c = lane_codes[..., i]
        words[..., w0] |= (c << np.uint64(off)) & np.uint64(0xFFFFFFFF)
        if off > 27:
            words[..., w0 + 1] |= c >> np.uint64(32 - off)
    w32 = words.astype("<u4")
    out[:, :, 32:544] = np.ascontiguousarray(w32[..., 0:4]).view(np.uint8).reshape(nt, nb, 512)
    out[:, :, 544:672] = np.ascontiguousarray(w32[..., 4]).view(np.uint8).reshape(nt, nb, 128)
    return out.reshape(-1)


def stq1_parse(packed, rows, K):
    """Packed bytes -> (codes [rows, K/256, 64] int64, d bits [rows, K/256] uint16)."""
    nb, nt = K // STQ_BLOCK, rows // STQ_TILE_ROWS
    b = np.asarray(packed, dtype=np.uint8).reshape(nt, nb, STQ_TILE_BLOCK_BYTES)
    dw = b[:, :, 0:32].copy().view("<u4").reshape(nt, nb, 8).astype(np.uint32)
    d = np.empty((nt, 16, nb), dtype=np.uint16)
    d[:, 0:8, :] = (dw & 0xFFFF).transpose(0, 2, 1)
    d[:, 8:16, :] = (dw >> 16).transpose(0, 2, 1)
    words = np.empty((nt, nb, 32, 5), dtype=np.uint64)
    words[..., 0:4] = b[:, :, 32:544].copy().view("<u4").reshape(nt, nb, 32, 4)
    words[..., 4] = b[:, :, 544:672].copy().view("<u4").reshape(nt, nb, 32)
    lane_codes = np.zeros((nt, nb, 32, 32), dtype=np.uint64)
    for i in range(32):
        sh = 5 * i
        w0, off = sh // 32, sh % 32
        c = words[..., w0] >> np.uint64(off)
        if off > 27:
            c |= words[..., w0 + 1] << np.uint64(32 - off)
        lane_codes[..., i] = c & np.uint64(31)
    code = np.zeros((nt, 16, nb, 64), dtype=np.int64)
    trow, tgrp = _lane_maps()
    code[:, trow, :, tgrp] = lane_codes.transpose(2, 3, 0, 1).astype(np.int64)
    return code.reshape(rows, nb, 64), d.reshape(rows, nb)


def stq1_pack(w):
    """float32 weights [rows, K] -> STQ1_0 bytes (rows * K/256 * 42)."""
    code, dbits = stq1_codes_from_float(w)
    return stq1_layout(code, dbits)


def stq1_unpack(packed, rows, K):
    """STQ1_0 bytes -> float64 weights [rows, K]: +-d on the non-zero lanes (the
    sign applied to d, so d = 0 gives +-0) and +0 on the zero lane.  Every value
    is exactly representable in binary32."""
    code, dbits = stq1_parse(packed, rows, K)
    d = fp16_decode(dbits)                                  # [rows, nb]
    pat = stq1_pattern(code)                                # [rows, nb, 64, 4]
    val = np.where(pat == 0, 0.0, np.where(pat < 0, -1.0, 1.0) * d[:, :, None, None])
    return val.reshape(rows, K)
