"""Low-precision formats of the separate-precision mode (oracle; test infrastructure only).

The pages let the recurrence checkpoint and the copy read for outputs use
different precisions, so that the read copy's rounding never re-enters the
recurrence ("Hybrid-model decoding has a new bottleneck", Interpretation, fourth
paragraph; "SSM decoding stops writing state every step", Interpretation, third
paragraph).  They name an FP16 recurrence with stochastic rounding (same page,
Perspective, second paragraph) and NVFP4 reads (E2M1 values with an E4M3 scale
per 16-element block).  They do not print the rounding rules, so this module
fixes them as follows (each is a reading of the pages; all are exact integer
or IEEE-fp32 procedures so that the CUDA library can match them bit for bit):

FP16 stochastic rounding of an fp32 value x with a uniform 32-bit word r:
    let u be the spacing of fp16 numbers at |x| (2^(floor(log2|x|) - 10), and
    2^-24 below 2^-14); write |x| = (q + f) u with integer q and f in [0, 1);
    round |x| up to (q + 1) u iff r < floor(f * 2^32), else down to q u; keep the
    sign; saturate magnitudes above 65504 to 65504.  P(up) = f up to 2^-32, so
    the rounding is unbiased.

E4M3 (OCP FP8 E4M3FN): bias 7, 3 mantissa bits, subnormal spacing 2^-9,
    largest finite 448; round to nearest, ties to even; saturate at 448.

E2M1 (OCP FP4): magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}; round to nearest,
    ties to the even code; saturate at 6.  Code = sign << 3 | magnitude index,
    with the sign bit set iff x < 0.

FP8 recurrence checkpoint (the pages evaluate NVFP4 reads with an FP16 or an FP8
recurrence, "Hybrid-model decoding has a new bottleneck", Interpretation, fourth
paragraph; the format and rounding are this reading, chosen like the FP16 mode).
Per tile of 64 consecutive rows of one head's state:
    s   = amax(tile) / 448 in fp32, or 1 if amax = 0
    y   = x / s (fp32 divide), stochastically rounded to the E4M3 grid with the
          FP16 rule above and E4M3 spacings (2^(floor(log2|y|) - 3), 2^-9 below
          2^-6), saturating at 448; the random words are those of FP16 SR
    value = E4M3(y) * s (fp32)

NVFP4 read copy.  A tile is 64 consecutive rows (fewer for the last rows) of
one sequence's and head's state matrix, all 128 columns; blocks are 16
consecutive elements along the contracted (contiguous) axis:
    g   = amax(tile) / 2688 in fp32 (2688 = 6 * 448), or 1 if amax = 0
    s_b = E4M3(amax(block) / (6 g))             (fp32 product, then fp32 divide)
    d_b = s_b * g                               (fp32)
    q   = E2M1(|x| / d_b) with the sign of x     (fp32 divide); q = 0 if d_b = 0
    dequantised value = value(q) * d_b          (fp32)
The tile has its own scale rather than one per head state so that a tile holds
the scale of the rows it covers: a state whose rows differ in magnitude (the
channels of a head) gets tighter scales, and the two-level scale stays the
usual NVFP4 layout of a 64 x 128 operand tile.

Two-axis NVFP4 read copy (finer scales: the pages name separate scales along
the state and channel dimensions as a way to cut the remaining read error,
"Hybrid-model decoding has a new bottleneck", Interpretation, fourth
paragraph, and give no format).  Reading taken: one E4M3 scale per column for
each group of 16 consecutive rows (a scale along the channel axis), then the
usual E4M3 block scales along each row's 16 consecutive columns (the state
axis) on the values divided by it:
    g   = amax(tile) / 2688 in fp32, or 1 if amax = 0   (as for NVFP4)
    c   = E4M3(amax over the group's rows of |x_ij| / (6 g))   (fp32 product, then fp32 divide)
    k   = c * g                                         (fp32; the column-group step)
    x'  = x / k                                         (fp32 divide; 0 where k = 0)
    s_b = E4M3(amax_b(|x'|) / (6 * 2^-8))               (fp32 divide by an exact constant)
    d_b = s_b * 2^-8                                    (exact)
    q   = E2M1(|x'| / d_b) with the sign of x'          (fp32 divide); q = 0 if d_b = 0
    dequantised value = (value(q) * d_b) * k            (fp32; the first product is exact)
Each element's step is the product of a scale of its column group and a scale
of its row block, so a state whose channels differ in magnitude along a column
no longer shares one block step across them.  A tile of equal magnitudes
2688 * 2^n round-trips exactly.  The column-group scales add one byte per 16
elements (the copy grows from 0.5625 to 0.625 bytes per element).
"""

from __future__ import annotations

import numpy as np

FP16_MAX = 65504.0
E4M3_MAX = 448.0
E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], np.float64)
NVFP4_BLOCK = 16
NVFP4_TILE_ROWS = 64


# --------------------------------------------------------------------------- FP16 stochastic rounding

def fp16_stochastic_round(x, r) -> np.ndarray:
    """Stochastically round fp32 ``x`` to fp16 with uint32 words ``r``; returns float16."""
    x = np.ascontiguousarray(x, np.float32)
    r = np.asarray(r, np.uint32).astype(np.uint64)
    bits = x.view(np.uint32).astype(np.uint64)
    sign = (bits >> np.uint64(31)) & np.uint64(1)
    E = ((bits >> np.uint64(23)) & np.uint64(0xFF)).astype(np.int64)
    mant = bits & np.uint64(0x7FFFFF)
    normal = E > 0
    M = np.where(normal, mant | np.uint64(0x800000), mant)       # |x| = M * 2^(Eeff - 150)
    Eeff = np.maximum(E, 1)
    s = np.maximum(13, 126 - Eeff).astype(np.uint64)             # fp32 bits below the fp16 spacing
    q = np.where(s >= np.uint64(24), np.uint64(0), M >> np.minimum(s, np.uint64(63)))
    F = np.where(s >= np.uint64(24), M, M & ((np.uint64(1) << np.minimum(s, np.uint64(63))) - np.uint64(1)))
    thr = np.where(s <= np.uint64(32), F << (np.uint64(32) - np.minimum(s, np.uint64(32))),
                   F >> (np.maximum(s, np.uint64(32)) - np.uint64(32)))
    up = (r < thr).astype(np.uint64)
    ulp_exp = np.maximum(Eeff - 127, -14) - 10
    mag = np.ldexp((q + up).astype(np.float64), ulp_exp)
    mag = np.minimum(mag, FP16_MAX)
    finite = E < 255
    mag = np.where(finite, mag, np.where(mant == 0, FP16_MAX, np.nan))
    out = np.where(sign == 1, -mag, mag)
    return out.astype(np.float16)      # exact: every value is on the fp16 grid


def e4m3_stochastic_round(y, r) -> np.ndarray:
    """Stochastically round fp32 ``y`` to the E4M3FN grid with uint32 words ``r`` (the FP16 rule with E4M3
    spacings), saturating at 448; returns float64 values on the grid."""
    y = np.ascontiguousarray(y, np.float32)
    r = np.asarray(r, np.uint32).astype(np.uint64)
    bits = y.view(np.uint32).astype(np.uint64)
    sign = (bits >> np.uint64(31)) & np.uint64(1)
    E = ((bits >> np.uint64(23)) & np.uint64(0xFF)).astype(np.int64)
    mant = bits & np.uint64(0x7FFFFF)
    M = np.where(E > 0, mant | np.uint64(0x800000), mant)        # |y| = M * 2^(Eeff - 150)
    Eeff = np.maximum(E, 1)
    s = np.maximum(20, 141 - Eeff).astype(np.uint64)             # fp32 bits below the E4M3 spacing
    q = np.where(s >= np.uint64(24), np.uint64(0), M >> np.minimum(s, np.uint64(63)))
    F = np.where(s >= np.uint64(24), M, M & ((np.uint64(1) << np.minimum(s, np.uint64(63))) - np.uint64(1)))
    thr = np.where(s <= np.uint64(32), F << (np.uint64(32) - np.minimum(s, np.uint64(32))),
                   F >> (np.maximum(s, np.uint64(32)) - np.uint64(32)))
    up = (r < thr).astype(np.uint64)
    ulp_exp = np.maximum(Eeff - 127, -6) - 3
    mag = np.minimum(np.ldexp((q + up).astype(np.float64), ulp_exp), E4M3_MAX)
    return np.where(sign == 1, -mag, mag)


def fp8_quantize_state(S, words) -> dict:
    """FP8 checkpoint of states [..., rows, 128] by 64-row tiles with uint32 ``words`` [..., rows, 128].

    Returns {"codes": uint8 [..., rows, 128] (E4M3 bit patterns), "s": float32 [..., ceil(rows/64)],
    "values": float32 [..., rows, 128]}."""
    x = np.ascontiguousarray(S, np.float32)
    words = np.asarray(words, np.uint32).reshape(x.shape)
    rows = x.shape[-2]
    codes, scales, values = [], [], []
    for r0 in range(0, rows, NVFP4_TILE_ROWS):
        t = x[..., r0:r0 + NVFP4_TILE_ROWS, :]
        amax = np.abs(t).reshape(*t.shape[:-2], -1).max(axis=-1)
        s = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
        y = (t / s[..., None, None]).astype(np.float32)
        q = e4m3_stochastic_round(y, words[..., r0:r0 + NVFP4_TILE_ROWS, :])
        codes.append(e4m3_code(q))
        scales.append(s)
        values.append((q.astype(np.float32) * s[..., None, None]).astype(np.float32))
    return {"codes": np.concatenate(codes, axis=-2), "s": np.stack(scales, axis=-1),
            "values": np.concatenate(values, axis=-2)}


# --------------------------------------------------------------------------- E4M3 / E2M1

def e4m3_round(v) -> np.ndarray:
    """Round to the E4M3FN grid (nearest, ties to even), saturating at 448.  Returns float64 values."""
    v = np.asarray(v, np.float64)
    a = np.abs(v)
    _, ex = np.frexp(a)                          # a = m * 2^ex, m in [0.5, 1)
    e = ex - 1                                   # floor(log2 a) for a > 0
    spacing = np.where(a >= 2.0 ** -6, np.ldexp(1.0, e - 3), 2.0 ** -9)
    q = np.rint(a / spacing) * spacing           # a / spacing is exact; rint rounds half to even
    q = np.minimum(q, E4M3_MAX)
    return np.where(v < 0, -q, q)


def e4m3_code(q) -> np.ndarray:
    """Bit pattern (uint8) of values already on the E4M3 grid."""
    q = np.asarray(q, np.float64)
    a = np.abs(q)
    _, ex = np.frexp(a)
    e = ex - 1
    normal = a >= 2.0 ** -6
    exp_field = np.where(normal, e + 7, 0)
    mant = np.where(normal, np.ldexp(a, -(e - 3)) - 8.0, np.ldexp(a, 9))
    code = (exp_field.astype(np.int64) << 3) | mant.astype(np.int64)
    code = np.where(q < 0, code | 0x80, code)
    return code.astype(np.uint8)


def e4m3_value(code) -> np.ndarray:
    code = np.asarray(code, np.int64)
    ef = (code >> 3) & 0xF
    m = code & 0x7
    mag = np.where(ef == 0, np.ldexp(m.astype(np.float64), -9), np.ldexp((8 + m).astype(np.float64), ef - 10))
    return np.where(code & 0x80, -mag, mag)


def e2m1_magnitude_code(y) -> np.ndarray:
    """Index into E2M1_VALUES of |y| rounded to nearest, ties to even code, saturating at 6."""
    a = np.abs(np.asarray(y, np.float64))
    spacing = np.where(a < 2.0, 0.5, np.where(a < 4.0, 1.0, 2.0))
    n = np.rint(a / spacing)
    code = np.where(a < 2.0, n, np.where(a < 4.0, n + 2, n + 4))
    return np.minimum(code, 7).astype(np.uint8)


# --------------------------------------------------------------------------- NVFP4 read copy

def nvfp4_quantize(tile) -> dict:
    """Quantise fp32 tiles [..., R, C] (C a multiple of 16) to NVFP4.

    Returns {"codes": uint8 [..., R, C] (one 4-bit code per element, unpacked),
    "packed": uint8 [..., R, C/2] (element 2j in the low nibble), "scales":
    uint8 [..., R, C/16] (E4M3 bit patterns), "g": float32 [...]}.
    """
    x = np.ascontiguousarray(tile, np.float32)
    *lead, R, C = x.shape
    assert C % NVFP4_BLOCK == 0
    ax = np.abs(x)
    amax = ax.reshape(*lead, -1).max(axis=-1) if R * C else np.zeros(lead, np.float32)
    g = np.where(amax > 0, amax / np.float32(2688.0), np.float32(1.0)).astype(np.float32)
    blocks = ax.reshape(*lead, R, C // NVFP4_BLOCK, NVFP4_BLOCK)
    amax_b = blocks.max(axis=-1)                                             # fp32
    t = (np.float32(6.0) * g).astype(np.float32)
    sb_in = (amax_b / t[..., None, None]).astype(np.float32)
    s_b = e4m3_round(sb_in).astype(np.float32)
    d_b = (s_b * g[..., None, None]).astype(np.float32)
    safe = np.where(d_b > 0, d_b, np.float32(1.0)).astype(np.float32)
    yb = (blocks / safe[..., None]).astype(np.float32)
    mag = e2m1_magnitude_code(yb)
    mag = np.where((d_b > 0)[..., None], mag, 0).astype(np.uint8)
    neg = (x.reshape(blocks.shape) < 0) & (d_b > 0)[..., None]
    codes = (mag | (neg.astype(np.uint8) << 3)).reshape(x.shape).astype(np.uint8)
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    return {"codes": codes, "packed": packed, "scales": e4m3_code(s_b), "g": g}


def nvfp4_dequantize(codes, scales, g) -> np.ndarray:
    """Inverse of the read-copy encoding: value(code) * (s_b * g) in fp32; returns float32 [..., R, C]."""
    codes = np.asarray(codes, np.uint8)
    *lead, R, C = codes.shape
    s_b = e4m3_value(scales).astype(np.float32)
    d_b = (s_b * np.asarray(g, np.float32)[..., None, None]).astype(np.float32)
    mag = E2M1_VALUES[codes & 7].astype(np.float32)
    val = (mag.reshape(*lead, R, C // NVFP4_BLOCK, NVFP4_BLOCK) * d_b[..., None]).astype(np.float32)
    val = val.reshape(codes.shape)
    return np.where(codes & 8, -val, val).astype(np.float32)


def nvfp4_roundtrip(tile) -> np.ndarray:
    q = nvfp4_quantize(tile)
    return nvfp4_dequantize(q["codes"], q["scales"], q["g"])


def nvfp4_quantize_state(S) -> dict:
    """Quantise states [..., rows, 128] tile by tile (64-row tiles).  Returns packed codes
    [..., rows, 64], scales [..., rows, 8] and g [..., ceil(rows/64)]."""
    S = np.ascontiguousarray(S, np.float32)
    rows = S.shape[-2]
    parts = [nvfp4_quantize(S[..., r0:r0 + NVFP4_TILE_ROWS, :]) for r0 in range(0, rows, NVFP4_TILE_ROWS)]
    return {"codes": np.concatenate([p["codes"] for p in parts], axis=-2),
            "packed": np.concatenate([p["packed"] for p in parts], axis=-2),
            "scales": np.concatenate([p["scales"] for p in parts], axis=-2),
            "g": np.stack([p["g"] for p in parts], axis=-1)}


def nvfp4_roundtrip_state(S) -> np.ndarray:
    """fp32 values of the read copy of states [..., rows, 128] (64-row tiles)."""
    S = np.ascontiguousarray(S, np.float32)
    rows = S.shape[-2]
    return np.concatenate([nvfp4_roundtrip(S[..., r0:r0 + NVFP4_TILE_ROWS, :])
                           for r0 in range(0, rows, NVFP4_TILE_ROWS)], axis=-2)


# --------------------------------------------------------------------------- two-axis NVFP4 read copy

NVFP4D_GROUP_ROWS = 16
NVFP4D_BLOCK_STEP = np.float32(2.0 ** -8)


def nvfp4d_quantize(tile) -> dict:
    """Two-axis NVFP4 encoding of fp32 tiles [..., R, C] (R <= 64, C a multiple of 16).  Returns "codes"
    (unpacked), "packed" [..., R, C/2], "scales" [..., R, C/16] (E4M3 row-block scales), "colscales"
    [..., ceil(R/16), C] (E4M3 column-group scales) and "g" [...]."""
    x = np.ascontiguousarray(tile, np.float32)
    *lead, R, C = x.shape
    assert C % NVFP4_BLOCK == 0
    ax = np.abs(x)
    amax = ax.reshape(*lead, -1).max(axis=-1) if R * C else np.zeros(lead, np.float32)
    g = np.where(amax > 0, amax / np.float32(2688.0), np.float32(1.0)).astype(np.float32)
    six_g = (np.float32(6.0) * g).astype(np.float32)
    ngr = -(-R // NVFP4D_GROUP_ROWS)
    cs = np.empty(tuple(lead) + (ngr, C), np.float32)
    k = np.empty_like(x)
    for gi in range(ngr):
        rows = slice(gi * NVFP4D_GROUP_ROWS, min(R, (gi + 1) * NVFP4D_GROUP_ROWS))
        gm = ax[..., rows, :].max(axis=-2)                                   # [..., C]
        c = e4m3_round((gm / six_g[..., None]).astype(np.float32)).astype(np.float32)
        cs[..., gi, :] = c
        k[..., rows, :] = (c * g[..., None]).astype(np.float32)[..., None, :]
    xp = np.where(k > 0, x / np.where(k > 0, k, np.float32(1.0)), np.float32(0.0)).astype(np.float32)
    blocks = np.abs(xp).reshape(*lead, R, C // NVFP4_BLOCK, NVFP4_BLOCK)
    amax_b = blocks.max(axis=-1)
    s_b = e4m3_round((amax_b / np.float32(6.0 * 2.0 ** -8)).astype(np.float32)).astype(np.float32)
    d_b = (s_b * NVFP4D_BLOCK_STEP).astype(np.float32)
    safe = np.where(d_b > 0, d_b, np.float32(1.0)).astype(np.float32)
    mag = e2m1_magnitude_code((blocks / safe[..., None]).astype(np.float32))
    mag = np.where((d_b > 0)[..., None], mag, 0).astype(np.uint8)
    neg = (xp.reshape(blocks.shape) < 0) & (d_b > 0)[..., None]
    codes = (mag | (neg.astype(np.uint8) << 3)).reshape(x.shape).astype(np.uint8)
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    return {"codes": codes, "packed": packed, "scales": e4m3_code(s_b), "colscales": e4m3_code(cs), "g": g}


def nvfp4d_dequantize(codes, scales, colscales, g) -> np.ndarray:
    """value(code) * (s_b * 2^-8) * (c * g) in fp32; returns float32 [..., R, C]."""
    codes = np.asarray(codes, np.uint8)
    *lead, R, C = codes.shape
    d_b = (e4m3_value(scales).astype(np.float32) * NVFP4D_BLOCK_STEP).astype(np.float32)
    mag = E2M1_VALUES[codes & 7].astype(np.float32)
    v = (mag.reshape(*lead, R, C // NVFP4_BLOCK, NVFP4_BLOCK) * d_b[..., None]).astype(np.float32).reshape(codes.shape)
    k = (e4m3_value(colscales).astype(np.float32) * np.asarray(g, np.float32)[..., None, None]).astype(np.float32)
    k_rows = np.repeat(k, NVFP4D_GROUP_ROWS, axis=-2)[..., :R, :]
    v = (v * k_rows).astype(np.float32)
    return np.where(codes & 8, -v, v).astype(np.float32)


def nvfp4d_quantize_state(S) -> dict:
    """Two-axis encoding of states [..., rows, 128] by 64-row tiles: packed codes [..., rows, 64], row-block
    scales [..., rows, 8], column-group scales [..., ceil(rows/16), 128] and g [..., tiles]."""
    S = np.ascontiguousarray(S, np.float32)
    rows = S.shape[-2]
    parts = [nvfp4d_quantize(S[..., r0:r0 + NVFP4_TILE_ROWS, :]) for r0 in range(0, rows, NVFP4_TILE_ROWS)]
    return {"codes": np.concatenate([p["codes"] for p in parts], axis=-2),
            "packed": np.concatenate([p["packed"] for p in parts], axis=-2),
            "scales": np.concatenate([p["scales"] for p in parts], axis=-2),
            "colscales": np.concatenate([p["colscales"] for p in parts], axis=-2),
            "g": np.stack([p["g"] for p in parts], axis=-1)}


def nvfp4d_roundtrip_state(S) -> np.ndarray:
    """fp32 values of the two-axis read copy of states [..., rows, 128]."""
    S = np.ascontiguousarray(S, np.float32)
    rows = S.shape[-2]
    out = []
    for r0 in range(0, rows, NVFP4_TILE_ROWS):
        q = nvfp4d_quantize(S[..., r0:r0 + NVFP4_TILE_ROWS, :])
        out.append(nvfp4d_dequantize(q["codes"], q["scales"], q["colscales"], q["g"]))
    return np.concatenate(out, axis=-2)
