"""CPU oracle for the frozen-NF4 linear layer with a bf16 LoRA adapter.

TEST INFRASTRUCTURE ONLY.  This module is a plain, slow, obviously-correct
restatement of the method in numpy (fp32 where the method fixes fp32, fp64
elsewhere).  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
and reference legs of ``bench.py`` may import it.  The CUDA library never calls
it, and it imports nothing from the CUDA path: the two share no code, tables or
constants.  Every function names the passage of the pages it follows:

  * "QLoRA, explained" (pofe.ai), section "The math: what is stored and what is
    computed" -- sub-sections "Blockwise absmax quantisation", "NormalFloat 4
    (NF4)", "Double quantisation", "The forward pass and gradients";
  * same page, section "Worked example: quantising one block by hand";
  * same page, section "A toy run: how much does NF4 lose ...";
  * same page, section "The algorithm, step by step";
  * same page, section "Minimal implementation" (two indices per byte).

Readings taken where the pages are silent or garbled (the displayed formulas
and the codebook table did not survive extraction) are stated at each function.

Pins (tests/test_oracle.py) tie every function here to something other than
itself: printed codebook digits and the worked example, closed forms, two
independent inverse-normal routines, torch's own float8/bf16 casts, brute-force
argmin on tiny inputs, finite differences, and the page's toy statistics.
No function in this file is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

# ---------------------------------------------------------------------------
# Fixed format parameters.  "QLoRA, explained" -- "Blockwise absmax
# quantisation" fixes B = 64; "Double quantisation" fixes 256 scales per
# second-level constant.
# ---------------------------------------------------------------------------
BLOCK = 64
GROUP = 256
E4M3_MAX = 448.0


# ---------------------------------------------------------------------------
# a1. The NF4 codebook.
# ---------------------------------------------------------------------------
def norm_ppf(p: float) -> float:
    """Standard-normal quantile Q_X(p), by bisection on math.erfc in fp64.

    Phi(x) = erfc(-x / sqrt(2)) / 2 is monotone, so 200 halvings of [-40, 40]
    pin x to the last bit fp64 can resolve.  Deliberately independent of any
    library quantile routine (the tests compare against two of those).
    """
    if not 0.0 < p < 1.0:
        raise ValueError("p must lie in (0, 1)")
    lo, hi = -40.0, 40.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if 0.5 * math.erfc(-mid / math.sqrt(2.0)) < p:
            lo = mid
        else:
            hi = mid
        if hi - lo <= 0.0:
            break
    return 0.5 * (lo + hi)


def nf4_levels_fp64(ppf=norm_ppf) -> np.ndarray:
    """The 16 NF4 levels in fp64, before rounding to fp32.

    "QLoRA, explained", "NormalFloat 4 (NF4)": codes sit at averages of
    adjacent standard-normal quantiles (k = 4 bits), the negative and positive
    halves are built separately -- 8 levels on one side and 9 on the other,
    sharing an exact zero -- and the set is renormalised into [-1, 1].  The
    displayed formula is lost; the reading used here (it reproduces all nine
    codes the worked example prints, to 4 dp):

      delta = ((1 - 1/(2*15)) + (1 - 1/(2*16))) / 2
      positive half: Q(p) for the 8 probabilities of linspace(delta, 1/2, 9)
                     without the final 1/2  (9 levels counting the zero);
      negative half: -Q(p) for the 7 of linspace(delta, 1/2, 8) without 1/2;
      add 0, sort, divide by Q(delta).
    """
    delta = 0.5 * ((1.0 - 1.0 / (2 * 15)) + (1.0 - 1.0 / (2 * 16)))
    pos_p = [delta - i * (delta - 0.5) / 8.0 for i in range(8)]
    neg_p = [delta - j * (delta - 0.5) / 7.0 for j in range(7)]
    pos = [ppf(p) for p in pos_p]
    neg = [-ppf(p) for p in neg_p]
    levels = np.array(sorted(neg + [0.0] + pos), dtype=np.float64)
    return levels / ppf(delta)


def nf4_codebook() -> tuple[np.ndarray, np.ndarray]:
    """(codes, midpoints): 16 fp32 codes ascending and 15 fp32 midpoints.

    Codes are the fp64 levels rounded to fp32.  Midpoint i is the exact
    average of fp32 codes i and i+1 (exact in fp64), rounded to nearest fp32.
    """
    codes = nf4_levels_fp64().astype(np.float32)
    c64 = codes.astype(np.float64)
    mids = ((c64[:-1] + c64[1:]) / 2.0).astype(np.float32)
    return codes, mids


# ---------------------------------------------------------------------------
# a2/a3.  Block absmax, nearest code, nibble packing.
# ---------------------------------------------------------------------------
def block_absmax(w_flat: np.ndarray, block: int = BLOCK) -> np.ndarray:
    """c_b = max_j |w_{b,j}| over consecutive blocks of the flattened tensor.

    "QLoRA, explained", "Blockwise absmax quantisation".  A final partial
    block is padded with zeros (zero padding cannot change a max of |w|).
    """
    w = np.asarray(w_flat, dtype=np.float32).reshape(-1)
    nblocks = -(-w.size // block)
    padded = np.zeros(nblocks * block, dtype=np.float32)
    padded[: w.size] = w
    return np.abs(padded.reshape(nblocks, block)).max(axis=1)


def nearest_code_index(x: np.ndarray, midpoints: np.ndarray) -> np.ndarray:
    """Index of the nearest code of fp32 x: the number of midpoints lying
    strictly below x.  A value equal to a midpoint goes to the lower code.

    "QLoRA, explained", "Blockwise absmax quantisation" (store the index of the
    nearest code).  Written as a plain per-element count over all midpoints.
    """
    x = np.asarray(x, dtype=np.float32)
    m = np.asarray(midpoints, dtype=np.float32)
    idx = np.zeros(x.shape, dtype=np.uint8)
    for mi in m:
        idx += (x > mi).astype(np.uint8)
    return idx


def normalise_blocks(w_flat: np.ndarray, absmax: np.ndarray,
                     block: int = BLOCK) -> np.ndarray:
    """x = w / c_b in fp32, correctly rounded (numpy fp32 division).

    Zero blocks (c_b = 0) give x = 0, whose nearest code is the exact zero.
    """
    w = np.asarray(w_flat, dtype=np.float32).reshape(-1)
    nblocks = absmax.size
    padded = np.zeros(nblocks * block, dtype=np.float32)
    padded[: w.size] = w
    padded = padded.reshape(nblocks, block)
    c = absmax.astype(np.float32).reshape(nblocks, 1)
    safe = np.where(c == 0, np.float32(1.0), c).astype(np.float32)
    x = (padded / safe).astype(np.float32)
    x[(c == 0).reshape(-1)] = np.float32(0.0)
    return x.reshape(-1)


def pack_nibbles(idx: np.ndarray) -> np.ndarray:
    """Two 4-bit indices per byte: element 2j in the low nibble, 2j+1 in the
    high nibble ("QLoRA, explained", "Minimal implementation"; the nibble
    order is not printed, low-first is the reading).  Odd length pads with
    the zero code's index 7."""
    i = np.asarray(idx, dtype=np.uint8).reshape(-1)
    if i.size % 2:
        i = np.concatenate([i, np.array([7], dtype=np.uint8)])
    lo = i[0::2] & 0x0F
    hi = i[1::2] & 0x0F
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray, count: int) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8).reshape(-1)
    out = np.empty(p.size * 2, dtype=np.uint8)
    out[0::2] = p & 0x0F
    out[1::2] = p >> 4
    return out[:count]


# ---------------------------------------------------------------------------
# a4.  Double quantisation of the scales: 8-bit floats, one fp32 constant per
# 256 scales.  "QLoRA, explained", "Double quantisation" and "The algorithm,
# step by step" (quantise c1 to FP8 in blocks of 256 with fp32 constants c2).
# The 8-bit float format is not named; the reading is OCP FP8 E4M3 (e4m3fn:
# bias 7, no infinities, largest finite 448), the constant is the group's
# largest scale divided by 448, and the code is the round-to-nearest-even
# E4M3 value of c_b / c2, saturated to 448.
# ---------------------------------------------------------------------------
def e4m3_value_table() -> np.ndarray:
    """Values of the 127 non-negative finite E4M3 codes 0x00..0x7E (fp64).

    Code c = eeee mmm: exponent field 0 is subnormal, m/8 * 2^-6; otherwise
    (1 + m/8) * 2^(e - 7).  0x7F is NaN and is never produced.
    """
    vals = np.empty(127, dtype=np.float64)
    for c in range(127):
        e, m = c >> 3, c & 7
        vals[c] = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_E4M3 = e4m3_value_table()


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Non-negative fp32 -> E4M3 code: the nearest representable value, ties to
    the even code, anything above 448 saturated to 448 (0x7E).  Enumerates all
    127 candidates for every element."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64).reshape(-1)
    if np.any(x < 0) or not np.all(np.isfinite(x)):
        raise ValueError("e4m3_encode takes finite non-negative values")
    out = np.empty(x.size, dtype=np.uint8)
    for i, v in enumerate(x):
        if v >= E4M3_MAX:
            out[i] = 0x7E
            continue
        d = np.abs(_E4M3 - v)
        best = np.flatnonzero(d == d.min())
        if best.size > 1:                      # a tie between two neighbours
            best = best[best % 2 == 0]
        out[i] = best[0]
    return out


def _encode_sorted(x: np.ndarray, table: np.ndarray, what: str) -> np.ndarray:
    """Nearest value of an ascending table of a float format's non-negative
    finite values (code i has value table[i]): a binary search
    (np.searchsorted) finds each element's two neighbours lo <= x <= hi; the
    nearer one wins, an exact tie takes the even code, and anything at or
    above the largest value takes the largest code (saturation)."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64).reshape(-1)
    if np.any(x < 0) or not np.all(np.isfinite(x)):
        raise ValueError(f"{what} takes finite non-negative values")
    top = table.size - 1
    hi = np.clip(np.searchsorted(table, x, side="left"), 1, top)
    lo = hi - 1
    d_lo = x - table[lo]
    d_hi = table[hi] - x
    even = np.where(lo % 2 == 0, lo, hi)
    code = np.where(d_lo < d_hi, lo, np.where(d_hi < d_lo, hi, even))
    return np.where(x >= table[top], top, code).astype(np.uint8)


def e4m3_encode_sorted(x: np.ndarray) -> np.ndarray:
    """The same encoding as e4m3_encode, written for whole arrays (the 127
    values ascend in code order; at or above 448 -> 0x7E)."""
    return _encode_sorted(x, _E4M3, "e4m3_encode_sorted")


def e4m3_decode(code: np.ndarray) -> np.ndarray:
    c = np.asarray(code, dtype=np.uint8).reshape(-1)
    if np.any(c == 0x7F) or np.any(c >= 0x80):
        raise ValueError("only non-negative finite E4M3 codes are produced")
    return _E4M3[c].astype(np.float32)


# The other 8-bit scale encodings ("Double quantisation" names only "8-bit
# floats"; "A toy run ..." measures what the choice costs): OCP FP8 E5M2
# (bias 15, two mantissa bits, largest finite 57344) and a linear unsigned
# 8-bit code (c2 = max / 255, code = rint(fp32(c_b / c2)), ties to even).
E5M2_MAX = 57344.0
U8_MAX = 255.0


def e5m2_value_table() -> np.ndarray:
    """Values of the 124 non-negative finite E5M2 codes 0x00..0x7B (fp64).

    Code c = eeeee mm: exponent field 0 is subnormal, m/4 * 2^-14; otherwise
    (1 + m/4) * 2^(e - 15).  0x7C is +inf and 0x7D..0x7F are NaN, never
    produced."""
    vals = np.empty(124, dtype=np.float64)
    for c in range(124):
        e, m = c >> 2, c & 3
        vals[c] = (m / 4.0) * 2.0 ** -14 if e == 0 else (1.0 + m / 4.0) * 2.0 ** (e - 15)
    return vals


_E5M2 = e5m2_value_table()


def e5m2_encode(x: np.ndarray) -> np.ndarray:
    """Non-negative fp32 -> E5M2 code, nearest with ties to the even code,
    at or above 57344 saturated to 0x7B."""
    return _encode_sorted(x, _E5M2, "e5m2_encode")


def e5m2_decode(code: np.ndarray) -> np.ndarray:
    c = np.asarray(code, dtype=np.uint8).reshape(-1)
    if np.any(c >= 0x7C):
        raise ValueError("only non-negative finite E5M2 codes are produced")
    return _E5M2[c].astype(np.float32)


def u8_encode(x: np.ndarray) -> np.ndarray:
    """Non-negative fp32 x (the ratio c_b / c2, at most about 255) -> the
    linear code rint(x), ties to even, clamped to 255."""
    x = np.asarray(x, dtype=np.float32).reshape(-1)
    if np.any(x < 0) or not np.all(np.isfinite(x)):
        raise ValueError("u8_encode takes finite non-negative values")
    return np.minimum(np.rint(x), np.float32(U8_MAX)).astype(np.uint8)


SCALE_CODES = {"e4m3": (E4M3_MAX, e4m3_encode_sorted),
               "e5m2": (E5M2_MAX, e5m2_encode),
               "u8": (U8_MAX, u8_encode)}


def decode_scale_codes(codes: np.ndarray, fmt: str = "e4m3") -> np.ndarray:
    """fp32 value of each 8-bit scale code (exact in every format)."""
    if fmt == "e4m3":
        return e4m3_decode(codes)
    if fmt == "e5m2":
        return e5m2_decode(codes)
    if fmt == "u8":
        return np.asarray(codes, dtype=np.uint8).astype(np.float32).reshape(-1)
    raise ValueError(fmt)


def double_quantize(absmax: np.ndarray, group: int = GROUP, fmt: str = "e4m3"
                    ) -> tuple[np.ndarray, np.ndarray]:
    """(scale_codes u8[nblocks], meta fp32[ngroups]).

    c2_g = fp32(max_{b in g} c_b / TOP); code_b = ENC(fp32(c_b / c2_g)), with
    TOP and ENC those of the 8-bit format (E4M3: 448 and round-to-nearest-even
    E4M3; E5M2: 57344 and E5M2; u8: 255 and rint).  An all-zero group has
    c2 = 0 and codes 0.  A final partial group is padded with zero scales,
    which cannot change its max.
    """
    top, encode = SCALE_CODES[fmt]
    c = np.asarray(absmax, dtype=np.float32).reshape(-1)
    nblocks = c.size
    ngroups = -(-nblocks // group)
    padded = np.zeros(ngroups * group, dtype=np.float32)
    padded[:nblocks] = c
    padded = padded.reshape(ngroups, group)
    meta = (padded.max(axis=1) / np.float32(top)).astype(np.float32)
    live = meta > 0
    safe = np.where(live, meta, np.float32(1.0)).astype(np.float32)
    ratio = (padded / safe.reshape(ngroups, 1)).astype(np.float32)
    codes = encode(ratio).reshape(ngroups, group)
    codes[~live] = 0
    return codes.reshape(-1)[:nblocks], meta


def dequantize_scales(scale_codes: np.ndarray, meta: np.ndarray,
                      group: int = GROUP, fmt: str = "e4m3") -> np.ndarray:
    """First step of dDQ ("The forward pass and gradients"): c~_b = fp32(
    decode(code_b) * c2_g), a single correctly rounded fp32 product."""
    codes = np.asarray(scale_codes, dtype=np.uint8).reshape(-1)
    g = np.arange(codes.size) // group
    return (decode_scale_codes(codes, fmt) * np.asarray(meta, dtype=np.float32)[g]).astype(np.float32)


# ---------------------------------------------------------------------------
# bf16 round-to-nearest-even from fp32 (the compute type fixed by
# "QLoRA, explained": weights are dequantised to bf16).
# ---------------------------------------------------------------------------
def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit pattern, round to nearest, ties to even.  Finite input
    only (the method never produces non-finite weights)."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    return ((b + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_float(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    return bf16_bits_to_float(bf16_bits(x))


# ---------------------------------------------------------------------------
# The whole storage step, "The algorithm, step by step" (split into blocks of
# 64, absmax, nearest NF4 code, FP8 scales in groups of 256).
# ---------------------------------------------------------------------------
class NonFiniteWeight(ValueError):
    pass


def quantize(W: np.ndarray) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """W (any shape, fp32, flattened in C order) -> (packed, scale_codes, meta).

    packed holds 32 bytes per block of 64 (a final partial block is padded
    with the zero code, index 7), scale_codes one byte per block, meta one
    fp32 per group of 256 blocks.
    """
    w = np.asarray(W, dtype=np.float32).reshape(-1)
    if not np.all(np.isfinite(w)):
        raise NonFiniteWeight("weights must be finite")
    _, mids = nf4_codebook()
    absmax = block_absmax(w)
    x = normalise_blocks(w, absmax)
    idx = nearest_code_index(x, mids)
    packed = pack_nibbles(idx)
    scale_codes, meta = double_quantize(absmax)
    return packed, scale_codes, meta


def dequantize_bits(packed: np.ndarray, scale_codes: np.ndarray,
                    meta: np.ndarray, numel: int) -> np.ndarray:
    """dDQ, "The forward pass and gradients": c~_b from the FP8 code and the
    fp32 constant, then w~ = bf16_RNE(fp32(q[idx] * c~_b)).  Returns bf16 bits
    for the first numel elements in flattened order."""
    codes, _ = nf4_codebook()
    ctilde = dequantize_scales(scale_codes, meta)
    nblocks = ctilde.size
    idx = unpack_nibbles(packed, nblocks * BLOCK).reshape(nblocks, BLOCK)
    prod = (codes[idx] * ctilde.reshape(nblocks, 1)).astype(np.float32)
    return bf16_bits(prod).reshape(-1)[:numel]


def dequantize(packed, scale_codes, meta, rows: int, cols: int) -> np.ndarray:
    """bf16 W~ as fp32 values, shape (rows, cols)."""
    bits = dequantize_bits(packed, scale_codes, meta, rows * cols)
    return bf16_bits_to_float(bits).reshape(rows, cols)


def single_quant_roundtrip(w: np.ndarray, codes: np.ndarray, block: int,
                           nearest=None) -> np.ndarray:
    """Blockwise absmax quantise-dequantise with fp32 scales (no double
    quantisation, no bf16 rounding): the toy of "A toy run ..." for any
    codebook and blocksize.  Nearest code by brute-force argmin."""
    w = np.asarray(w, dtype=np.float32).reshape(-1)
    absmax = block_absmax(w, block)
    x = normalise_blocks(w, absmax, block).reshape(-1, block)
    idx = brute_nearest_index(x, codes) if nearest is None else nearest(x)
    rec = (np.asarray(codes, dtype=np.float32)[idx] * absmax.reshape(-1, 1)).astype(np.float32)
    return rec.reshape(-1)[: w.size]


def brute_nearest_index(x: np.ndarray, codes: np.ndarray) -> np.ndarray:
    """argmin_i |x - q_i| evaluated in fp64, ties to the lower index."""
    x64 = np.asarray(x, dtype=np.float64)[..., None]
    d = np.abs(x64 - np.asarray(codes, dtype=np.float64))
    return np.argmin(d, axis=-1).astype(np.uint8)   # argmin keeps the first


def fp4_e2m1_codebook() -> np.ndarray:
    """E2M1 FP4 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6} with sign, scaled to
    [-1, 1] ("A toy run ...").  +0 and -0 coincide, leaving 15 values."""
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64) / 6.0
    return np.unique(np.concatenate([-mags, mags])).astype(np.float32)


def int4_codebook() -> np.ndarray:
    """Symmetric 15-level integer grid {-7..7}/7 ("A toy run ...")."""
    return (np.arange(-7, 8, dtype=np.float64) / 7.0).astype(np.float32)


# ---------------------------------------------------------------------------
# Storage cost, "Double quantisation" and "Compute and memory cost".
# ---------------------------------------------------------------------------
def storage_bits_per_param(block: int = BLOCK, group: int = GROUP,
                           double_quant: bool = True) -> float:
    """4 bits of index + the scale's share: 8/B + 32/(B*group) with double
    quantisation, 32/B without."""
    if double_quant:
        return 4.0 + 8.0 / block + 32.0 / (block * group)
    return 4.0 + 32.0 / block


def quantized_nbytes(numel: int) -> tuple[int, int, int]:
    """(packed, scale-code, meta) byte counts of the stored tensor."""
    nblocks = -(-numel // BLOCK)
    ngroups = -(-nblocks // GROUP)
    return nblocks * BLOCK // 2, nblocks, 4 * ngroups


# ---------------------------------------------------------------------------
# a6-a8.  The adapted linear layer, "The forward pass and gradients" and "The
# algorithm, step by step":  Y = X W~^T + gamma X A^T B^T;  dX = dY (W~ +
# gamma B A);  dA = gamma B^T G, dB = gamma G A^T with G = dY^T X the weight
# gradient (never formed, and no gradient for the stored NF4 weights).
# gamma = alpha / r, the usual LoRA scale.  Everything in fp64 from the
# bf16-exact inputs and the bf16 W~.
# ---------------------------------------------------------------------------
def linear_forward(X, Wt, A, B, gamma):
    """X [M,K], Wt = W~ [N,K], A [r,K], B [N,r] -> (Y [M,N], T = X A^T [M,r])."""
    X = np.asarray(X, np.float64)
    T = X @ np.asarray(A, np.float64).T
    Y = X @ np.asarray(Wt, np.float64).T + gamma * (T @ np.asarray(B, np.float64).T)
    return Y, T


def linear_backward(dY, X, Wt, A, B, gamma):
    """-> (dX [M,K], dA [r,K], dB [N,r], U = dY B [M,r])."""
    dY = np.asarray(dY, np.float64)
    X = np.asarray(X, np.float64)
    A = np.asarray(A, np.float64)
    B = np.asarray(B, np.float64)
    U = dY @ B
    dX = dY @ np.asarray(Wt, np.float64) + gamma * (U @ A)
    dA = gamma * (U.T @ X)
    dB = gamma * (dY.T @ (X @ A.T))
    return dX, dA, dB, U


# ---------------------------------------------------------------------------
# Merge for export.  "QLoRA, explained", "The forward pass and gradients": the
# fine-tuned model is W~ + gamma B A (the adapter on the quantised base); the
# same page's "Failure modes" ("Quality loss at merge time") names
# dequantising W~ to bf16, adding the adapter and keeping the result in bf16
# as the merge that preserves it.  "QLoRA" (finetunellm.com), "What it costs
# you": a 4-bit deployment then quantises the merged bf16 weight again
# (quantize() applied to its values).  Reading: the sum is exact (fp64 here)
# and rounded to bf16 once, to nearest with ties to even.
# ---------------------------------------------------------------------------
BF16_MIN_SUBNORMAL_EXP = -133          # 2**-133, the smallest positive bf16


def bf16_rne_f64(x: np.ndarray) -> np.ndarray:
    """bf16 bits of fp64 values rounded to nearest, ties to even, directly
    from fp64 (no intermediate fp32 rounding).  bf16 keeps 8 significant
    bits, so the spacing at x = m 2^e (0.5 <= |m| < 1) is 2^(e-8), never finer
    than the smallest subnormal; values that round to 2^128 or beyond become
    infinities."""
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    step = np.maximum(e - 8, BF16_MIN_SUBNORMAL_EXP)
    with np.errstate(invalid="ignore", over="ignore"):
        y = np.ldexp(np.rint(np.ldexp(x, -step)), step)     # rint: ties to even
        y = np.where(np.abs(y) >= 2.0 ** 128, np.copysign(np.inf, x), y)
        bits = (y.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    return np.where(np.isnan(x), np.uint16(0x7FC0), bits)


def merge(packed, scale_codes, meta, rows: int, cols: int, A, B, gamma):
    """-> (exact [rows, cols] fp64 value of W~ + gamma B A, its bf16 bits).
    gamma is taken at fp32, the precision the library receives it in."""
    Wt = dequantize(packed, scale_codes, meta, rows, cols).astype(np.float64)
    g = float(np.float32(gamma))
    exact = Wt + g * (np.asarray(B, np.float64) @ np.asarray(A, np.float64))
    return exact, bf16_rne_f64(exact)


# ---------------------------------------------------------------------------
# Format variants.  "QLoRA, explained", "A toy run: how much does NF4 lose
# ...": the same blockwise absmax scheme with other 4-bit codebooks (E2M1
# FP4, a symmetric 15-level INT4 grid) and other blocksizes (16 to 4096), and
# "Double quantisation" as an option (without it every block keeps its fp32
# absmax).  The steps are those of quantize() with the codebook, blocksize
# and scale storage as parameters; the nearest code is again the number of
# midpoints strictly below x (midpoints = exact averages of adjacent fp32
# codes rounded to fp32), a zero block and the padding of a final partial
# block take the index nearest to 0.
# ---------------------------------------------------------------------------
SCALES_FP32 = "fp32"
SCALES_E4M3 = "e4m3"
SCALES_E5M2 = "e5m2"
SCALES_U8 = "u8"


def midpoints_of(codes: np.ndarray) -> np.ndarray:
    c64 = np.asarray(codes, dtype=np.float32).astype(np.float64)
    return ((c64[:-1] + c64[1:]) / 2.0).astype(np.float32)


def quantize_fmt(W: np.ndarray, codes: np.ndarray, block: int, scales: str):
    """W (flattened, fp32) -> (packed, scales, meta).  scales 'fp32': one fp32
    absmax per block and meta None; 'e4m3' (as quantize()), 'e5m2' or 'u8':
    8-bit codes and fp32 constants per 256 blocks (double_quantize)."""
    w = np.asarray(W, dtype=np.float32).reshape(-1)
    if not np.all(np.isfinite(w)):
        raise NonFiniteWeight("weights must be finite")
    mids = midpoints_of(codes)
    absmax = block_absmax(w, block)
    idx = nearest_code_index(normalise_blocks(w, absmax, block), mids)
    packed = pack_nibbles(idx)
    if scales == SCALES_FP32:
        return packed, absmax.astype(np.float32), None
    sc, meta = double_quantize(absmax, fmt=scales)
    return packed, sc, meta


def dequantize_fmt_bits(packed, scale_data, meta, numel: int, codes: np.ndarray, block: int,
                        scales: str) -> np.ndarray:
    """bf16 bits of w~ = bf16_rne(fp32(q[idx] * c~_b)), c~_b the fp32 absmax
    ('fp32') or fp32(decode(code) * c2) (the 8-bit formats)."""
    c = (np.asarray(scale_data, dtype=np.float32) if scales == SCALES_FP32
         else dequantize_scales(scale_data, meta, fmt=scales))
    nblocks = c.size
    idx = unpack_nibbles(packed, nblocks * block).reshape(nblocks, block)
    prod = (np.asarray(codes, dtype=np.float32)[idx] * c.reshape(nblocks, 1)).astype(np.float32)
    return bf16_bits(prod).reshape(-1)[:numel]


def format_nbytes(numel: int, block: int, scales: str) -> tuple[int, int, int]:
    """(packed, scale, meta) byte counts of a stored tensor in a variant format."""
    nblocks = -(-numel // block)
    if scales == SCALES_FP32:
        return nblocks * block // 2, 4 * nblocks, 0
    return nblocks * block // 2, nblocks, 4 * (-(-nblocks // GROUP))


# ---------------------------------------------------------------------------
# Layer chaining with gradient checkpointing.  "QLoRA, explained", "The
# algorithm, step by step" (gradient checkpointing enabled) and "Compute and
# memory cost" (checkpointing is effectively mandatory; a recomputed forward
# dequantises every block a third time per step).  The chained block is the
# MLP of the Llama-shaped workloads, y = down(silu(gate(x)) * up(x)), every
# linear an adapted NF4 layer; the pages print no activation, so SwiGLU is
# the reading taken from those shapes.  With checkpointing only x is kept
# from the forward and the backward recomputes gate(x), up(x) and h.
# ---------------------------------------------------------------------------
def silu(z):
    z = np.asarray(z, np.float64)
    return z / (1.0 + np.exp(-z))


def silu_grad(z):
    """d silu / dz = s (1 + z (1 - s)), s the logistic sigmoid."""
    z = np.asarray(z, np.float64)
    s = 1.0 / (1.0 + np.exp(-z))
    return s * (1.0 + z * (1.0 - s))


def _bf16_of(x):
    """fp64 -> the nearest bf16 value (ties to even), as fp64."""
    return bf16_bits_to_float(bf16_rne_f64(x)).astype(np.float64)


def mlp_forward(X, layers, gamma, bf16_activations: bool = False):
    """layers = {'gate': (Wt, A, B), 'up': ..., 'down': ...} with Wt = W~
    [out, in].  -> (Y, saved) where saved = (G, U, H) are the activations a
    non-checkpointed backward keeps.

    bf16_activations: the activations that pass between the block's steps
    (the outputs of gate, up and down, and h) are rounded to bf16, the compute
    type the pages fix ("Failure modes", "Loss spikes and NaNs": use bf16
    compute; "Minimal implementation": bnb_4bit_compute_dtype bf16); each
    step itself stays exact in fp64."""
    rnd = _bf16_of if bf16_activations else (lambda a: a)
    G, _ = linear_forward(X, *layers["gate"], gamma)
    U, _ = linear_forward(X, *layers["up"], gamma)
    G, U = rnd(G), rnd(U)
    H = rnd(silu(G) * U)
    Y, _ = linear_forward(H, *layers["down"], gamma)
    return rnd(Y), (G, U, H)


def mlp_backward(dY, X, layers, gamma, saved=None, bf16_activations: bool = False):
    """-> (dX, {name: (dA, dB)}).  saved = None recomputes the forward from X
    (gradient checkpointing: the third dequantisation of gate and up).
    bf16_activations as mlp_forward, for dH, dG, dU and each linear's input
    gradient (the two parts of dX rounded, then their sum)."""
    rnd = _bf16_of if bf16_activations else (lambda a: a)
    if saved is None:
        _, saved = mlp_forward(X, layers, gamma, bf16_activations)
    G, U, H = saved
    Wd, Ad, Bd = layers["down"]
    dH, dAd, dBd, _ = linear_backward(dY, H, Wd, Ad, Bd, gamma)
    dH = rnd(dH)
    dG = rnd(dH * U * silu_grad(G))
    dU = rnd(dH * silu(G))
    Wg, Ag, Bg = layers["gate"]
    Wu, Au, Bu = layers["up"]
    dXg, dAg, dBg, _ = linear_backward(dG, X, Wg, Ag, Bg, gamma)
    dXu, dAu, dBu, _ = linear_backward(dU, X, Wu, Au, Bu, gamma)
    return rnd(rnd(dXg) + rnd(dXu)), {"gate": (dAg, dBg), "up": (dAu, dBu), "down": (dAd, dBd)}


# ---------------------------------------------------------------------------
# Optimiser state for the adapter.  "QLoRA, explained", "The algorithm, step
# by step" (AdamW over A and B only, 32-bit or 8-bit state) and "Hyperparameters
# that matter" (the 8-bit variant quantises Adam's moments blockwise).  The
# pages give no 8-bit format; the reading reuses the blockwise absmax scheme:
# blocks of `block` consecutive state entries, an fp32 absmax c per block, the
# first moment as a symmetric linear 8-bit code q = rint(fp32(m / c) * 127) in
# [-127, 127], the second through its square root, q = rint(fp32(sqrt(v) / c)
# * 255) in [0, 255] (the quotient rounded to fp32, then the product, ties to
# even); decoding is fp32(q * fp32(c / 127)) (or / 255,
# then squared).  A linear code of v itself flushes every v below 1/510 of its
# block's largest to zero while m is still non-zero, and the step m / (0 + eps)
# then diverges; the square root keeps v's resolution on the scale of m's.
# The update itself is AdamW in fp32 on the decoded state, after which the
# state is re-encoded.
# ---------------------------------------------------------------------------
def adamw_step(p, g, m, v, t: int, lr: float, beta1: float, beta2: float, eps: float,
               weight_decay: float):
    """One AdamW step in fp32 (decoupled weight decay, bias-corrected moments).
    Returns new (p, m, v); t counts from 1."""
    f = np.float32
    p, g, m, v = (np.asarray(a, np.float32) for a in (p, g, m, v))
    p = (p * f(1.0 - lr * weight_decay)).astype(np.float32)
    m = (f(beta1) * m + f(1.0 - beta1) * g).astype(np.float32)
    v = (f(beta2) * v + f(1.0 - beta2) * g * g).astype(np.float32)
    mhat = m / f(1.0 - beta1 ** t)
    vhat = v / f(1.0 - beta2 ** t)
    p = (p - f(lr) * mhat / (np.sqrt(vhat) + f(eps))).astype(np.float32)
    return p, m, v


def encode_state8(x: np.ndarray, signed: bool, block: int):
    """(codes, absmax): codes int8 (signed) or uint8, absmax fp32 per block."""
    x = np.asarray(x, np.float32).reshape(-1)
    c = block_absmax(x, block)
    levels = np.float32(127.0 if signed else 255.0)
    nb = c.size
    pad = np.zeros(nb * block, np.float32)
    pad[: x.size] = x
    safe = np.where(c == 0, np.float32(1.0), c).astype(np.float32).reshape(nb, 1)
    q = np.rint((pad.reshape(nb, block) / safe).astype(np.float32) * levels)
    q[(c == 0)] = 0
    q = q.reshape(-1)[: x.size]
    return (q.astype(np.int8) if signed else q.astype(np.uint8)), c


def decode_state8(codes: np.ndarray, absmax: np.ndarray, signed: bool, block: int):
    levels = np.float32(127.0 if signed else 255.0)
    q = np.asarray(codes).astype(np.float32).reshape(-1)
    step = (np.asarray(absmax, np.float32) / levels).astype(np.float32)
    return (q * step[np.arange(q.size) // block]).astype(np.float32)


def adamw8_step(p, g, m_state, v_state, t: int, lr: float, beta1: float, beta2: float,
                eps: float, weight_decay: float, block: int = BLOCK):
    """AdamW with 8-bit blockwise state: m_state = (int8 codes, absmax) of m,
    v_state = (uint8 codes, absmax) of sqrt(v).  Returns (p, m_state, v_state)."""
    m = decode_state8(*m_state, True, block).reshape(np.shape(p))
    u = decode_state8(*v_state, False, block).reshape(np.shape(p))
    v = (u * u).astype(np.float32)
    p, m, v = adamw_step(p, g, m, v, t, lr, beta1, beta2, eps, weight_decay)
    return (p, encode_state8(m, True, block),
            encode_state8(np.sqrt(v).astype(np.float32), False, block))
