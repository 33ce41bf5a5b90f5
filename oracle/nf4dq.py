"""NF4 blockwise quantization, Double Quantization and doubleDequant (oracle).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: "QLoRA: Efficient Finetuning of Quantized LLMs"
(aiingo.vercel.app/paper/paper-2305-14314):
  §2 "Block-wise k-bit Quantization" (Eqs. 1-2 and the blocking paragraph),
  §3 "4-bit NormalFloat Quantization" (Eq. 4) and Appendix E (exact NF4 values),
  §3 "Double Quantization",
  §3 "QLoRA" (Eq. 6: doubleDequant; block sizes 64 for W and 256 for c2; FP8
  for c2; NF4 for W; BFloat16 compute type).

Readings of points the paper leaves open (each is a decision, listed with its
reason in the design notes of the repository):
  * the block constant stored for a block is its absmax, a positive
    multiplier: dequant is code value x constant (Eq. 2 read as the inverse of
    Eq. 1);
  * blocks are consecutive runs of the row-major flattened tensor; a final
    partial block uses only its real elements;
  * the nearest NF4 level is chosen with ties going to the lower index, the
    comparison against the exact midpoints of adjacent levels being exact;
  * x = w / absmax is the IEEE round-to-nearest-even float32 quotient;
  * an all-zero block (absmax 0) encodes every element as the exact-zero code 7;
  * the Double-Quantization mean is one float32 per tensor, the correctly
    rounded float64 mean of the float32 constants rounded to float32;
  * the "8-bit float" is OCP E4M3 (max 448, no infinities), the second-level
    constant of each 256-block is absmax(c2 - mean)/448 so that the block's
    extreme maps to +/-448, codes are round-to-nearest-even with saturation;
  * doubleDequant rounds twice: c2_hat = fma_f32(E4M3(code8), c1, mean), then
    W_hat = bf16_rne(f32(NF4[code] * c2_hat)).
  * nibble order: element 2i sits in the low nibble of byte i, element 2i+1 in
    the high nibble; an odd element count leaves the last high nibble 0.
"""

from __future__ import annotations

import math

import numpy as np

# --------------------------------------------------------------------------
# The NF4 data type: the 16 exact values printed in Appendix E of the paper.
# All sixteen are exactly representable in float32.
# --------------------------------------------------------------------------
NF4_VALUES = np.array(
    [
        -1.0,
        -0.6961928009986877,
        -0.5250730514526367,
        -0.39491748809814453,
        -0.28444138169288635,
        -0.18477343022823334,
        -0.09105003625154495,
        0.0,
        0.07958029955625534,
        0.16093020141124725,
        0.24611230194568634,
        0.33791524171829224,
        0.44070982933044434,
        0.5626170039176941,
        0.7229568362236023,
        1.0,
    ],
    dtype=np.float32,
)

NF4_ZERO_CODE = 7          # index of the exact zero (§3: "a discrete zeropoint of 0")
W_BLOCK = 64               # block size of W (§3 "QLoRA": "blocksize of 64 for W")
C2_BLOCK = 256             # block size of c2 (§3 "Double Quantization": "blocksize of 256")
E4M3_MAX = 448.0           # largest finite OCP E4M3 value

# Decision thresholds between adjacent levels, in float64.  The sum of two
# float32 values is exact in float64 and halving it is exact, so these are the
# exact midpoints.
NF4_MIDPOINTS = (NF4_VALUES[:-1].astype(np.float64) + NF4_VALUES[1:].astype(np.float64)) / 2.0

# --------------------------------------------------------------------------
# The 4-bit float FP4 (E2M1) that the paper compares NF4 against (§4,
# Tables 2-4: "Float4 (E2M1)").  Its value set {0, 0.5, 1, 1.5, 2, 3, 4, 6}
# and their negatives, normalised by the largest value 6 so that a block's
# absmax maps to +-1 as for NF4, rounded to float32, in ascending order.  The
# format has a positive and a negative zero; both codes hold +0 here, so code
# 7 is the exact zero of either table.  (Its encoding: sign, a 2-bit exponent
# with bias 1, a 1-bit mantissa; exponent 0 is subnormal: 0.5 * m.)
# --------------------------------------------------------------------------
def e2m1_value(bits: int) -> float:
    """Value of a 4-bit E2M1 code (sign bit 3, exponent bits 2-1, mantissa bit 0)."""
    sign = -1.0 if bits & 8 else 1.0
    e, m = (bits >> 1) & 3, bits & 1
    mag = 0.5 * m if e == 0 else (1.0 + 0.5 * m) * 2.0 ** (e - 1)
    return sign * mag


def _fp4_table() -> np.ndarray:
    vals = sorted({e2m1_value(b) for b in range(16)})           # 15 distinct values, one zero
    vals = vals[:7] + [0.0] + vals[7:]                          # both zero codes
    return np.array([np.float32(v) / np.float32(6.0) for v in vals], dtype=np.float32)


FP4_VALUES = _fp4_table()
TABLES = {"nf4": NF4_VALUES, "fp4": FP4_VALUES}


def midpoints(levels: np.ndarray) -> np.ndarray:
    levels = np.asarray(levels, dtype=np.float32).astype(np.float64)
    return (levels[:-1] + levels[1:]) / 2.0


# --------------------------------------------------------------------------
# Small exact-rounding helpers.
# --------------------------------------------------------------------------
def f32(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float32)


def bf16_rne_bits(x32: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even).

    Returns the 16-bit patterns (uint16).  Finite inputs only: bfloat16 keeps
    the top 16 bits of the float32 pattern, and the discarded low half is
    rounded by adding 0x7FFF plus the lowest kept bit.
    """
    x32 = np.ascontiguousarray(x32, dtype=np.float32)
    if not np.all(np.isfinite(x32)):
        raise ValueError("bf16_rne_bits: non-finite input")
    u = x32.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = u + np.uint64(0x7FFF) + lsb
    return (u >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _fp32_neighbour(r: np.ndarray, towards_up: np.ndarray) -> np.ndarray:
    up = np.nextafter(r, np.float32(np.inf), dtype=np.float32)
    dn = np.nextafter(r, np.float32(-np.inf), dtype=np.float32)
    return np.where(towards_up, up, dn)


def fma_f32(a, b, c) -> np.ndarray:
    """float32 fused multiply-add a*b + c with a single round-to-nearest-even.

    The product of two float32 values has at most 48 significant bits and is
    exact in float64.  The float64 sum s = p + c is then exact up to the error
    term e recovered by Knuth's TwoSum (s + e == p + c exactly).  Rounding s to
    float32 gives the correctly rounded result unless s lies exactly on the
    midpoint of two float32 neighbours while e != 0 (a double-rounding tie); in
    that case the true value lies on the side of e and that neighbour is taken.
    """
    a = f32(a).astype(np.float64)
    b = f32(b).astype(np.float64)
    c = f32(c).astype(np.float64)
    p = a * b                                   # exact
    s = p + c
    bb = s - p
    e = (p - (s - bb)) + (c - bb)               # TwoSum: s + e == p + c exactly
    r = s.astype(np.float32)
    r64 = r.astype(np.float64)
    # Only a tie in the float32 rounding of s can have gone the wrong way.
    other = _fp32_neighbour(r, s > r64)
    mid = (r64 + other.astype(np.float64)) / 2.0  # exact in float64
    tie = (s != r64) & (s == mid) & (e != 0)
    if np.any(tie):
        up_true = e > 0
        lo = np.minimum(r, other)
        hi = np.maximum(r, other)
        r = np.where(tie, np.where(up_true, hi, lo), r).astype(np.float32)
    return r


# --------------------------------------------------------------------------
# OCP E4M3 ("fn": no infinities, max 448) codec.
# --------------------------------------------------------------------------
def e4m3_decode(codes) -> np.ndarray:
    """Value of each 8-bit E4M3 code as float32 (0x7F/0xFF are NaN).

    Layout: sign bit 7, exponent bits 6..3 (bias 7), mantissa bits 2..0.
    Exponent 0 is subnormal: m/8 * 2^-6.
    """
    codes = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(codes & 0x80, -1.0, 1.0)
    e = (codes >> 3) & 0xF
    m = codes & 0x7
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = sign * mag
    val = np.where((codes & 0x7F) == 0x7F, np.nan, val)
    return val.astype(np.float32)


def _e4m3_magnitude_table():
    codes = np.arange(0x7F, dtype=np.uint8)      # 0x00..0x7E: all finite magnitudes
    return e4m3_decode(codes).astype(np.float64)  # increasing in the code


_E4M3_MAGS = _e4m3_magnitude_table()


def e4m3_encode_rne_satfinite(x) -> np.ndarray:
    """Encode float32 values as E4M3: round to nearest, ties to even, saturate.

    Brute force over the 127 finite magnitudes: the nearest magnitude wins; on
    an exact tie the code with an even mantissa (even code) wins; magnitudes
    above 448 saturate to 448.  The sign bit is copied from the input (so -0.0
    encodes to 0x80).  Finite inputs only.
    """
    x = f32(x)
    if not np.all(np.isfinite(x)):
        raise ValueError("e4m3 encode: non-finite input")
    mag = np.abs(x.astype(np.float64))
    sat = mag >= E4M3_MAX
    hi = np.searchsorted(_E4M3_MAGS, mag, side="left")          # first table value >= mag
    hi = np.clip(hi, 0, len(_E4M3_MAGS) - 1)
    lo = np.clip(hi - 1, 0, len(_E4M3_MAGS) - 1)
    d_hi = np.abs(_E4M3_MAGS[hi] - mag)
    d_lo = np.abs(mag - _E4M3_MAGS[lo])
    pick = np.where(d_lo < d_hi, lo, hi)
    tie = (d_lo == d_hi) & (lo != hi)
    pick = np.where(tie, np.where(lo % 2 == 0, lo, hi), pick)
    pick = np.where(sat, 0x7E, pick)
    sign = np.signbit(x).astype(np.int64) << 7
    return (pick.astype(np.int64) | sign).astype(np.uint8)


# --------------------------------------------------------------------------
# First-level quantization: NF4 with absmax blocks of 64.
# --------------------------------------------------------------------------
def nf4_code(x32, levels: np.ndarray = NF4_VALUES) -> np.ndarray:
    """Nearest level of a 16-level table (NF4 by default) for normalised inputs x in [-1, 1].

    code = number of exact midpoints that x lies strictly above, so an input
    exactly on a midpoint takes the lower level.
    """
    mids = NF4_MIDPOINTS if levels is NF4_VALUES else midpoints(levels)
    x = f32(x32).astype(np.float64)
    flat = x.reshape(-1)
    out = np.empty(flat.size, dtype=np.uint8)
    step = 1 << 20                      # bounded temporaries only; no effect on the result
    for s in range(0, flat.size, step):
        out[s:s + step] = (flat[s:s + step, None] > mids).sum(axis=-1)
    return out.reshape(x.shape)


def _blocks(n: int, bs: int):
    """(start, stop) of consecutive blocks of size bs over n elements."""
    return [(s, min(s + bs, n)) for s in range(0, n, bs)]


def block_absmax(flat32: np.ndarray, bs: int) -> np.ndarray:
    n = flat32.size
    nfull = n // bs
    out = np.empty((n + bs - 1) // bs, dtype=np.float32)
    if nfull:
        out[:nfull] = np.abs(flat32[: nfull * bs].reshape(nfull, bs)).max(axis=1)
    if n % bs:
        out[nfull] = np.abs(flat32[nfull * bs:]).max()
    return out


def quantize_nf4(w, levels: np.ndarray = NF4_VALUES) -> tuple[np.ndarray, np.ndarray]:
    """NF4-quantize (or, with ``levels``, quantize to another 16-level table) a
    tensor in absmax blocks of 64 (§2 blocking, §3 NF4).

    w: any float array (float32 or bfloat16 values widened to float32); it is
    flattened row-major.  Returns (codes uint8 [numel], c2 float32 [nblocks]).
    """
    flat = f32(w).reshape(-1)
    if not np.all(np.isfinite(flat)):
        raise ValueError("quantize_nf4: non-finite weight")
    c2 = block_absmax(flat, W_BLOCK)
    scale = np.repeat(c2, W_BLOCK)[: flat.size]
    with np.errstate(invalid="ignore", divide="ignore"):
        x = (flat / scale).astype(np.float32)      # IEEE float32 quotient
    codes = nf4_code(np.where(scale == 0, np.float32(0), x), levels)
    codes = np.where(scale == 0, NF4_ZERO_CODE, codes).astype(np.uint8)
    return codes, c2


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Two 4-bit codes per byte: element 2i low nibble, element 2i+1 high nibble."""
    codes = np.asarray(codes, dtype=np.uint8).reshape(-1)
    if codes.size % 2:
        codes = np.concatenate([codes, np.zeros(1, np.uint8)])
    return (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray, numel: int) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8).reshape(-1)
    out = np.empty(packed.size * 2, dtype=np.uint8)
    out[0::2] = packed & 0xF
    out[1::2] = packed >> 4
    return out[:numel]


# --------------------------------------------------------------------------
# Double Quantization of the first-level constants c2 (§3 "Double Quantization").
# --------------------------------------------------------------------------
def dq_mean(c2) -> np.float32:
    """The mean subtracted from c2 before its 8-bit quantization.

    Correctly rounded float64 sum of the float32 constants (math.fsum), divided
    by their count in float64, rounded to float32.
    """
    c2 = f32(c2).reshape(-1)
    if c2.size == 0:
        return np.float32(0.0)
    return np.float32(math.fsum(c2.astype(np.float64).tolist()) / c2.size)


def double_quantize(c2, mu=None):
    """Quantize the constants c2 to E4M3 codes in blocks of 256.

    For each block: d = f32(c2 - mu); A = max|d|; c1 = f32(A / 448);
    code8 = E4M3_rne_satfinite(f32(d / c1)), or code 0 for every element if
    c1 == 0.  Returns (code8 uint8 [n], c1 float32 [ceil(n/256)], mu float32).
    ``mu`` may be given (to check codes given another implementation's mean).
    """
    c2 = f32(c2).reshape(-1)
    if mu is None:
        mu = dq_mean(c2)
    mu = np.float32(mu)
    d = (c2 - mu).astype(np.float32)
    c1 = np.empty((c2.size + C2_BLOCK - 1) // C2_BLOCK, dtype=np.float32)
    code8 = np.zeros(c2.size, dtype=np.uint8)
    for bi, (s, e) in enumerate(_blocks(c2.size, C2_BLOCK)):
        a = np.abs(d[s:e]).max()
        c1[bi] = np.float32(a) / np.float32(E4M3_MAX)
        if c1[bi] == 0:
            code8[s:e] = 0
        else:
            q = (d[s:e] / c1[bi]).astype(np.float32)
            code8[s:e] = e4m3_encode_rne_satfinite(q)
    return code8, c1, mu


def dequant_c2(code8, c1, mu) -> np.ndarray:
    """Inner dequant of Eq. 6: c2_hat = fma_f32(E4M3(code8), c1[block], mu)."""
    code8 = np.asarray(code8, dtype=np.uint8).reshape(-1)
    c1 = f32(c1).reshape(-1)
    c1_per = np.repeat(c1, C2_BLOCK)[: code8.size]
    return fma_f32(e4m3_decode(code8), c1_per, np.float32(mu))


def double_dequant_bits(codes, code8, c1, mu, shape, levels: np.ndarray = NF4_VALUES) -> np.ndarray:
    """doubleDequant (Eq. 6) to bfloat16, returned as uint16 bit patterns.

    W_hat = bf16_rne(f32(NF4[code] * c2_hat[block])) with c2_hat from
    ``dequant_c2``.  ``codes`` are unpacked (one per element).
    """
    codes = np.asarray(codes, dtype=np.uint8).reshape(-1)
    c2_hat = dequant_c2(code8, c1, mu)
    scale = np.repeat(c2_hat, W_BLOCK)[: codes.size]
    prod = (np.asarray(levels, np.float32)[codes] * scale).astype(np.float32)
    return bf16_rne_bits(prod).reshape(shape)


def quantize_nf4_dq(w, levels: np.ndarray = NF4_VALUES):
    """The full quantizer of the QLoRA storage format.

    Returns a dict with the packed codes (uint8 [ceil(numel/2)]), the E4M3
    codes of c2 (uint8 [nblk64]), c1 (float32 [ceil(nblk64/256)]), the mean mu
    (float32), plus the unpacked codes and the float32 c2 for checking.
    """
    w = np.asarray(w)
    codes, c2 = quantize_nf4(w, levels)
    code8, c1, mu = double_quantize(c2)
    return {
        "shape": tuple(w.shape),
        "codes": codes,
        "packed": pack_nibbles(codes),
        "c2": c2,
        "c2_fp8": code8,
        "c1": c1,
        "mu": mu,
        "levels": np.asarray(levels, np.float32),
    }


def dequantize(q) -> np.ndarray:
    """doubleDequant of a ``quantize_nf4_dq`` result, as float32 values of bf16."""
    bits = double_dequant_bits(q["codes"], q["c2_fp8"], q["c1"], q["mu"], q["shape"], q.get("levels", NF4_VALUES))
    return bf16_bits_to_f32(bits)


def dequantize_rows(w, rows, levels: np.ndarray = NF4_VALUES) -> np.ndarray:
    """doubleDequant of selected rows of a 2-D weight, for sampled checks.

    The same steps as ``quantize_nf4_dq`` + ``dequantize``: every block's c2
    (the mean needs all of them), then the second-level constants of the
    256-groups holding the selected rows' blocks, then those rows' codes.
    Requires k_in % 64 == 0 (blocks do not straddle rows).
    """
    w = f32(w)
    n_out, k_in = w.shape
    if k_in % W_BLOCK:
        raise ValueError("dequantize_rows: k_in must be a multiple of 64")
    c2 = block_absmax(w.reshape(-1), W_BLOCK)
    mu = dq_mean(c2)
    bpr = k_in // W_BLOCK
    out = np.empty((len(rows), k_in), np.float32)
    for i, row in enumerate(rows):
        b0, b1 = row * bpr, (row + 1) * bpr
        g0, g1 = b0 // C2_BLOCK, (b1 - 1) // C2_BLOCK + 1
        seg = c2[g0 * C2_BLOCK: min(c2.size, g1 * C2_BLOCK)]
        code8, c1, _ = double_quantize(seg, mu)
        c2_hat = dequant_c2(code8, c1, mu)[b0 - g0 * C2_BLOCK: b1 - g0 * C2_BLOCK]
        codes, c2_row = quantize_nf4(w[row], levels)
        assert np.array_equal(c2_row, c2[b0:b1])
        prod = (np.asarray(levels, np.float32)[codes] * np.repeat(c2_hat, W_BLOCK)).astype(np.float32)
        out[i] = bf16_bits_to_f32(bf16_rne_bits(prod))
    return out


def dequantize_cols(w, cols, levels: np.ndarray = NF4_VALUES) -> np.ndarray:
    """doubleDequant of selected columns of a 2-D weight: [n_out, len(cols)].

    The same steps as ``quantize_nf4_dq`` + ``dequantize``: every block's c2
    and their Double Quantization (the mean and each 256-group need all of
    them), then the codes of the selected elements only.  Requires
    k_in % 64 == 0 (blocks do not straddle rows).
    """
    w = f32(w)
    n_out, k_in = w.shape
    if k_in % W_BLOCK:
        raise ValueError("dequantize_cols: k_in must be a multiple of 64")
    cols = np.asarray(cols, dtype=np.int64)
    bpr = k_in // W_BLOCK
    c2 = block_absmax(w.reshape(-1), W_BLOCK)
    code8, c1, mu = double_quantize(c2)
    c2_hat = dequant_c2(code8, c1, mu).reshape(n_out, bpr)[:, cols // W_BLOCK]
    c2_sel = c2.reshape(n_out, bpr)[:, cols // W_BLOCK]
    with np.errstate(invalid="ignore", divide="ignore"):
        x = (w[:, cols] / c2_sel).astype(np.float32)      # IEEE float32 quotient
    codes = nf4_code(np.where(c2_sel == 0, np.float32(0), x), levels)
    codes = np.where(c2_sel == 0, NF4_ZERO_CODE, codes).astype(np.uint8)
    prod = (np.asarray(levels, np.float32)[codes] * c2_hat).astype(np.float32)
    return bf16_bits_to_f32(bf16_rne_bits(prod))


def dequant_nf4_no_dq(codes, c2, shape) -> np.ndarray:
    """First-level dequant only (Eq. 2 with the absmax constant), float64."""
    codes = np.asarray(codes, dtype=np.uint8).reshape(-1)
    scale = np.repeat(f32(c2).astype(np.float64), W_BLOCK)[: codes.size]
    return (NF4_VALUES[codes].astype(np.float64) * scale).reshape(shape)


# --------------------------------------------------------------------------
# Storage accounting (§3 "Double Quantization" paragraph).
# --------------------------------------------------------------------------
def bits_per_parameter(numel: int, double_quant: bool = True) -> float:
    """Average storage bits per weight of the NF4 format.

    4 bits per code, plus per 64-block either a 32-bit constant (no DQ) or an
    8-bit constant, plus one 32-bit second-level constant per 256 first-level
    constants (DQ).  The single per-tensor mean is not counted.
    """
    nblk = (numel + W_BLOCK - 1) // W_BLOCK
    if double_quant:
        n1 = (nblk + C2_BLOCK - 1) // C2_BLOCK
        bits = 4 * numel + 8 * nblk + 32 * n1
    else:
        bits = 4 * numel + 32 * nblk
    return bits / numel
