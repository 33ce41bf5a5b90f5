"""Pins of the oracle's E4M3 codec, float32 fma, Double Quantization and
doubleDequant: library special cases (torch's float8_e4m3fn cast on CPU),
exact rational arithmetic, and error bounds.
"""

from fractions import Fraction

import numpy as np
import torch

from oracle import nf4dq
from synth import inputs


def test_e4m3_decode_all_codes_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = nf4dq.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    assert np.array_equal(np.signbit(ours[ok]), np.signbit(ref[ok]))
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9


def test_e4m3_encode_matches_torch_in_range():
    g = inputs.rng(21)
    parts = [inputs.normal_f32(g, 300000, s) for s in (1e-3, 0.05, 1.0, 30.0, 150.0)]
    mags = nf4dq._E4M3_MAGS
    mids = ((mags[:-1] + mags[1:]) / 2).astype(np.float32)      # exact ties
    near = np.concatenate([np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9))])
    x = np.concatenate(parts + [mids, -mids, near, -near, mags.astype(np.float32)])
    x = x[np.abs(x) <= 464.0]                 # beyond 464 torch's cast gives NaN (no saturation)
    ours = nf4dq.e4m3_encode_rne_satfinite(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_encode_saturates_and_signed_zero():
    x = np.array([448.0, 464.0, 465.0, 1e6, -1e6, -500.0, 0.0, -0.0], np.float32)
    assert nf4dq.e4m3_encode_rne_satfinite(x).tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x00, 0x80]


def _round_fraction_to_f32(q: Fraction) -> np.float32:
    """Exact round-to-nearest-even of a rational to float32 (normal and subnormal)."""
    if q == 0:
        return np.float32(0.0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)
    ulp = Fraction(2) ** (e - 23)
    n, rem = divmod(a, ulp)
    if rem * 2 > ulp or (rem * 2 == ulp and n % 2 == 1):
        n += 1
    return np.float32(sign * float(n * ulp))


def test_fma_f32_exact_against_rationals():
    g = inputs.rng(22)
    a = inputs.normal_f32(g, 3000, 1.0)
    b = inputs.normal_f32(g, 3000, 1e-3)
    c = inputs.normal_f32(g, 3000, 1e-2)
    # crafted double-rounding traps: a*b = 2^-24 - 2^-70, so a*b + c lies 2^-70
    # below the float32 midpoint 1 + 3*2^-24 (between an odd and an even
    # neighbour); a float64 sum rounds onto the midpoint and float32 RNE would
    # then go up, while the exact value rounds down.  Mirrored for negatives.
    u = 2.0 ** -23
    c2 = np.array([1 + u, -(1 + u), 1 + u], np.float32)
    a2 = np.array([2.0 ** -24 * (1 + u), -2.0 ** -24 * (1 + u), 2.0 ** -24 * 3], np.float32)
    b2 = np.array([1 - u, 1 - u, 1.0], np.float32)
    a = np.concatenate([a, a2])
    b = np.concatenate([b, b2])
    c = np.concatenate([c, c2])
    ours = nf4dq.fma_f32(a, b, c)
    ref = np.array([_round_fraction_to_f32(Fraction(float(x)) * Fraction(float(y)) + Fraction(float(z)))
                    for x, y, z in zip(a, b, c)], np.float32)
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))
    # the crafted cases really are double-rounding traps
    naive = (a2.astype(np.float64) * b2 + c2).astype(np.float32)
    assert not np.array_equal(naive[:2], ours[-3:-1])


def test_dq_mean_is_the_exact_mean():
    g = inputs.rng(23)
    c2 = np.abs(inputs.normal_f32(g, 5000, 0.05))
    exact = sum(Fraction(float(v)) for v in c2) / c2.size
    assert nf4dq.dq_mean(c2) == _round_fraction_to_f32(exact)


def test_double_quant_invariants_and_error_bound():
    g = inputs.rng(24)
    w = inputs.normal_f32(g, (128, 64 * 256 // 64 * 8), 0.02)     # 2048 blocks -> 8 c2 blocks... and more
    q = nf4dq.quantize_nf4_dq(w)
    c2, code8, c1, mu = q["c2"], q["c2_fp8"], q["c1"], q["mu"]
    n = c2.size
    assert code8.shape == (n,) and c1.shape == ((n + 255) // 256,)
    d = (c2 - mu).astype(np.float32)
    for b in range(c1.size):
        db = d[256 * b: 256 * (b + 1)]
        assert c1[b] == np.float32(np.abs(db).max()) / np.float32(448)
        # the block's extreme maps to +/-448
        i = np.abs(db).argmax()
        assert code8[256 * b + i] & 0x7F == 0x7E
    c2_hat = nf4dq.dequant_c2(code8, c1, mu).astype(np.float64)
    c1_per = np.repeat(c1.astype(np.float64), 256)[:n]
    # E4M3 keeps 3 mantissa bits: relative error <= 2^-4 in the normal range,
    # absolute <= 2^-10 (in units of c1) in the subnormal range; plus float32 roundings
    bound = np.maximum(2.0 ** -4 * np.abs(d), 2.0 ** -10 * c1_per) + 2.0 ** -22 * np.abs(c2)
    assert np.all(np.abs(c2_hat - c2) <= bound)


def test_double_quant_constant_block_is_exact():
    c2 = np.full(300, 0.037, np.float32)
    code8, c1, mu = nf4dq.double_quantize(c2)
    assert mu == np.float32(0.037) and np.all(c1 == 0) and np.all(code8 == 0)
    assert np.array_equal(nf4dq.dequant_c2(code8, c1, mu), c2)


def test_double_dequant_round_trip_bound():
    g = inputs.rng(25)
    w = inputs.normal_f32(g, (64, 1024), 0.02)
    q = nf4dq.quantize_nf4_dq(w)
    what = nf4dq.dequantize(q).astype(np.float64)
    c2 = np.repeat(q["c2"].astype(np.float64), 64).reshape(w.shape)
    c2_hat = np.repeat(nf4dq.dequant_c2(q["c2_fp8"], q["c1"], q["mu"]).astype(np.float64), 64).reshape(w.shape)
    lvl = nf4dq.NF4_VALUES.astype(np.float64)[q["codes"]].reshape(w.shape)
    # |w - W_hat| <= c2 * half max gap + |level| * |c2_hat - c2| + bf16 rounding
    bound = 0.1519036 * c2 + np.abs(lvl) * np.abs(c2_hat - c2) + 2.0 ** -8 * np.abs(what) + 1e-12
    assert np.all(np.abs(what - w) <= bound)
    # W_hat is exactly the bf16 rounding of level * c2_hat
    ref = torch.from_numpy((lvl * c2_hat).astype(np.float32)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(what.astype(np.float32), ref)


def test_double_dequant_codes7_is_zero():
    w = np.zeros((4, 128), np.float32)
    q = nf4dq.quantize_nf4_dq(w)
    assert np.all(q["codes"] == 7)
    assert np.all(nf4dq.dequantize(q) == 0.0)


def test_dequantize_rows_equals_full_dequantize():
    g = inputs.rng(26)
    w = inputs.normal_f32(g, (40, 1024), 0.02)   # 640 blocks: rows straddle 256-groups
    full = nf4dq.dequantize(nf4dq.quantize_nf4_dq(w))
    rows = [0, 3, 4, 17, 39]
    assert np.array_equal(nf4dq.dequantize_rows(w, rows), full[rows])


def test_dequantize_cols_equals_full_dequantize():
    g = inputs.rng(27)
    w = inputs.normal_f32(g, (40, 1024), 0.02)
    w[5, 128:192] = 0.0                          # an all-zero block: code 7 -> 0
    full = nf4dq.dequantize(nf4dq.quantize_nf4_dq(w))
    cols = [0, 63, 64, 130, 131, 700, 1023]
    assert np.array_equal(nf4dq.dequantize_cols(w, cols), full[:, cols])
