"""Pins of the oracle's NF4 table, nearest-code rule, blocking, packing and
storage accounting against what the QLoRA paper prints and against brute force.
"""

import numpy as np
import pytest
import torch
from scipy.optimize import minimize_scalar
from scipy.stats import norm

from conftest import read_golden
from oracle import nf4dq
from synth import inputs


def test_table_matches_appendix_e():
    printed = np.array([float(r[0]) for r in read_golden("nf4_table.txt")])
    assert printed.size == 16
    assert np.array_equal(nf4dq.NF4_VALUES.astype(np.float64), printed)
    # every printed value is exactly a float32
    assert np.array_equal(printed.astype(np.float32).astype(np.float64), printed)


def test_table_structure():
    t = nf4dq.NF4_VALUES.astype(np.float64)
    assert t.size == 16                      # 2^k values for k = 4
    assert np.all(np.diff(t) > 0)            # strictly increasing
    assert t[0] == -1.0 and t[15] == 1.0     # normalised to [-1, 1]
    assert t[nf4dq.NF4_ZERO_CODE] == 0.0     # exact zero
    assert (t < 0).sum() == 7 and (t > 0).sum() == 8   # 2^(k-1) negative + (2^(k-1)+1) positive - shared 0


def _asym_quantile_table(p_max):
    # §3 Eq. 4 and the asymmetric construction after it: quantiles of N(0, 1)
    # on an even probability grid, 2^(k-1)=8 levels for the negative half and
    # 2^(k-1)+1=9 for the positive half (both including 0), each half
    # normalised to [-1, 1], the duplicated zero dropped.
    pos = norm.ppf(np.linspace(p_max, 0.5, 9))
    neg = norm.ppf(np.linspace(p_max, 0.5, 8))
    return np.sort(np.concatenate([-(neg / neg[0])[:-1], pos / pos[0]]))


def test_table_is_the_asymmetric_normal_quantile_construction():
    t = nf4dq.NF4_VALUES.astype(np.float64)
    res = minimize_scalar(lambda p: np.abs(_asym_quantile_table(p) - t).max(),
                          bounds=(0.9, 0.999), method="bounded", options={"xatol": 1e-12})
    assert res.fun < 2e-7, res.fun
    assert abs(res.x - 0.96771) < 1e-4


def test_eq4_literal_first_term_is_unbounded():
    # Read literally, Eq. 4 evaluates the quantile function at i/(2^k+1) = 0 for
    # i = 0, which is -inf: the printed table (Appendix E) is the authority.
    assert norm.ppf(0.0) == -np.inf


def _brute_code(x):
    x = np.asarray(x, np.float32).astype(np.float64)
    d = np.abs(x[:, None] - nf4dq.NF4_VALUES.astype(np.float64)[None, :])
    # argmin returns the first (lowest) index on ties
    return d.argmin(axis=1).astype(np.uint8)


def test_nearest_code_exhaustive_over_bf16_in_range():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    x = nf4dq.bf16_bits_to_f32(bits)
    x = x[np.isfinite(x) & (np.abs(x) <= 1.0)]
    assert np.array_equal(nf4dq.nf4_code(x), _brute_code(x))


def test_nearest_code_random_and_midpoints():
    g = inputs.rng(7)
    x = (g.random(200000, dtype=np.float32) * 2 - 1).astype(np.float32)
    assert np.array_equal(nf4dq.nf4_code(x), _brute_code(x))
    # float32 values closest to each midpoint: exact ties go to the lower index
    m = nf4dq.NF4_MIDPOINTS
    cands = []
    for v in m:
        f = np.float32(v)
        cands += [np.nextafter(f, np.float32(-2)), f, np.nextafter(f, np.float32(2))]
    cands = np.array(cands, np.float32)
    assert np.array_equal(nf4dq.nf4_code(cands), _brute_code(cands))


def test_quantize_tiny_vs_brute_force():
    g = inputs.rng(11)
    w = inputs.normal_f32(g, (3, 128), 0.02)
    codes, c2 = nf4dq.quantize_nf4(w)
    flat = w.reshape(-1)
    assert c2.shape == (6,)
    for b in range(6):
        blk = flat[64 * b: 64 * (b + 1)]
        assert c2[b] == np.abs(blk).max()
        x = (blk / c2[b]).astype(np.float32)
        assert np.array_equal(codes[64 * b: 64 * (b + 1)], _brute_code(x))


def test_zero_block_and_tail_block():
    w = np.zeros(100, np.float32)
    w[70] = -0.5
    w[99] = 0.25
    codes, c2 = nf4dq.quantize_nf4(w)
    assert c2.tolist() == [0.0, 0.5]                   # block 0 all zero; tail block of 36
    assert np.all(codes[:64] == nf4dq.NF4_ZERO_CODE)
    assert codes[70] == 0                              # -0.5/0.5 = -1 -> code 0
    assert codes[99] == 12                             # 0.25/0.5 = 0.5 -> nearest level 0.4407 (code 12)
    assert np.all(np.delete(codes[64:], [6, 35]) == nf4dq.NF4_ZERO_CODE)


def test_round_trip_error_bound_without_dq():
    g = inputs.rng(12)
    w = inputs.normal_f32(g, (64, 256), 0.02)
    codes, c2 = nf4dq.quantize_nf4(w)
    wq = nf4dq.dequant_nf4_no_dq(codes, c2, w.shape)
    scale = np.repeat(c2.astype(np.float64), 64).reshape(w.shape)
    err = np.abs(wq - w.astype(np.float64))
    half_gap = np.diff(nf4dq.NF4_VALUES.astype(np.float64)).max() / 2
    assert abs(half_gap - 0.1519036) < 1e-6
    assert np.all(err <= half_gap * scale * (1 + 1e-6))
    # the local bound: half the gap around the chosen level
    t = nf4dq.NF4_VALUES.astype(np.float64)
    gaps = np.diff(t)
    lo = np.concatenate([[0.0], gaps])[codes]
    hi = np.concatenate([gaps, [0.0]])[codes]
    local = np.maximum(lo, hi).reshape(w.shape) / 2
    assert np.all(err <= local * scale * (1 + 1e-6) + 1e-12)
    # block extremes are represented exactly (the absmax maps to +/-1)
    blk = w.reshape(-1, 64)
    amax = np.abs(blk).argmax(axis=1)
    ex = codes.reshape(-1, 64)[np.arange(blk.shape[0]), amax]
    assert np.all((ex == 0) | (ex == 15))


def test_pack_nibbles_order():
    codes = np.array([1, 2, 3], np.uint8)
    packed = nf4dq.pack_nibbles(codes)
    assert packed.tolist() == [0x21, 0x03]
    assert nf4dq.unpack_nibbles(packed, 3).tolist() == [1, 2, 3]
    g = inputs.rng(3)
    c = g.integers(0, 16, 1001).astype(np.uint8)
    assert np.array_equal(nf4dq.unpack_nibbles(nf4dq.pack_nibbles(c), 1001), c)


def test_bits_accounting_matches_paper():
    gold = {r[0]: (float(r[1]), float(r[2])) for r in read_golden("bits_accounting.txt")}
    n = 64 * 256 * 1000
    no_dq = nf4dq.bits_per_parameter(n, double_quant=False) - 4
    dq = nf4dq.bits_per_parameter(n, double_quant=True) - 4
    assert no_dq == 0.5 and dq == 0.126953125
    for key, val in (("constants_bits_no_dq", no_dq), ("constants_bits_dq", dq),
                     ("saving_bits", no_dq - dq)):
        printed, tol = gold[key]
        assert abs(val - printed) <= tol, key
    saved_gb = 65e9 * (no_dq - dq) / 8 / 1e9
    printed, tol = gold["saving_gb_65b"]
    assert abs(saved_gb - printed) <= tol
    # the oracle's actual output sizes agree with the accounting
    q = nf4dq.quantize_nf4_dq(np.ones((256, 64 * 4), np.float32))
    numel = 256 * 256
    bits = 8 * (q["packed"].nbytes + q["c2_fp8"].nbytes + q["c1"].nbytes)
    assert bits / numel == nf4dq.bits_per_parameter(numel, True)


def test_bf16_rounding_matches_torch():
    g = inputs.rng(5)
    x = np.concatenate([inputs.normal_f32(g, 100000, 3.0),
                        inputs.normal_f32(g, 1000, 1e-30),
                        np.array([0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8)], np.float32)])
    ours = nf4dq.bf16_rne_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
