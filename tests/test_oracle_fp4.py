"""Pins of the oracle's FP4 (E2M1) storage table, the 4-bit float the paper
compares NF4 against (§4, Tables 2-4).

The table is pinned to the E2M1 encoding's definition (value of each of the
16 bit patterns), the nearest-level rule to a brute-force argmin, and the
comparison itself to the property the pages report: on normally distributed
weights NF4 reconstructs blocks with less error than FP4."""

import numpy as np

from oracle import nf4dq


def test_fp4_table_is_the_normalised_e2m1_value_set():
    t = nf4dq.FP4_VALUES
    assert t.dtype == np.float32 and t.size == 16
    assert np.all(np.diff(t.astype(np.float64)) >= 0)          # ascending (the two zeros equal)
    assert t[7] == 0.0 and t[8] == 0.0 and t[0] == -1.0 and t[15] == 1.0
    # the distinct values times 6 are exactly E2M1's value set
    e2m1 = sorted({nf4dq.e2m1_value(b) for b in range(16)})
    assert e2m1 == [-6, -4, -3, -2, -1.5, -1, -0.5, 0, 0.5, 1, 1.5, 2, 3, 4, 6]
    for v in e2m1:
        assert np.float32(v) / np.float32(6.0) in t
    # E2M1 encoding spot checks: 0b0111 = +6, 0b0001 = +0.5 (subnormal), 0b1100 = -2
    assert nf4dq.e2m1_value(0b0111) == 6.0 and nf4dq.e2m1_value(0b0001) == 0.5 and nf4dq.e2m1_value(0b1100) == -2.0


def test_fp4_nearest_level_matches_brute_force():
    g = np.random.default_rng(3)
    t = nf4dq.FP4_VALUES.astype(np.float64)
    mids = nf4dq.midpoints(nf4dq.FP4_VALUES)
    x = np.concatenate([g.uniform(-1, 1, 20000), mids, np.nextafter(mids, 2), np.nextafter(mids, -2),
                        [0.0, -0.0, 1.0, -1.0]]).astype(np.float32)
    codes = nf4dq.nf4_code(x, nf4dq.FP4_VALUES)
    xd = x.astype(np.float64)
    dist = np.abs(xd[:, None] - t[None, :])
    best = dist.min(axis=1, keepdims=True)
    lowest = np.argmax(dist == best, axis=1)          # ties to the lowest index
    # the two zero codes hold the same value: the decoded levels must agree,
    # and the codes wherever the nearest level is not zero
    np.testing.assert_array_equal(t[codes], t[lowest])
    nz = t[lowest] != 0
    np.testing.assert_array_equal(codes[nz], lowest[nz])
    # the midpoint rule sends x <= 0 to code 7 and 0 < x <= 1/24 to code 8
    assert np.all(codes[(xd > 0) & (t[codes] == 0)] == 8) and np.all(codes[(xd <= 0) & (t[codes] == 0)] == 7)


def test_fp4_round_trip_and_zero_code():
    g = np.random.default_rng(4)
    w = (g.standard_normal((8, 256)) * 0.02).astype(np.float32)
    w[3, :64] = 0.0                                    # an all-zero block
    q = nf4dq.quantize_nf4_dq(w, nf4dq.FP4_VALUES)
    assert np.all(q["codes"].reshape(8, 256)[3, :64] == nf4dq.NF4_ZERO_CODE)
    wh = nf4dq.dequantize(q)
    assert np.all(wh[3, :64] == 0.0)
    # first-level error bound: half the largest gap between adjacent levels, times c2
    gap = np.max(np.diff(nf4dq.FP4_VALUES.astype(np.float64))) / 2
    c2 = q["c2"].astype(np.float64)
    err = np.abs(nf4dq.FP4_VALUES[q["codes"]].astype(np.float64) * np.repeat(c2, 64) - w.reshape(-1))
    assert np.all(err <= gap * np.repeat(c2, 64) + 1e-12)


def test_nf4_reconstructs_normal_weights_better_than_fp4():
    """The comparison of §4 in its simplest form: quantization error of
    N(0, 0.02^2) weights in absmax blocks of 64, NF4 against FP4 (E2M1)."""
    g = np.random.default_rng(5)
    w = (g.standard_normal((256, 4096)) * 0.02).astype(np.float32)
    err = {}
    for name, levels in nf4dq.TABLES.items():
        q = nf4dq.quantize_nf4_dq(w, levels)
        err[name] = float(np.sqrt(np.mean((nf4dq.dequantize(q).astype(np.float64) - w) ** 2)))
    assert err["nf4"] < err["fp4"]
    assert err["nf4"] < 0.95 * err["fp4"]
