"""The facts the quantizer's division-free code table rests on, checked on the
host for both code tables (NF4, QLoRA §3 "4-bit NormalFloat Quantization" and
Appendix E; FP4 (E2M1), §4 Tables 2-4).

The kernel (nf4_quantize_kernel) estimates a weight's position X = (x + 1) *
8192 in bins of 2^-13, x = fp32(w / absmax), from one fused multiply-add whose
error is at most 2^-10 of a bin, and looks its code up per estimated bin e.
Bins whose interval widened by d = 2^-8 of a bin holds a threshold are marked
for the exact division; every other bin stores #{j : threshold j below it}.
Here: the thresholds are exact in the kernel's fixed point (2^16 units per
bin) and far enough apart for its 128-bin build passes, and, brute force over
fp32 values around every threshold, every estimate within the error bound
that lands in an unmarked bin reads the code the exact rule gives (the
oracle's nearest level), while a marked bin's index j leaves only j or j + 1.
The GPU tests check the kernel's own table against the oracle bit for bit."""

import math

import numpy as np
import pytest

from oracle import nf4dq

BINS = 16384
FIX = 1 << 16             # fixed-point units per bin
MARGIN = FIX >> 8         # d = 2^-8 of a bin
EST_ERR = 2.0 ** -10      # bound on |estimate - X| in bins


def _thresholds(levels):
    """Midpoints of neighbouring levels rounded toward -inf to fp32 (x > m_j
    <=> x > RD(m_j) for an fp32 x)."""
    lev = np.asarray(levels, np.float32).astype(np.float64)
    out = []
    for j in range(15):
        m = (lev[j] + lev[j + 1]) * 0.5
        f = np.float32(m)
        if float(f) > m:
            f = np.nextafter(f, np.float32(-np.inf))
        out.append(float(f))
    return out


def _table(pos, margin=MARGIN):
    """Entry e + 1 for the estimated bin e in [-1, BINS]: 0x80 | j when the
    bin widened by `margin` holds threshold j, else the count of thresholds
    below it."""
    ent = np.zeros(BINS + 2, np.int64)
    for i in range(BINS + 2):
        e = i - 1
        lo, hi = e * FIX - margin, (e + 1) * FIX + margin
        js = [j for j, p in enumerate(pos) if lo <= p <= hi]
        assert len(js) <= 1
        ent[i] = (0x80 | js[0]) if js else sum(p < lo for p in pos)
    return ent


TABLES = {"nf4": nf4dq.NF4_VALUES, "fp4": nf4dq.FP4_VALUES}


@pytest.mark.parametrize("name", sorted(TABLES))
def test_thresholds_exact_in_fixed_point_and_far_apart(name):
    t = _thresholds(TABLES[name])
    for tj in t:
        p = (tj + 1.0) * (1 << 29)
        assert p == math.floor(p) and 0 < p < 2 ** 30
    pos = [(tj + 1.0) * 8192 for tj in t]
    gaps = np.diff(pos)
    # a build pass covers 128 bins plus margins: at most one threshold matters to it
    assert gaps.min() > 341 and gaps.min() > 128 + 2
    # the last upper edge in fixed point stays a positive 32-bit int
    assert (BINS + 2) * FIX + MARGIN < 2 ** 31


@pytest.mark.parametrize("name", sorted(TABLES))
def test_unmarked_bins_give_the_exact_code(name):
    t = _thresholds(TABLES[name])
    pos = [int((tj + 1.0) * (1 << 29)) for tj in t]
    lut = _table(pos)
    marked = int((lut & 0x80).astype(bool).sum())
    # one bin per threshold, two only when it sits within d of a bin edge
    assert 15 <= marked <= 30
    tt = np.asarray(t, np.float32)
    xs = []
    for tj in t:
        f = np.float32(tj)
        ulp = float(np.spacing(f)) if f != 0 else float(np.spacing(np.float32(2.0 ** -20)))
        xs.append(tj + ulp * np.arange(-400, 401))
        xs.append(tj + np.linspace(-3, 3, 1201) * 2.0 ** -13)
    xs.append(np.linspace(-1, 1, 20001))
    x = np.clip(np.float32(np.concatenate(xs)), -1, 1)
    code = (x[:, None] > tt[None, :]).sum(1)          # the nearest-level rule on fp32 x
    X = (x.astype(np.float64) + 1.0) * 8192.0
    for dev in (-EST_ERR, -EST_ERR / 2, 0.0, EST_ERR / 2, EST_ERR):
        e = np.floor(X + dev).astype(np.int64)
        ent = lut[e + 1]
        plain = (ent & 0x80) == 0
        assert np.array_equal(ent[plain], code[plain])
        j = ent[~plain] & 0xF
        assert np.all((code[~plain] == j) | (code[~plain] == j + 1))


def test_wider_estimate_error_would_break_an_unmarked_bin():
    """Planted mistake: with no margin and an estimate error of a full bin the
    table is not exact, so the check above can fail."""
    t = _thresholds(TABLES["nf4"])
    pos = [int((tj + 1.0) * (1 << 29)) for tj in t]
    lut = _table(pos, margin=0)
    tt = np.asarray(t, np.float32)
    x = np.float32(np.concatenate([tj + np.linspace(-2, 2, 401) * 2.0 ** -13 for tj in t]))
    code = (x[:, None] > tt[None, :]).sum(1)
    e = np.floor((x.astype(np.float64) + 1.0) * 8192.0 + 1.0).astype(np.int64)   # one bin off
    ent = lut[np.clip(e + 1, 0, BINS + 1)]
    plain = (ent & 0x80) == 0
    assert not np.array_equal(ent[plain], code[plain])
