"""GPU parity of the quantizer and doubleDequant against the oracle: bit-exact
codes, E4M3 constant codes, c1, mean and dequantized bf16 weights."""

import numpy as np
import pytest
import torch

from oracle import nf4dq
from parity import gpu_quant_to_np, oracle_quant
from synth import inputs, workloads

pytestmark = pytest.mark.gpu

qlora = pytest.importorskip("bit_nf4_quantized_02_b200")


def _check_bit_exact(W_cpu: torch.Tensor):
    q = qlora.quantize_nf4_dq(W_cpu.cuda())
    got = gpu_quant_to_np(q)
    oq = oracle_quant(W_cpu)
    assert got["mu"] == oq["mu"], (got["mu"], oq["mu"])
    assert np.array_equal(got["packed"], oq["packed"])
    assert np.array_equal(got["c2_fp8"], oq["c2_fp8"])
    assert np.array_equal(got["c1"].view(np.uint32), oq["c1"].view(np.uint32))
    w_hat = qlora.dequant(q)
    ref_bits = nf4dq.double_dequant_bits(oq["codes"], oq["c2_fp8"], oq["c1"], oq["mu"], oq["shape"])
    got_bits = w_hat.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got_bits, ref_bits)
    assert qlora.last_device_error() == 0
    return q, oq


@pytest.mark.parametrize("shape", [(1, 64), (1, 1), (3, 100), (7, 333), (2, 256), (5, 320), (64, 4096),
                                   (257, 64 * 257), (33, 1000), (1, 8205), (3, 8192), (1, 8192 * 9 + 64)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quantize_dequant_bit_exact_small(shape, dtype):
    g = inputs.rng(100 + shape[0] * 7 + shape[1])
    W = torch.from_numpy(inputs.normal_f32(g, shape, 0.02)).to(dtype)
    _check_bit_exact(W)


def test_quantize_special_values():
    # zero blocks, a block whose absmax is negative, exact midpoints, signed zeros
    W = torch.zeros(4, 256, dtype=torch.float32)
    W[1, :64] = torch.linspace(-1, 1, 64)
    W[2, 64:128] = -3.0
    mids = (nf4dq.NF4_MIDPOINTS.astype(np.float32))
    W[3, :15] = torch.from_numpy(mids)
    W[3, 15] = 1.0
    W[3, 16] = -0.0
    W[0, 200] = 1e-38
    _check_bit_exact(W)


def _near_threshold_blocks(seed: int) -> np.ndarray:
    """64-blocks whose first element fixes the absmax (alternating sign) and
    whose others sit at, within 40 ulps of, and within five 2^-13 steps of,
    every decision threshold, at several absmax scales."""
    g = np.random.default_rng(seed)
    xs = []
    for m in nf4dq.NF4_MIDPOINTS.astype(np.float64):
        t = np.float32(m)
        up, down = t, t
        xs.append(t)
        for _ in range(40):
            up = np.nextafter(up, np.float32(np.inf), dtype=np.float32)
            down = np.nextafter(down, np.float32(-np.inf), dtype=np.float32)
            xs += [up, down]
        xs += [np.float32(m + k * 2.0 ** -13 + g.uniform(-2.0 ** -14, 2.0 ** -14)) for k in range(-5, 6)]
    xs = np.array(xs, dtype=np.float32)
    blocks = []
    for amax in (1.0, 0.37, 3.1e-5, 1234.5, 3 * 2.0 ** -20, 7e-3):
        a = np.float32(amax)
        v = np.clip((xs.astype(np.float64) * amax).astype(np.float32), -a, a)
        for n, i in enumerate(range(0, v.size, 63)):
            blk = np.zeros(64, dtype=np.float32)
            blk[0] = a if n % 2 == 0 else -a
            blk[1:1 + v[i:i + 63].size] = v[i:i + 63]
            blocks.append(blk)
    return np.stack(blocks)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quantize_near_every_threshold(dtype):
    """Weights at and around each NF4 decision threshold: the nearest-level
    decision must match the oracle's exact division bit for bit (this drives
    the boundary bins of the kernel's table and their exact-division path)."""
    B = _near_threshold_blocks(77)
    W = torch.from_numpy(B[: B.shape[0] // 8 * 8].reshape(-1, 512).copy())
    _check_bit_exact(W.to(dtype))


def test_quantize_constant_c2_gives_zero_c1():
    W = torch.ones(16, 64 * 256 // 16, dtype=torch.float32) * 0.5
    q, oq = _check_bit_exact(W)
    assert np.all(oq["c1"] == 0)


def test_config1_weight_fp32():
    wl = workloads.SINGLE_1024
    g = inputs.rng(wl.seed)
    W = torch.from_numpy(inputs.weight_f32(g, 1024, 1024))
    _check_bit_exact(W)


def test_config3_style_bf16_with_outliers_medium():
    g = inputs.rng(777)
    W = inputs.weight_bf16_with_outliers(g, 512, 4096)
    _check_bit_exact(W)


def test_zero_sized_weight():
    q = qlora.quantize_nf4_dq(torch.empty(0, 64, device="cuda"))
    assert float(q.c2_mean.cpu()[0]) == 0.0


@pytest.mark.slow
def test_config3_full_size_sampled():
    """All 8 matrices of the quantizer workload at full size: every c2_fp8, c1 and
    the mean compared in full; codes and dequantized weights on sampled blocks."""
    wl = workloads.QUANTIZER_7B
    rs = np.random.default_rng(5)
    for i, lin in enumerate(wl.linears):
        Wd = inputs.device_weight_with_outliers(lin.n_out, lin.k_in, wl.seed + i, "cuda")
        q = qlora.quantize_nf4_dq(Wd)
        w_hat = qlora.dequant(q)
        got = gpu_quant_to_np(q)
        flat = Wd.float().cpu().numpy().reshape(-1)
        c2 = nf4dq.block_absmax(flat, 64)
        code8, c1, mu = nf4dq.double_quantize(c2)
        assert got["mu"] == mu
        assert np.array_equal(got["c2_fp8"], code8)
        assert np.array_equal(got["c1"].view(np.uint32), c1.view(np.uint32))
        blocks = rs.choice(c2.size, size=4096, replace=False)
        idx = (blocks[:, None] * 64 + np.arange(64)[None, :]).reshape(-1)
        codes_ref, c2_ref = nf4dq.quantize_nf4(flat[idx])
        assert np.array_equal(c2_ref, c2[blocks])
        got_codes = nf4dq.unpack_nibbles(got["packed"], flat.size)[idx]
        assert np.array_equal(got_codes, codes_ref)
        c2_hat = nf4dq.dequant_c2(code8, c1, mu)[blocks]
        ref_bits = nf4dq.bf16_rne_bits((nf4dq.NF4_VALUES[codes_ref] * np.repeat(c2_hat, 64)).astype(np.float32))
        got_bits = w_hat.view(torch.int16).reshape(-1)[torch.from_numpy(idx).cuda()].cpu().numpy().view(np.uint16)
        assert np.array_equal(got_bits, ref_bits)
        del Wd, q, w_hat
    assert qlora.last_device_error() == 0


@pytest.mark.slow
@pytest.mark.parametrize("dtype,shape", [(torch.float32, (4096, 4096)), (torch.bfloat16, (8192, 4096))])
def test_streamed_ring_reuse_repeated(dtype, shape):
    """Weights large enough that every CTA of the quantizer refills each slot of
    its shared-memory ring many times (fp32 16.7 M and bf16 33.5 M weights
    against 148 CTAs of 5 and 10 slots of 8192 weights), quantized repeatedly:
    bit-exact every time.  A refill that overtook the reads of a slot gave a
    few groups the codes of the chunk five slots later."""
    g = inputs.rng(4242 + shape[0])
    W = torch.from_numpy(inputs.weight_f32(g, *shape)).to(dtype)
    oq = oracle_quant(W)
    Wd = W.cuda()
    for _ in range(4):
        q = qlora.quantize_nf4_dq(Wd)
        got = gpu_quant_to_np(q)
        assert got["mu"] == oq["mu"]
        assert np.array_equal(got["packed"], oq["packed"])
        assert np.array_equal(got["c2_fp8"], oq["c2_fp8"])
        assert np.array_equal(got["c1"].view(np.uint32), oq["c1"].view(np.uint32))
    ref_bits = nf4dq.double_dequant_bits(oq["codes"], oq["c2_fp8"], oq["c1"], oq["mu"], oq["shape"])
    for _ in range(3):
        got_bits = qlora.dequant(q).cpu().view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(got_bits, ref_bits)
    assert qlora.last_device_error() == 0
