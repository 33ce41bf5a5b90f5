"""bench.py's host arithmetic, on the CPU: the algorithmic FLOP and byte
counts behind every rate it reports, and the per-kernel table and launch
count it builds from the library's event log.

The counts are pinned to figures worked out by hand for the workloads:
fwd+bwd of a QLoRA linear is 4MKN + 6Mr(K+N) FLOPs (the two base products
plus T, T·L2, G, G·L1^T, dL1 and dL2, each 2Mr(K or N)); a stored NF4 + DQ
weight is 4 + 8/64 + 32/(64·256) bits per parameter plus one fp32 mean
(QLoRA §3 "Double Quantization")."""

import pytest

import bench
from synth import workloads


def test_linear_flops_partition():
    M, N, K, r = 300, 520, 192, 16
    f = bench.linear_flops(M, N, K, r)
    base = 2 * M * N * K
    assert f["fwd"] + f["bwd"] == f["fwd_bwd"] == 4 * M * N * K + 6 * M * r * (K + N)
    assert f["fwd"] == base + 2 * M * r * K + 2 * M * r * N            # X·W^T, T = X·L1, T·L2
    assert f["gemm_Y"] == base + 2 * M * r * N and f["gemm_dX"] == base + 2 * M * r * K
    # what the two big products leave: T, G, dL1, dL2
    assert f["fwd_bwd"] - f["gemm_Y"] - f["gemm_dX"] == 2 * M * r * (K + N) * 2


@pytest.mark.parametrize("wl, tflop", [(workloads.LLAMA7B_LAYER, 6.88), (workloads.LLAMA65B_LAYER, 27.0)])
def test_step_flops_of_the_training_layers(wl, tflop):
    assert bench.step_flops(wl.linears, wl.M, wl.r) / 1e12 == pytest.approx(tflop, abs=0.05)


def test_step_flops_llama7b_exact():
    M, r = 8192, 64
    base = 4 * M * (4 * 4096 * 4096 + 3 * 4096 * 11008)
    lora = 6 * M * r * (4 * (4096 + 4096) + 3 * (4096 + 11008))
    assert bench.step_flops() == base + lora == 6_877_047_947_264


def test_stack_flops_llama33b():
    wl = workloads.LLAMA33B_STACK
    assert wl.layers * bench.step_flops(wl.linears, wl.M, wl.r) / 1e12 == pytest.approx(143.5, abs=0.05)


def test_nf4_bytes_per_parameter():
    # 4096 x 4096: codes n/2, one E4M3 code per 64, one fp32 c1 per 64*256, one fp32 mean
    n = 4096 * 4096
    assert bench.nf4_nbytes(4096, 4096) == n // 2 + n // 64 + 4 * n // (64 * 256) + 4
    assert bench.nf4_nbytes(4096, 4096) / n == pytest.approx(0.51587, abs=1e-5)
    # ragged: a tail 64-block and a tail 256-group still take a code and a constant
    assert bench.nf4_nbytes(3, 65) == 98 + 4 + 4 + 4


def test_decode_step_bytes_llama65b_16_tokens():
    b = bench.decode_step_bytes(16, 64)
    nf4 = sum(bench.nf4_nbytes(l.n_out, l.k_in) for l in workloads.LLAMA65B_LAYER.linears)
    assert nf4 / 1e6 == pytest.approx(417.6, abs=0.05)
    assert b / 1e6 == pytest.approx(442.6, abs=0.05)
    assert b == 442_610_716


def test_quantizer_bytes():
    lins = workloads.QUANTIZER_7B.linears
    params = sum(l.n_out * l.k_in for l in lins)
    assert params == 333_447_168
    stored = sum(bench.nf4_nbytes(l.n_out, l.k_in) for l in lins)
    # quantize reads the bf16 weights and writes the stored format; dequant the reverse
    assert 2 * params / 1e6 == pytest.approx(667, abs=0.5) and stored / 1e6 == pytest.approx(172, abs=0.5)
    assert 2 * params + stored == 838_909_472


def test_kernel_table_and_launch_count():
    launches = [("gemm_Y", 1.0), ("quantize", 0.5), ("gemm_Y", 2.0), ("fused_fwd", 0.25), ("quantize", 0.5)]
    per_kind, table = bench._kernel_table(launches, steps=2)
    assert per_kind["gemm_Y"] == [2, 3.0] and per_kind["quantize"] == [2, 1.0]
    assert list(table) == ["gemm_Y", "quantize", "fused_fwd"]            # by time per step
    assert table["gemm_Y"]["launches_per_step"] == 1.0 and table["gemm_Y"]["ms_per_step"] == 1.5
    assert sum(v["share"] for v in table.values()) == pytest.approx(1.0)
    assert table["fused_fwd"]["share"] == pytest.approx(0.25 / 4.25)
    # one few-token forward entry stands for its three kernels
    assert bench._kernel_count(launches) == 4 + 3
    assert bench._kernel_table([], steps=1) == ({}, {})


def test_training_configs_name_the_token_batches():
    import argparse
    args = argparse.Namespace(workload="llama7b-train", linear=None, dropout=0.0)
    c = bench.train_config(args, workloads.LLAMA7B_LAYER, 1)
    assert (c["global_batch"], c["seq_len"], c["tokens_per_rank"]) == (16, 512, 8192)
    assert c["parallelism"] == "single"
    args.workload = "llama65b-train"
    c = bench.train_config(args, workloads.LLAMA65B_LAYER, 2)
    assert (c["global_batch"], c["seq_len"], c["parallelism"]) == (8, 2048, "dp2")
