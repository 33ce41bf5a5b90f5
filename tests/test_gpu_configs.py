"""Full-size parity of the LLaMA-65B layer linears at 8192 tokens (forward
and backward, in the launch configuration the benchmark times), on sampled
outputs the oracle computes one by one."""

import numpy as np
import pytest
import torch

from parity import check_linear_sampled
from synth import inputs, workloads

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

qlora = pytest.importorskip("bit_nf4_quantized_02_b200")

WL = workloads.LLAMA65B_LAYER


@pytest.mark.parametrize("lin", [WL.linears[0], WL.linears[4], WL.linears[6]], ids=lambda l: l.name)
def test_llama65b_linear_full_size_sampled(lin):
    M, N, K, r, s = WL.M, lin.n_out, lin.k_in, WL.r, WL.s
    g = inputs.rng(WL.seed + N + K)
    W = inputs.weight_f32(g, N, K)
    X = inputs.normal_bf16(g, (M, K)).cuda()
    L1, L2 = (t.cuda() for t in inputs.lora_factors(g, K, N, r))
    dY = inputs.normal_bf16(g, (M, N)).cuda()
    q = qlora.quantize_nf4_dq(torch.from_numpy(W).cuda())
    Y, T = qlora.linear_fwd(X, q, L1, L2, s)
    dX, dL1, dL2 = qlora.linear_bwd(dY, X, T, q, L1, L2, s, grad_dtype=torch.float32)
    torch.cuda.synchronize()
    assert qlora.last_device_error() == 0
    check_linear_sampled(W, X, dY, L1, L2, s, Y, T, dX, dL1, dL2, tag=f"65B {lin.name} ")
