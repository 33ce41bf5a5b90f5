"""Argument checks of the Python binding that run before any device pointer is
taken (no GPU needed): the grouped forward's member count and shapes."""

import pytest
import torch

qlora = pytest.importorskip("bit_nf4_quantized_02_b200")


def _member(M=4, N=16, K=64, r=8, k_l1=None):
    q = qlora.NF4Tensor(N, K, torch.zeros(N * K // 2, dtype=torch.uint8), torch.zeros(N * K // 64, dtype=torch.uint8),
                        torch.zeros(1), torch.zeros(1))
    return {"X": torch.zeros(M, K, dtype=torch.bfloat16), "q": q,
            "L1": torch.zeros(k_l1 or K, r, dtype=torch.bfloat16), "L2": torch.zeros(r, N, dtype=torch.bfloat16),
            "s": 1.0}


def test_group_size_bounds():
    with pytest.raises(ValueError, match="group holds"):
        qlora.linear_fwd_group([])
    with pytest.raises(ValueError, match="group holds"):
        qlora.linear_fwd_group([_member() for _ in range(9)])


def test_group_member_shape_mismatch():
    with pytest.raises(ValueError, match="shape mismatch"):
        qlora.linear_fwd_group([_member(k_l1=128)])
    bad = _member()
    bad["L2"] = torch.zeros(8, 24, dtype=torch.bfloat16)     # N of L2 differs from the weight's
    with pytest.raises(ValueError, match="shape mismatch"):
        qlora.linear_fwd_group([bad])


def test_host_tensors_are_refused():
    # a well-formed member on the host: the binding refuses to pass host memory as device pointers
    with pytest.raises(ValueError, match="CUDA device"):
        qlora.linear_fwd_group([_member()])
