"""Argument checks of the Python binding that run before the library is loaded
or any device pointer is taken (no GPU, no built library needed): member
counts and shapes, caller-supplied outputs of the wrong shape or dtype,
tensors on different devices, and grouped outputs that overlap inputs; and
that without the built library the binding raises instead of computing."""

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


def _linear_args(M=4, N=16, K=64, r=8):
    m = _member(M, N, K, r)
    return m["X"], m["q"], m["L1"], m["L2"]


@pytest.mark.parametrize("name,bad", [
    ("Y", lambda M, N, K, r: torch.zeros(M - 1, N, dtype=torch.bfloat16)),      # too small: written past its end
    ("Y", lambda M, N, K, r: torch.zeros(M, N, dtype=torch.float32)),
    ("T", lambda M, N, K, r: torch.zeros(M, r, dtype=torch.bfloat16)),          # T is the [M, 2r] hi/lo pair
])
def test_forward_outputs_are_checked(name, bad):
    M, N, K, r = 4, 16, 64, 8
    X, q, L1, L2 = _linear_args(M, N, K, r)
    with pytest.raises(ValueError, match=f"{name} must be"):
        qlora.linear_fwd(X, q, L1, L2, 1.0, **{name: bad(M, N, K, r)})


@pytest.mark.parametrize("name,bad,kw", [
    ("dX", lambda M, N, K, r: torch.zeros(M, K + 64, dtype=torch.bfloat16), {}),
    ("dL1", lambda M, N, K, r: torch.zeros(K, r, dtype=torch.bfloat16), {"grad_dtype": torch.float32}),
    ("dL2", lambda M, N, K, r: torch.zeros(r, N, dtype=torch.float32), {}),
    ("dL2", lambda M, N, K, r: torch.zeros(r, N - 8, dtype=torch.bfloat16), {}),
])
def test_backward_outputs_are_checked(name, bad, kw):
    M, N, K, r = 4, 16, 64, 8
    X, q, L1, L2 = _linear_args(M, N, K, r)
    dY = torch.zeros(M, N, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match=f"{name} must be"):
        qlora.linear_bwd(dY, X, None, q, L1, L2, 1.0, **{name: bad(M, N, K, r)}, **kw)


def test_backward_saved_T_shape_is_checked():
    M, N, K, r = 4, 16, 64, 8
    X, q, L1, L2 = _linear_args(M, N, K, r)
    dY = torch.zeros(M, N, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="hi/lo pair"):
        qlora.linear_bwd(dY, X, torch.zeros(M, r, dtype=torch.bfloat16), q, L1, L2, 1.0)


def test_tensors_on_another_device_are_refused():
    X, q, L1, L2 = _linear_args()
    with pytest.raises(ValueError, match="L2 is on meta"):
        qlora.linear_fwd(X, q, L1, L2.to("meta"), 1.0)
    m = _member()
    m["L1"] = m["L1"].to("meta")
    with pytest.raises(ValueError, match="L1 is on meta"):
        qlora.linear_fwd_group([m])


def test_group_outputs_may_not_overlap_inputs_or_each_other():
    M, N, K, r = 4, 16, 64, 8
    a, b = _member(M, N, K, r), _member(M, N, K, r)
    b["X"] = a["X"]                                        # shared input: allowed
    a["Y"] = a["X"].view(-1)[:M * N].view(M, N)            # output aliasing the shared input
    with pytest.raises(ValueError, match="member 0's Y overlaps member 0's X"):
        qlora.linear_fwd_group([a, b])
    a, b = _member(M, N, K, r), _member(M, N, K, r)
    buf = torch.zeros(M * N + 8, dtype=torch.bfloat16)
    a["Y"] = buf[:M * N].view(M, N)
    b["Y"] = buf[8:].view(M, N)                            # two outputs sharing bytes
    with pytest.raises(ValueError, match="member 0's Y overlaps member 1's Y"):
        qlora.linear_fwd_group([a, b])


def _bwd_member(M=4, N=16, K=64, r=8, **kw):
    m = _member(M, N, K, r)
    m.update({"dY": torch.zeros(M, N, dtype=torch.bfloat16), "T": None})
    m.update(kw)
    return m


def test_bwd_group_size_and_shapes():
    with pytest.raises(ValueError, match="group holds"):
        qlora.linear_bwd_group([])
    with pytest.raises(ValueError, match="group holds"):
        qlora.linear_bwd_group([_bwd_member() for _ in range(9)])
    with pytest.raises(ValueError, match="shape mismatch"):
        qlora.linear_bwd_group([_bwd_member(dY=torch.zeros(4, 24, dtype=torch.bfloat16))])
    with pytest.raises(ValueError, match="T must be"):
        qlora.linear_bwd_group([_bwd_member(T=torch.zeros(4, 8, dtype=torch.bfloat16))])
    with pytest.raises(ValueError, match="share the token count"):
        qlora.linear_bwd_group([_bwd_member(), _bwd_member(M=8)])


@pytest.mark.parametrize("name,bad", [
    ("dX", torch.zeros(4, 128, dtype=torch.bfloat16)),
    ("dL1", torch.zeros(64, 8, dtype=torch.float32)),     # grad_dtype is bf16
    ("dL2", torch.zeros(8, 24, dtype=torch.bfloat16)),
])
def test_bwd_group_outputs_are_checked(name, bad):
    with pytest.raises(ValueError, match=f"{name} must be"):
        qlora.linear_bwd_group([_bwd_member(**{name: bad})])


def test_bwd_group_outputs_may_not_overlap():
    a, b = _bwd_member(), _bwd_member()
    shared = torch.zeros(64, 8, dtype=torch.bfloat16)
    a["dL1"], b["dL1"] = shared, shared
    with pytest.raises(ValueError, match="overlaps"):
        qlora.linear_bwd_group([a, b])
    c = _bwd_member()
    c["dX"] = c["X"]                                        # an output on top of an input
    with pytest.raises(ValueError, match="overlaps"):
        qlora.linear_bwd_group([c])


def test_bwd_group_host_tensors_are_refused():
    with pytest.raises(ValueError, match="CUDA device"):
        qlora.linear_bwd_group([_bwd_member()])


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """Without libqlora.so the binding raises; it has no other way to compute."""
    from bit_nf4_quantized_02_b200 import _lib
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "libqlora.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        _lib.load()
    # public calls reach the loader and stop there
    with pytest.raises(RuntimeError, match="not built"):
        qlora.last_device_error()
    with pytest.raises(RuntimeError, match="not built"):
        qlora.profile_start(16)
