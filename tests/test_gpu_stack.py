"""GPU parity of the decoder-layer stack (seven QLoRA linears per layer, run
forward then backward in sequence), layer by layer against the oracle.

Each layer is checked on the GPU's own inputs to it ("teacher forcing"): the
outputs U = up(H) and D = down(U), every linear's saved T, the propagated
gradients dU and dH, and every adapter gradient, against the float64
oracle; the residual add and the gradient sum bit for bit against the
oracle's wiring definitions.
"""

import numpy as np
import pytest
import torch

from oracle import nf4dq, qlora_linear
from oracle import stack as ostack
from parity import assert_close, bf16_to_np, check_linear_sampled, pow2_unit, sample_idx
from synth import inputs, workloads

pytestmark = pytest.mark.gpu

qlora = pytest.importorskip("bit_nf4_quantized_02_b200")
from bit_nf4_quantized_02_b200 import stack as qstack  # noqa: E402


def _make(device):
    return lambda shape, std, seed, dtype: inputs.device_normal(shape, std, seed, device, dtype)


def _t_value(T):
    r = T.shape[1] // 2
    return (T[:, :r].float() + T[:, r:].float()).cpu().numpy()


def _check_layer_full(st, l):
    """Every output of layer l, in full (small shapes), in the units of its inputs."""
    row, s = st.lin[l], st.s
    H, U, D = bf16_to_np(st.H[l]), bf16_to_np(st.U[l]), bf16_to_np(st.D[l])
    uh, uu, ud, udu = (pow2_unit(t) for t in (st.H[l], st.U[l], st.dH[l + 1], st.dU[l]))
    w = {name: nf4dq.dequantize(nf4dq.quantize_nf4_dq(x.W.cpu().numpy())) for name, x in row.items()}
    L = {name: (bf16_to_np(x.L1), bf16_to_np(x.L2)) for name, x in row.items()}
    for name in qstack.READS_H:
        Y_ref, T_ref = qlora_linear.forward(H, w[name], *L[name], s)
        assert_close(_t_value(row[name].T), T_ref, f"L{l} {name} T", unit=uh)
        if name == "up":
            assert_close(U, Y_ref, f"L{l} U", unit=uh)
    D_ref, T_ref = qlora_linear.forward(U, w["down"], *L["down"], s)
    assert_close(D, D_ref, f"L{l} D", unit=uu)
    assert_close(_t_value(row["down"].T), T_ref, f"L{l} down T", unit=uu)
    np.testing.assert_array_equal(bf16_to_np(st.H[l + 1]), ostack.next_input(D, bf16_to_np(st.R[l])))
    dD = bf16_to_np(st.dH[l + 1])
    dU_ref, dL1_ref, dL2_ref = qlora_linear.backward(dD, U, w["down"], *L["down"], s)
    assert_close(bf16_to_np(st.dU[l]), dU_ref, f"L{l} dU", unit=ud)
    assert_close(row["down"].dL1.float().cpu().numpy(), dL1_ref, f"L{l} down dL1", unit=ud * uu)
    assert_close(row["down"].dL2.float().cpu().numpy(), dL2_ref, f"L{l} down dL2", unit=ud * uu)
    dU = bf16_to_np(st.dU[l])
    dH_ref = 0.0
    for name in qstack.READS_H:
        dY = dU if name == "up" else bf16_to_np(row[name].dY)
        uy = udu if name == "up" else 1.0
        dX_ref, dL1_ref, dL2_ref = qlora_linear.backward(dY, H, w[name], *L[name], s)
        dH_ref = dH_ref + dX_ref
        assert_close(row[name].dL1.float().cpu().numpy(), dL1_ref, f"L{l} {name} dL1", unit=uy * uh)
        assert_close(row[name].dL2.float().cpu().numpy(), dL2_ref, f"L{l} {name} dL2", unit=uy * uh)
    assert_close(bf16_to_np(st.dH[l]), dH_ref, f"L{l} dH", unit=udu)


@pytest.mark.parametrize("M", [200, 24])     # 24 tokens: the few-token forward
def test_small_stack_layer_by_layer(M):
    dev = torch.device("cuda")
    st = qstack.QLoRAStack(qlora, hidden=192, mlp=320, layers=3, M=M, r=16, alpha=16.0, seed=4321 + M,
                           device=dev, make=_make(dev))
    st.step()
    torch.cuda.synchronize()
    assert qlora.last_device_error() == 0
    for l in range(st.layers):
        _check_layer_full(st, l)


@pytest.mark.slow
def test_llama33b_stack_full_size_sampled():
    """The LLaMA-33B eight-layer stack at 4x2048 tokens: the first and last
    layers checked on sampled outputs (every adapter gradient in full), the
    wiring of every layer bit for bit."""
    wl = workloads.LLAMA33B_STACK
    hidden, mlp = wl.linears[0].n_out, wl.linears[4].n_out
    dev = torch.device("cuda")
    st = qstack.QLoRAStack(qlora, hidden=hidden, mlp=mlp, layers=wl.layers, M=wl.M, r=wl.r, alpha=wl.alpha,
                           seed=wl.seed, device=dev, make=_make(dev))
    st.step()
    torch.cuda.synchronize()
    assert qlora.last_device_error() == 0
    for l in range(st.layers):
        np.testing.assert_array_equal(bf16_to_np(st.H[l + 1]),
                                      ostack.next_input(bf16_to_np(st.D[l]), bf16_to_np(st.R[l])))
    s = st.s
    for l in (0, st.layers - 1):
        row = st.lin[l]
        rows = sample_idx(st.M, 256, l)
        rows_d = torch.as_tensor(rows, device=dev)
        H, U = st.H[l], st.U[l]
        # down: X = U, dY = dH[l+1]; up: X = H, dY = dU; the rest: X = H, seeded dY.
        # Discarded outputs (q, k, v, o, gate Y) are not kept: check their T and gradients.
        d = row["down"]
        check_linear_sampled(d.W.cpu().numpy(), U, st.dH[l + 1], d.L1, d.L2, s, st.D[l], d.T, st.dU[l],
                             d.dL1, d.dL2, tag=f"L{l} down ", seed=10 * l)
        u = row["up"]
        check_linear_sampled(u.W.cpu().numpy(), H, st.dU[l], u.L1, u.L2, s, U, u.T, None,
                             u.dL1, u.dL2, tag=f"L{l} up ", seed=10 * l + 1)
        # dH on sampled rows x columns: sum of the six dX through the columns of each weight.
        xcols = sample_idx(hidden, 256, 10 * l + 2)
        uh, udu = pow2_unit(H), pow2_unit(st.dU[l])
        dH_ref = 0.0
        for name in qstack.READS_H:
            x = row[name]
            dY = st.dU[l] if name == "up" else x.dY
            w_c = nf4dq.dequantize_cols(x.W.cpu().numpy(), xcols)
            dH_ref = dH_ref + qlora_linear.backward_dx_rows(bf16_to_np(dY[rows_d]), w_c, bf16_to_np(x.L1)[xcols],
                                                            bf16_to_np(x.L2), s)
            if name not in ("up",):
                dL1_ref, dL2_ref = qlora_linear.adapter_grads(bf16_to_np(dY), bf16_to_np(H), bf16_to_np(x.L1),
                                                              bf16_to_np(x.L2), s)
                assert_close(x.dL1.float().cpu().numpy(), dL1_ref, f"L{l} {name} dL1", unit=uh)
                assert_close(x.dL2.float().cpu().numpy(), dL2_ref, f"L{l} {name} dL2", unit=uh)
                T_ref = s * (bf16_to_np(H[rows_d]).astype(np.float64) @ bf16_to_np(x.L1).astype(np.float64))
                assert_close(_t_value(x.T)[rows], T_ref, f"L{l} {name} T[rows]", unit=uh)
        assert_close(bf16_to_np(st.dH[l])[rows][:, xcols], dH_ref, f"L{l} dH[rows, cols]", unit=udu)
