"""GPU parity of the grouped backward (several QLoRA linears whose output
gradients are available together, their rank-r products in two launches)
against the float64 oracle, member by member: every member's dX, dL1 and dL2
are what the oracle's backward of that linear gives (QLoRA §3, the paragraph
after Eq. 6: adapter gradients only, the input gradient through the weight
dequantized to bf16)."""

import numpy as np
import pytest
import torch

from oracle import qlora_linear
from parity import assert_close, bf16_to_np, oracle_bwd, oracle_quant, oracle_w_hat
from synth import inputs, workloads

pytestmark = pytest.mark.gpu

qlora = pytest.importorskip("bit_nf4_quantized_02_b200")

# A scaled-down decoder layer (hidden 192, MLP 320) in the order its backward
# meets the gradients: down first, then gate and up (on H), o, then q, k, v (on H).
LAYER_GROUPS = [[("down", 192, 320, "U")], [("gate", 320, 192, "H"), ("up", 320, 192, "H")],
                [("o", 192, 192, "A")], [("q", 192, 192, "H"), ("k", 192, 192, "H"), ("v", 192, 192, "H")]]


def _make(M, spec, r, seed, save_T=True):
    """Host and device members of a group; inputs named in `spec` are shared."""
    g = inputs.rng(seed)
    xs, host, dev = {}, [], []
    for name, N, K, src in spec:
        if src not in xs:
            X = inputs.normal_bf16(g, (M, K))
            xs[src] = (X, X.cuda())
        X, Xd = xs[src]
        rr = r if isinstance(r, int) else r[name]
        W = torch.from_numpy(inputs.weight_f32(g, N, K))
        L1, L2 = inputs.lora_factors(g, K, N, rr)
        dY = inputs.normal_bf16(g, (M, N))
        s = 16.0 / rr
        q = qlora.quantize_nf4_dq(W.cuda())
        L1d, L2d = L1.cuda(), L2.cuda()
        T = None
        if save_T is True or (save_T and name in save_T):
            _, T = qlora.linear_fwd(Xd, q, L1d, L2d, s)
        host.append((name, W, X, L1, L2, dY, s))
        dev.append({"dY": dY.cuda(), "X": Xd, "T": T, "q": q, "L1": L1d, "L2": L2d, "s": s})
    return host, dev


def _check(host, outs, grad_dtype=torch.bfloat16):
    for (name, W, X, L1, L2, dY, s), (dX, dL1, dL2) in zip(host, outs):
        w_hat = oracle_w_hat(oracle_quant(W))
        dX_ref, dL1_ref, dL2_ref = oracle_bwd(dY, X, w_hat, L1, L2, s)
        if dX is not None:
            assert_close(bf16_to_np(dX), dX_ref, f"{name} dX")
        assert dL1.dtype == grad_dtype and dL2.dtype == grad_dtype
        assert_close(dL1.float().cpu().numpy(), dL1_ref, f"{name} dL1")
        assert_close(dL2.float().cpu().numpy(), dL2_ref, f"{name} dL2")


@pytest.mark.parametrize("r", [16, 64])
@pytest.mark.parametrize("M", [1, 64, 129, 300, 1000])
def test_layer_backward_groups(M, r):
    """A layer's backward as its data flow groups it, on ranks that take the
    per-member dL1 (r = 16) and the shared-X dL1 (r = 64)."""
    for gi, spec in enumerate(LAYER_GROUPS):
        host, dev = _make(M, spec, r, 8000 + 10 * M + gi + r)
        outs = qlora.linear_bwd_group(dev)
        torch.cuda.synchronize()
        assert qlora.last_device_error() == 0
        _check(host, outs)


def test_mixed_ranks_and_recomputed_T():
    """Ranks that take the grouped kernel (8, 32, 64) next to ranks that do
    not (24, 136), some members without a saved T, fp32 gradients, ragged N
    and K, and members that share X next to one that does not."""
    M = 333
    spec = [("a", 72, 320, "P"), ("b", 520, 320, "P"), ("c", 264, 64, "Q"), ("d", 1032, 320, "P"),
            ("e", 8, 128, "R"), ("f", 136, 320, "P")]
    ranks = {"a": 8, "b": 32, "c": 64, "d": 24, "e": 136, "f": 32}
    host, dev = _make(M, spec, ranks, 8100, save_T={"a", "d", "f"})
    outs = qlora.linear_bwd_group(dev, grad_dtype=torch.float32)
    torch.cuda.synchronize()
    assert qlora.last_device_error() == 0
    _check(host, outs, torch.float32)


def test_skip_dx_and_single_member():
    """need_dX=False leaves dX alone; a group of one matches the single-linear call."""
    spec = [("q", 264, 192, "H")]
    host, dev = _make(200, spec, 64, 8200)
    outs = qlora.linear_bwd_group(dev, need_dX=False)
    torch.cuda.synchronize()
    assert outs[0][0] is None
    _check(host, outs)
    m = dev[0]
    dX, dL1, dL2 = qlora.linear_bwd(m["dY"], m["X"], m["T"], m["q"], m["L1"], m["L2"], m["s"])
    torch.cuda.synchronize()
    # the same launches on the same shapes: bit-identical
    assert torch.equal(dL1, outs[0][1]) and torch.equal(dL2, outs[0][2])


def test_reproducible():
    """Split reductions are summed in a fixed order: two runs give the same bits."""
    spec = LAYER_GROUPS[3]
    _, dev = _make(1000, spec, 64, 8300)
    a = [[t.clone() for t in o] for o in qlora.linear_bwd_group(dev)]
    b = qlora.linear_bwd_group(dev)
    torch.cuda.synchronize()
    for oa, ob in zip(a, b):
        for x, y in zip(oa, ob):
            assert torch.equal(x, y)


def test_no_tokens():
    spec = LAYER_GROUPS[1]
    _, dev = _make(4, spec, 64, 8400)
    for m in dev:
        m["dY"], m["X"], m["T"] = m["dY"][:0], m["X"][:0], m["T"][:0]
    outs = qlora.linear_bwd_group(dev)
    torch.cuda.synchronize()
    for dX, dL1, dL2 in outs:
        assert dX.shape[0] == 0
        assert not dL1.any() and not dL2.any()


@pytest.mark.slow
def test_llama7b_qkv_full_size_sampled():
    """q, k and v of a LLaMA-7B layer at 8192 tokens as one group, in the launch
    configuration the benchmark times: dX on 256 sampled token rows, dL1 and
    dL2 in full."""
    wl = workloads.LLAMA7B_LAYER
    M, r, s = wl.M, wl.r, wl.s
    g = inputs.rng(wl.seed + 77)
    X = inputs.normal_bf16(g, (M, 4096))
    Xd = X.cuda()
    host, dev = [], []
    for lin in wl.linears[:3]:
        N, K = lin.n_out, lin.k_in
        W = torch.from_numpy(inputs.weight_f32(g, N, K))
        L1, L2 = inputs.lora_factors(g, K, N, r)
        dY = inputs.normal_bf16(g, (M, N))
        q = qlora.quantize_nf4_dq(W.cuda())
        L1d, L2d = L1.cuda(), L2.cuda()
        _, T = qlora.linear_fwd(Xd, q, L1d, L2d, s)
        host.append((W, L1, L2, dY))
        dev.append({"dY": dY.cuda(), "X": Xd, "T": T, "q": q, "L1": L1d, "L2": L2d, "s": s})
    outs = qlora.linear_bwd_group(dev)
    torch.cuda.synchronize()
    assert qlora.last_device_error() == 0
    rows = np.sort(np.random.default_rng(0).choice(M, 256, replace=False))
    Xn = bf16_to_np(X)
    for (W, L1, L2, dY), (dX, dL1, dL2), lin in zip(host, outs, wl.linears[:3]):
        w_hat = oracle_w_hat(oracle_quant(W))
        dYn = bf16_to_np(dY)
        dX_ref = qlora_linear.backward_dx_rows(dYn[rows], w_hat, bf16_to_np(L1), bf16_to_np(L2), s)
        assert_close(bf16_to_np(dX)[rows], dX_ref, f"{lin.name} dX[rows]")
        dL1_ref, dL2_ref = qlora_linear.adapter_grads(dYn, Xn, bf16_to_np(L1), bf16_to_np(L2), s)
        assert_close(dL1.float().cpu().numpy(), dL1_ref, f"{lin.name} dL1")
        assert_close(dL2.float().cpu().numpy(), dL2_ref, f"{lin.name} dL2")


@pytest.mark.slow
def test_llama7b_layer_groups_full_size_sampled():
    """The training benchmark's launch configuration at full size: q, k, v,
    gate and up on the layer input as one grouped forward (one adapter launch
    over their L1 side by side), then gate and up as one grouped backward (its
    G and dL2 problems split across the grid).  Y on 64 sampled output
    features of every member, T in full; dX of gate and up on 256 sampled
    token rows, dL1 and dL2 in full."""
    from oracle import nf4dq
    wl = workloads.LLAMA7B_LAYER
    M, r, s = wl.M, wl.r, wl.s
    lins = {l.name: l for l in wl.linears}
    names = ("q", "k", "v", "gate", "up")
    g = inputs.rng(wl.seed + 91)
    H = inputs.normal_bf16(g, (M, lins["q"].k_in))
    Hd = H.cuda()
    host, dev = {}, {}
    for i, name in enumerate(names):
        N, K = lins[name].n_out, lins[name].k_in
        Wd = inputs.device_normal((N, K), inputs.WEIGHT_STD, wl.seed + 300 + 10 * i, "cuda")
        L1, L2 = inputs.lora_factors(inputs.rng(wl.seed + 301 + 10 * i), K, N, r)
        host[name] = (Wd, L1, L2)
        dev[name] = {"X": Hd, "q": qlora.quantize_nf4_dq(Wd), "L1": L1.cuda(), "L2": L2.cuda(), "s": s}
    outs = qlora.linear_fwd_group([dev[n] for n in names])
    torch.cuda.synchronize()
    assert qlora.last_device_error() == 0
    Hf = bf16_to_np(H).astype(np.float64)
    for name, (Y, T) in zip(names, outs):
        Wd, L1, L2 = host[name]
        N = Wd.shape[0]
        cols = np.sort(np.random.default_rng(N + len(name)).choice(N, 64, replace=False))
        w_rows = nf4dq.dequantize_rows(Wd.cpu().numpy(), cols)
        L1f, L2f = bf16_to_np(L1).astype(np.float64), bf16_to_np(L2).astype(np.float64)
        Y_ref, T_ref = qlora_linear.forward(Hf, w_rows, L1f, L2f[:, cols], s)
        assert_close(bf16_to_np(Y)[:, cols], Y_ref, f"{name} Y[:, sampled features]")
        assert_close(qlora.t_value(T).cpu().numpy(), T_ref, f"{name} T")
        dev[name]["T"] = T
    dys = {}
    for name in ("gate", "up"):
        dys[name] = inputs.normal_bf16(g, (M, lins[name].n_out))
        dev[name]["dY"] = dys[name].cuda()
    bouts = qlora.linear_bwd_group([dev["gate"], dev["up"]])
    torch.cuda.synchronize()
    assert qlora.last_device_error() == 0
    rows = np.sort(np.random.default_rng(3).choice(M, 256, replace=False))
    for name, (dX, dL1, dL2) in zip(("gate", "up"), bouts):
        Wd, L1, L2 = host[name]
        w_hat = oracle_w_hat(oracle_quant(Wd.cpu()))
        dYn = bf16_to_np(dys[name])
        dX_ref = qlora_linear.backward_dx_rows(dYn[rows], w_hat, bf16_to_np(L1), bf16_to_np(L2), s)
        assert_close(bf16_to_np(dX)[rows], dX_ref, f"{name} dX[rows]")
        dL1_ref, dL2_ref = qlora_linear.adapter_grads(dYn, Hf, bf16_to_np(L1), bf16_to_np(L2), s)
        assert_close(dL1.float().cpu().numpy(), dL1_ref, f"{name} dL1")
        assert_close(dL2.float().cpu().numpy(), dL2_ref, f"{name} dL2")
