"""GPU parity of the grouped forward (several QLoRA linears on the same tokens
in one call; at <= 128 tokens one launch chain over all of them) against the
float64 oracle, member by member: every member's Y and T are what the oracle's
forward of that linear gives (QLoRA §2 Eq. 3, §3 Eq. 5)."""

import ctypes

import numpy as np
import pytest
import torch

from oracle import nf4dq, qlora_linear
from parity import assert_close, bf16_to_np, oracle_fwd
from synth import inputs, workloads

pytestmark = pytest.mark.gpu

qlora = pytest.importorskip("bit_nf4_quantized_02_b200")
from bit_nf4_quantized_02_b200 import _lib  # noqa: E402

# A scaled-down decoder layer (hidden 192, MLP 320): q, k, v, gate and up read
# the layer input H, o reads A, down reads U; r = 16.
LAYER = [("q", 192, 192, "H"), ("k", 192, 192, "H"), ("v", 192, 192, "H"), ("o", 192, 192, "A"),
         ("gate", 320, 192, "H"), ("up", 320, 192, "H"), ("down", 192, 320, "U")]
# Ragged shapes and ranks: N not a multiple of the 64/128-row tiles, K not a
# multiple of the 512-wide unit, mixed r (each reads its own input).
RAGGED = [("a", 72, 320, 8), ("b", 520, 1088, 64), ("c", 264, 64, 16), ("d", 1032, 2048, 136), ("e", 8, 128, 8)]


def _layer_members(M, seed, tables=None):
    g = inputs.rng(seed)
    xs = {"H": inputs.normal_bf16(g, (M, 192)), "A": inputs.normal_bf16(g, (M, 192)),
          "U": inputs.normal_bf16(g, (M, 320))}
    host, dev = [], []
    xd = {k: v.cuda() for k, v in xs.items()}
    for i, (name, N, K, src) in enumerate(LAYER):
        W = torch.from_numpy(inputs.weight_f32(g, N, K))
        L1, L2 = inputs.lora_factors(g, K, N, 16)
        table = tables[i] if tables else "nf4"
        host.append((name, W, xs[src], L1, L2, table))
        dev.append({"X": xd[src], "q": qlora.quantize_nf4_dq(W.cuda(), table=table), "L1": L1.cuda(),
                    "L2": L2.cuda(), "s": 1.0})
    return host, dev


def _check(host, outs, s_of=lambda i: 1.0):
    for i, ((name, W, X, L1, L2, table), (Y, T)) in enumerate(zip(host, outs)):
        oq = nf4dq.quantize_nf4_dq(W.numpy(), levels=nf4dq.TABLES[table])
        w_hat = nf4dq.dequantize(oq)
        Y_ref, T_ref = oracle_fwd(X, w_hat, L1, L2, s_of(i))
        assert_close(bf16_to_np(Y), Y_ref, f"{name} Y")
        if T is not None:
            assert_close(qlora.t_value(T).cpu().numpy(), T_ref, f"{name} T")


@pytest.mark.parametrize("M", [1, 7, 8, 9, 16, 29, 32, 33, 64, 65, 100, 128, 200])
def test_layer_group_parity(M):
    """The seven projections of a layer as one group, on every token-count path."""
    host, dev = _layer_members(M, 7000 + M)
    outs = qlora.linear_fwd_group(dev)
    torch.cuda.synchronize()
    assert qlora.last_device_error() == 0
    _check(host, outs)


@pytest.mark.parametrize("M", [1, 16, 32, 64, 128])
def test_ragged_group_parity(M):
    """Members of unrelated shapes and ranks, each with its own input and scale."""
    g = inputs.rng(7100 + M)
    host, dev = [], []
    for name, N, K, r in RAGGED:
        W = torch.from_numpy(inputs.weight_f32(g, N, K))
        X = inputs.normal_bf16(g, (M, K))
        L1, L2 = inputs.lora_factors(g, K, N, r)
        host.append((name, W, X, L1, L2, "nf4"))
        dev.append({"X": X.cuda(), "q": qlora.quantize_nf4_dq(W.cuda()), "L1": L1.cuda(), "L2": L2.cuda(),
                    "s": 16.0 / r})
    outs = qlora.linear_fwd_group(dev)
    torch.cuda.synchronize()
    assert qlora.last_device_error() == 0
    _check(host, outs, s_of=lambda i: 16.0 / RAGGED[i][3])


@pytest.mark.parametrize("M", [4, 24, 100])
def test_mixed_code_tables(M):
    """NF4 and FP4 members in one group: one chain per table, each decoding its own levels."""
    tables = ["nf4", "fp4", "nf4", "fp4", "fp4", "nf4", "fp4"]
    host, dev = _layer_members(M, 7200 + M, tables)
    outs = qlora.linear_fwd_group(dev)
    torch.cuda.synchronize()
    assert qlora.last_device_error() == 0
    _check(host, outs)


def test_group_without_T_and_preallocated_outputs():
    M = 12
    host, dev = _layer_members(M, 7300)
    for m, (name, W, X, L1, L2, _) in zip(dev, host):
        m["Y"] = torch.full((M, W.shape[0]), float("nan"), dtype=torch.bfloat16, device="cuda")
    outs = qlora.linear_fwd_group(dev, save_T=False)
    torch.cuda.synchronize()
    for m, (Y, T) in zip(dev, outs):
        assert T is None and Y.data_ptr() == m["Y"].data_ptr()
    _check(host, outs)


def test_repeated_group_calls_reuse_workspace():
    """Back-to-back groups on one workspace (the zero region is re-cleared)."""
    M = 16
    host, dev = _layer_members(M, 7400)
    runs = [qlora.linear_fwd_group(dev) for _ in range(3)]
    torch.cuda.synchronize()
    for outs in runs:
        _check(host, outs)


def test_prepared_group_follows_its_inputs():
    """A FwdGroup marshalled once and run again after its inputs were
    overwritten in place computes the new inputs' forward."""
    M = 16
    host, dev = _layer_members(M, 7700)
    grp = qlora.FwdGroup(dev)
    grp()
    torch.cuda.synchronize()
    _check(host, grp.outputs)
    g = inputs.rng(7701)
    done = set()
    for m in dev:                          # H is shared by five members: overwrite it once
        if m["X"].data_ptr() not in done:
            done.add(m["X"].data_ptr())
            m["X"].copy_(inputs.normal_bf16(g, tuple(m["X"].shape)).cuda())
    new_host = [(name, W, m["X"].cpu(), L1, L2, t) for m, (name, W, X, L1, L2, t) in zip(dev, host)]
    grp()
    torch.cuda.synchronize()
    _check(new_host, grp.outputs)


def test_single_member_group_matches_linear_fwd_path():
    """A group of one is the single-linear call (same kernels, same work split)."""
    M = 16
    host, dev = _layer_members(M, 7500)
    (Yg, Tg), = qlora.linear_fwd_group(dev[:1])
    Y1, T1 = qlora.linear_fwd(dev[0]["X"], dev[0]["q"], dev[0]["L1"], dev[0]["L2"], 1.0)
    torch.cuda.synchronize()
    _check(host[:1], [(Yg, Tg)])
    # both sum split-K partials in an order set by CTA timing: equal to rounding
    assert (Yg.float() - Y1.float()).abs().max().item() <= 2e-2 * (Y1.float().abs().max().item() + 1)


def test_group_host_errors():
    lib = _lib.load()
    host, dev = _layer_members(8, 7600)
    assert lib.qlora_linear_fwd_group(None, 0, 8, None, 0, None) == _lib.QLORA_OK
    assert lib.qlora_linear_fwd_group(None, 1, 8, None, 0, None) == _lib.QLORA_ERR_INVALID_ARG
    arr = (_lib.FwdMember * 9)()
    assert lib.qlora_linear_fwd_group(arr, 9, 8, None, 0, None) == _lib.QLORA_ERR_INVALID_ARG
    # a workspace one byte short is refused before anything is enqueued
    w = dev[0]["q"].as_struct()
    m = _lib.FwdMember(dev[0]["X"].data_ptr(), ctypes.pointer(w), dev[0]["L1"].data_ptr(), dev[0]["L2"].data_ptr(),
                       16, 1.0, torch.empty(8, 192, dtype=torch.bfloat16, device="cuda").data_ptr(), None)
    one = (_lib.FwdMember * 1)(m)
    need = lib.qlora_linear_fwd_group_workspace_size(one, 1, 8)
    assert need == lib.qlora_linear_fwd_workspace_size(8, 192, 192, 16)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    assert lib.qlora_linear_fwd_group(one, 1, 8, ws.data_ptr(), need - 1, None) == _lib.QLORA_ERR_WORKSPACE
    assert lib.qlora_linear_fwd_group(one, 1, 8, ws.data_ptr(), need, None) == _lib.QLORA_OK
    torch.cuda.synchronize()


@pytest.mark.slow
def test_llama65b_layer_group_16_tokens_sampled():
    """The seven LLaMA-65B projections at 16 tokens as one group, in the launch
    configuration the decode benchmark times: each member's Y checked on 64
    sampled output features (the oracle dequantizes just those weight rows),
    all tokens, and its T in full."""
    wl = workloads.LLAMA65B_LAYER
    M, r, s = wl.extra["M_decode"], wl.r, wl.s
    g = inputs.rng(wl.seed + 77)
    xs = {"H": inputs.normal_bf16(g, (M, 8192)), "A": inputs.normal_bf16(g, (M, 8192)),
          "U": inputs.normal_bf16(g, (M, 22016))}
    src = {"q": "H", "k": "H", "v": "H", "o": "A", "gate": "H", "up": "H", "down": "U"}
    xd = {k: v.cuda() for k, v in xs.items()}
    dev, host = [], []
    for i, lin in enumerate(wl.linears):
        N, K = lin.n_out, lin.k_in
        Wd = inputs.device_normal((N, K), inputs.WEIGHT_STD, wl.seed + 100 * i, "cuda")
        L1, L2 = inputs.lora_factors(inputs.rng(wl.seed + 100 * i + 1), K, N, r)
        dev.append({"X": xd[src[lin.name]], "q": qlora.quantize_nf4_dq(Wd), "L1": L1.cuda(), "L2": L2.cuda(),
                    "s": s})
        host.append((lin.name, Wd, xs[src[lin.name]], L1, L2))
    outs = qlora.linear_fwd_group(dev)
    torch.cuda.synchronize()
    assert qlora.last_device_error() == 0
    for (name, Wd, X, L1, L2), (Y, T) in zip(host, outs):
        N = Wd.shape[0]
        rows = np.sort(np.random.default_rng(N).choice(N, 64, replace=False))
        w_rows = nf4dq.dequantize_rows(Wd.cpu().numpy(), rows)
        Xf, L1f, L2f = (bf16_to_np(t).astype(np.float64) for t in (X, L1, L2))
        Y_ref, T_ref = qlora_linear.forward(Xf, w_rows, L1f, L2f[:, rows], s)
        assert_close(bf16_to_np(Y)[:, rows], Y_ref, f"{name} Y[:, sampled features]")
        assert_close(qlora.t_value(T).cpu().numpy(), T_ref, f"{name} T")


@pytest.mark.parametrize("M", [129, 300])
def test_shared_input_sets_many_tokens(M):
    """Many tokens: members reading the same X share one adapter product, split
    into each member's T with its own rank and scale; an unshared member and a
    member without a saved T ride along."""
    g = inputs.rng(7800 + M)
    K1, K2 = 320, 192
    Xa, Xb = inputs.normal_bf16(g, (M, K1)), inputs.normal_bf16(g, (M, K2))
    spec = [("a0", Xa, 72, 8, 2.0), ("b0", Xb, 264, 16, 1.0), ("a1", Xa, 520, 64, 0.25),
            ("a2", Xa, 136, 136, 0.5), ("b1", Xb, 64, 32, 1.5)]
    xd = {id(Xa): Xa.cuda(), id(Xb): Xb.cuda()}
    host, dev = [], []
    for name, X, N, r, s in spec:
        K = X.shape[1]
        W = torch.from_numpy(inputs.weight_f32(g, N, K))
        L1, L2 = inputs.lora_factors(g, K, N, r)
        host.append((name, W, X, L1, L2, "nf4"))
        m = {"X": xd[id(X)], "q": qlora.quantize_nf4_dq(W.cuda()), "L1": L1.cuda(), "L2": L2.cuda(), "s": s}
        dev.append(m)
    outs = qlora.linear_fwd_group(dev)
    torch.cuda.synchronize()
    assert qlora.last_device_error() == 0
    _check(host, outs, s_of=lambda i: spec[i][4])
    # without saved T (the pairs live in the workspace); Y unchanged up to rounding order
    outs2 = qlora.linear_fwd_group(dev, save_T=False)
    torch.cuda.synchronize()
    _check(host, outs2, s_of=lambda i: spec[i][4])


def test_layer_group_mid_size_full_check():
    """A LLaMA-proportioned layer (hidden 1024, MLP 2816, r 64) at 1024 tokens,
    grouped as a layer's data flow groups it, checked in full."""
    M, hid, mlp, r, s = 1024, 1024, 2816, 64, 0.25
    g = inputs.rng(7900)
    xs = {"H": inputs.normal_bf16(g, (M, hid)), "A": inputs.normal_bf16(g, (M, hid)),
          "U": inputs.normal_bf16(g, (M, mlp))}
    shapes = [("q", hid, hid, "H"), ("k", hid, hid, "H"), ("v", hid, hid, "H"), ("o", hid, hid, "A"),
              ("gate", mlp, hid, "H"), ("up", mlp, hid, "H"), ("down", hid, mlp, "U")]
    xd = {k: v.cuda() for k, v in xs.items()}
    host, dev = {}, {}
    for name, N, K, src in shapes:
        W = torch.from_numpy(inputs.weight_f32(g, N, K))
        L1, L2 = inputs.lora_factors(g, K, N, r)
        host[name] = (name, W, xs[src], L1, L2, "nf4")
        dev[name] = {"X": xd[src], "q": qlora.quantize_nf4_dq(W.cuda()), "L1": L1.cuda(), "L2": L2.cuda(), "s": s}
    groups = [["q", "k", "v", "gate", "up"], ["o"], ["down"]]
    for grp in groups:
        outs = qlora.linear_fwd_group([dev[n] for n in grp])
        torch.cuda.synchronize()
        assert qlora.last_device_error() == 0
        _check([host[n] for n in grp], outs, s_of=lambda i: s)


@pytest.mark.parametrize("r", [64, 128])
def test_shared_input_equal_ranks_many_tokens(r):
    """Many tokens, members on one input with equal ranks of 64 or 128: one
    adapter product whose n-tile k is member k's L1, each T scaled on its own."""
    M, K = 300, 320
    g = inputs.rng(7950 + r)
    X = inputs.normal_bf16(g, (M, K))
    Xd = X.cuda()
    host, dev = [], []
    scales = [0.5, 1.0, 2.0]
    for i, N in enumerate((136, 264, 72)):
        W = torch.from_numpy(inputs.weight_f32(g, N, K))
        L1, L2 = inputs.lora_factors(g, K, N, r)
        host.append((f"m{i}", W, X, L1, L2, "nf4"))
        dev.append({"X": Xd, "q": qlora.quantize_nf4_dq(W.cuda()), "L1": L1.cuda(), "L2": L2.cuda(), "s": scales[i]})
    outs = qlora.linear_fwd_group(dev)
    torch.cuda.synchronize()
    assert qlora.last_device_error() == 0
    _check(host, outs, s_of=lambda i: scales[i])
