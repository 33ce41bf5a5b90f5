"""The C-ABI library loads, exports every entry point declared in
include/qlora.h, and rejects bad arguments on the host (no GPU needed)."""

import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "qlora.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(qlora_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from bit_nf4_quantized_02_b200 import _lib, build
    build.build()
    return _lib.load()


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("qlora_quantize_nf4_dq", "qlora_dequant", "qlora_linear_fwd", "qlora_linear_bwd"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_binding_covers_every_declared_symbol():
    from bit_nf4_quantized_02_b200 import _lib
    assert set(declared_functions()) <= set(_lib.SIGNATURES)


def test_exported_symbols_are_only_the_c_abi(lib):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", lib._name], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert exported == set(declared_functions())


def test_status_strings_and_version(lib):
    assert lib.qlora_version() >= 100
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert lib.qlora_status_str(code)


def test_host_argument_validation(lib):
    from bit_nf4_quantized_02_b200 import _lib
    # bad dtype / negative sizes are rejected before any CUDA call
    assert lib.qlora_quantize_nf4_dq(None, 7, 4, 64, None, None, None, None, None, 0, None) == _lib.QLORA_ERR_INVALID_ARG
    assert lib.qlora_quantize_nf4_dq(None, 0, -1, 64, None, None, None, None, None, 0, None) == _lib.QLORA_ERR_INVALID_ARG
    # a weight view with missing buffers
    w = _lib.NF4DQ(8, 64, None, None, None, None)
    assert lib.qlora_dequant(ctypes.byref(w), None, None) == _lib.QLORA_ERR_INVALID_ARG
    # shape rules of the linear: K % 64, N % 8, r % 8, r <= 256
    fake = 1 << 20  # aligned non-null placeholders: validation fails before any use
    for n_out, k_in, r, want in ((8, 60, 8, _lib.QLORA_ERR_UNSUPPORTED_SHAPE),
                                 (12, 64, 8, _lib.QLORA_ERR_UNSUPPORTED_SHAPE),
                                 (8, 64, 12, _lib.QLORA_ERR_UNSUPPORTED_SHAPE),
                                 (8, 64, 264, _lib.QLORA_ERR_UNSUPPORTED_SHAPE),
                                 (8, 64, 0, _lib.QLORA_ERR_INVALID_ARG)):
        wq = _lib.NF4DQ(n_out, k_in, fake, fake, fake, fake)
        rc = lib.qlora_linear_fwd(fake, 4, ctypes.byref(wq), fake, fake, r, 1.0, fake, None, fake, 1 << 30, None)
        assert rc == want, (n_out, k_in, r, rc)
    # misaligned weight buffers
    wq = _lib.NF4DQ(8, 64, fake + 4, fake, fake, fake)
    assert lib.qlora_linear_fwd(fake, 4, ctypes.byref(wq), fake, fake, 8, 1.0, fake, None, fake, 1 << 30,
                                None) == _lib.QLORA_ERR_MISALIGNED


def test_workspace_sizes_are_host_only(lib):
    # degenerate sizes never divide by zero
    assert lib.qlora_linear_fwd_workspace_size(0, 64, 128, 8) >= 0
    assert lib.qlora_linear_bwd_workspace_size(0, 64, 128, 8) >= 0
    assert lib.qlora_linear_fwd_workspace_size(1, 8, 64, 8) > 0
    assert lib.qlora_quantize_workspace_size(1 << 20) >= (1 << 20) // 64 * 4
    assert lib.qlora_linear_fwd_workspace_size(8192, 4096, 4096, 64) >= 4096 * 4096 * 2
    assert lib.qlora_linear_bwd_workspace_size(8192, 4096, 4096, 64) >= 4096 * 4096 * 2 + 2 * 8192 * 64 * 2


def test_group_forward_host_rules(lib):
    from bit_nf4_quantized_02_b200 import _lib
    fake = 1 << 20
    # an empty group does nothing; a NULL array or more than QLORA_MAX_GROUP members is refused
    assert lib.qlora_linear_fwd_group(None, 0, 8, None, 0, None) == _lib.QLORA_OK
    assert lib.qlora_linear_fwd_group(None, 1, 8, None, 0, None) == _lib.QLORA_ERR_INVALID_ARG
    big = (_lib.FwdMember * (_lib.QLORA_MAX_GROUP + 1))()
    assert lib.qlora_linear_fwd_group(big, _lib.QLORA_MAX_GROUP + 1, 8, None, 0, None) == _lib.QLORA_ERR_INVALID_ARG
    assert lib.qlora_linear_fwd_group_workspace_size(big, _lib.QLORA_MAX_GROUP + 1, 8) == 0
    # a member breaking a shape rule fails the whole group before anything runs
    good = _lib.NF4DQ(192, 192, fake, fake, fake, fake)
    bad = _lib.NF4DQ(192, 100, fake, fake, fake, fake)
    arr = (_lib.FwdMember * 2)(_lib.FwdMember(fake, ctypes.pointer(good), fake, fake, 16, 1.0, fake, None),
                               _lib.FwdMember(fake, ctypes.pointer(bad), fake, fake, 16, 1.0, fake, None))
    assert lib.qlora_linear_fwd_group(arr, 2, 8, fake, 1 << 30, None) == _lib.QLORA_ERR_UNSUPPORTED_SHAPE


def test_group_workspace_sizes(lib):
    from bit_nf4_quantized_02_b200 import _lib
    fake = 1 << 20
    shapes = [(192, 192, 16), (320, 192, 16), (192, 320, 8), (72, 320, 8)]
    views = [_lib.NF4DQ(n, k, fake, fake, fake, fake) for n, k, _ in shapes]
    arr = (_lib.FwdMember * len(shapes))(*[_lib.FwdMember(fake, ctypes.pointer(v), fake, fake, r, 1.0, fake, None)
                                           for v, (_, _, r) in zip(views, shapes)])
    for M in (1, 16, 128, 129, 4096):
        # a group of one needs what the single call needs
        for i, (n, k, r) in enumerate(shapes):
            one = (_lib.FwdMember * 1)(arr[i])
            assert lib.qlora_linear_fwd_group_workspace_size(one, 1, M) == lib.qlora_linear_fwd_workspace_size(M, n, k, r)
        total = lib.qlora_linear_fwd_group_workspace_size(arr, len(shapes), M)
        singles = [lib.qlora_linear_fwd_workspace_size(M, n, k, r) for n, k, r in shapes]
        if M <= 128:
            # few tokens: every member keeps its own fp32 accumulators [M x (N + r)]
            assert total >= sum(M * (n + r) * 4 for n, _, r in shapes)
            assert total <= sum(singles)
        else:
            # many tokens: one bf16 weight buffer reused member after member and
            # every member's T pair (the adapter products of a set run as one
            # launch of the rank kernel, whose split partials come on top)
            assert total >= max(n * k * 2 for n, k, _ in shapes) + sum(M * 2 * r * 2 for _, _, r in shapes)
            assert total <= sum(singles) + sum(M * 2 * r * 2 for _, _, r in shapes)


def test_group_shared_input_workspace(lib):
    """Many tokens: members that read the same X (same pointer and K) with equal
    ranks of 64 or 128 share one adapter product over L1_cat [K x sum r], which
    the workspace then holds; members with distinct inputs need no such space."""
    from bit_nf4_quantized_02_b200 import _lib
    fake = 1 << 20
    M, N, K, r = 4096, 512, 1024, 64
    view = _lib.NF4DQ(N, K, fake, fake, fake, fake)

    def size(xs):
        arr = (_lib.FwdMember * len(xs))(*[_lib.FwdMember(x, ctypes.pointer(view), fake, fake, r, 1.0, fake, None)
                                           for x in xs])
        return lib.qlora_linear_fwd_group_workspace_size(arr, len(xs), M)

    base = N * K * 2 + 3 * M * 2 * r * 2     # the bf16 weight buffer and the three T pairs
    distinct = size([fake, fake * 2, fake * 3])
    shared = size([fake, fake, fake])
    assert distinct >= base
    assert shared >= base + K * 3 * r * 2
    # one shared pair and one single member: the pair's L1_cat
    assert size([fake, fake * 2, fake]) >= base + K * 2 * r * 2
