"""B200-native QLoRA: NF4 + Double Quantization storage and the QLoRA linear layer.

Python face of libqlora.so (include/qlora.h).  PyTorch provides device
memory and streams only; every step of the quantizer, doubleDequant and the
linear forward/backward runs in the library's sm_100a kernels.  The functions
here allocate outputs and workspaces with torch and pass raw pointers through
the C ABI.  There is no CPU or PyTorch fallback: without a CUDA device or the
built library the calls raise.

Paper: "QLoRA: Efficient Finetuning of Quantized LLMs"
(aiingo.vercel.app/paper/paper-2305-14314), §2 Eqs. 1-3, §3 Eqs. 4-6,
Appendix E.
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import QLoRAError  # noqa: F401

__all__ = [
    "NF4Tensor",
    "quantize_nf4_dq",
    "dequant",
    "linear_fwd",
    "linear_fwd_group",
    "FwdGroup",
    "linear_bwd",
    "last_device_error",
    "t_value",
    "profile_start",
    "profile_stop",
    "QLoRAError",
]


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("qlora: tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("qlora: tensors must be contiguous")
    return t.data_ptr()


def _bits(t: torch.Tensor) -> torch.Tensor:
    if t.dtype != torch.bfloat16:
        raise TypeError(f"qlora: expected a bfloat16 tensor, got {t.dtype}")
    return t


def _check_out(t: torch.Tensor | None, shape, dtype, dev, name: str) -> None:
    """A caller-supplied output: exactly ``shape`` and ``dtype``, contiguous, on ``dev``.

    The kernels write the full extent the shapes imply, so a smaller buffer
    (or one of a narrower dtype) would be written past its end.
    """
    if t is None:
        return
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or t.device != dev or not t.is_contiguous():
        raise ValueError(f"qlora: {name} must be a contiguous {dtype} tensor of shape {tuple(shape)} on {dev}, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}")


def _check_device(dev, require_cuda: bool = True, **tensors) -> None:
    """Every tensor on the one device ``dev``, a CUDA device (a kernel given
    another GPU's memory would reach across devices)."""
    for name, t in tensors.items():
        if t is not None and t.device != dev:
            raise ValueError(f"qlora: {name} is on {t.device}, expected {dev} (all tensors of a call share a device)")
    if require_cuda and dev.type != "cuda":
        raise ValueError("qlora: tensors must live on a CUDA device")


def _span(t: torch.Tensor | None):
    if t is None or t.numel() == 0:
        return None
    return (t.data_ptr(), t.data_ptr() + t.numel() * t.element_size())


def _overlap(a, b) -> bool:
    return a is not None and b is not None and a[0] < b[1] and b[0] < a[1]


@dataclass
class NF4Tensor:
    """A weight in the QLoRA storage format (device buffers owned by torch).

    codes   uint8 [ceil(numel/2)]   NF4 codes, 2 per byte (even element low nibble)
    c2_fp8  uint8 [ceil(numel/64)]  E4M3 codes of the mean-centred block absmax
    c1      fp32  [ceil(nblk/256)]  second-level constants
    c2_mean fp32  [1]               mean of the first-level constants
    table   "nf4" (Appendix E levels) or "fp4" (E2M1, the 4-bit float of §4)
    """

    n_out: int
    k_in: int
    codes: torch.Tensor
    c2_fp8: torch.Tensor
    c1: torch.Tensor
    c2_mean: torch.Tensor
    table: str = "nf4"

    @property
    def shape(self):
        return (self.n_out, self.k_in)

    @property
    def device(self):
        return self.codes.device

    def as_struct(self) -> _lib.NF4DQ:
        return _lib.NF4DQ(self.n_out, self.k_in, _ptr(self.codes), _ptr(self.c2_fp8), _ptr(self.c1),
                          _ptr(self.c2_mean), _lib.TABLES[self.table])

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.codes, self.c2_fp8, self.c1, self.c2_mean))


def _empty_nf4(n_out: int, k_in: int, device) -> NF4Tensor:
    numel = n_out * k_in
    nblk = (numel + 63) // 64
    return NF4Tensor(
        n_out, k_in,
        torch.empty((numel + 1) // 2, dtype=torch.uint8, device=device),
        torch.empty(nblk, dtype=torch.uint8, device=device),
        torch.empty((nblk + 255) // 256, dtype=torch.float32, device=device),
        torch.empty(1, dtype=torch.float32, device=device),
    )


def quantize_nf4_dq(W: torch.Tensor, out: NF4Tensor | None = None, table: str = "nf4") -> NF4Tensor:
    """Quantize a 2-D fp32 or bf16 CUDA weight [n_out, k_in] to NF4 + DQ
    (``table="fp4"``: the FP4 E2M1 code table instead of NF4)."""
    lib = _lib.load()
    if W.dim() != 2:
        raise ValueError("qlora: W must be 2-D [n_out, k_in]")
    if W.dtype == torch.float32:
        wdt = _lib.QLORA_DTYPE_F32
    elif W.dtype == torch.bfloat16:
        wdt = _lib.QLORA_DTYPE_BF16
    else:
        raise TypeError("qlora: W must be float32 or bfloat16")
    n_out, k_in = W.shape
    if table not in _lib.TABLES:
        raise ValueError(f"qlora: unknown code table {table!r}")
    q = out if out is not None else _empty_nf4(n_out, k_in, W.device)
    q.table = table
    ws_bytes = lib.qlora_quantize_workspace_size(n_out * k_in)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=W.device)
    _lib.check(lib.qlora_quantize_4bit_dq(_ptr(W), wdt, n_out, k_in, _lib.TABLES[table], _ptr(q.codes),
                                          _ptr(q.c2_fp8), _ptr(q.c1), _ptr(q.c2_mean), _ptr(ws), ws_bytes,
                                          _stream(W.device)), "qlora_quantize_4bit_dq")
    return q


def dequant(q: NF4Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """doubleDequant (Eq. 6): the bf16 weight [n_out, k_in]."""
    _check_out(out, q.shape, torch.bfloat16, q.device, "out")
    _check_device(q.device, c2_fp8=q.c2_fp8, c1=q.c1, c2_mean=q.c2_mean)
    lib = _lib.load()
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    st = q.as_struct()
    _lib.check(lib.qlora_dequant(st, _ptr(_bits(out)), _stream(q.device)), "qlora_dequant")
    return out


class _Workspace:
    """Grow-only scratch buffers, one per (device, stream), reused across calls.

    Calls on one stream run in order, so they can share a buffer; a different
    stream gets its own.
    """

    def __init__(self):
        self.buf: dict = {}

    def get(self, nbytes: int, device) -> torch.Tensor:
        dev = torch.device(device)
        key = (dev, _stream(dev))
        b = self.buf.get(key)
        if b is None or b.numel() < nbytes:
            b = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
            self.buf[key] = b
        return b


_WS = _Workspace()


def _mask_arg(mask: torch.Tensor, M: int, K: int, dev) -> torch.Tensor:
    """Check a LoRA-dropout keep mask: int32/uint32 words [M, K/32] on ``dev``."""
    if mask.device != torch.device(dev) or mask.dtype not in (torch.int32, torch.uint32) or \
            tuple(mask.shape) != (M, K // 32) or not mask.is_contiguous():
        raise ValueError("qlora: dropout mask must be contiguous 32-bit words [M, K/32] on the device")
    return mask


def linear_fwd(X: torch.Tensor, q: NF4Tensor, L1: torch.Tensor, L2: torch.Tensor, s: float,
               save_T: bool = True, Y: torch.Tensor | None = None, T: torch.Tensor | None = None,
               dropout_mask: torch.Tensor | None = None, dropout_p: float = 0.0, Xm: torch.Tensor | None = None):
    """Y = X doubleDequant(W)^T + s X L1 L2 (Eq. 3 / Eq. 5).  Returns (Y, T or None).

    X [M, K] bf16, L1 [K, r] bf16, L2 [r, N] bf16.  T [M, 2r] bf16 holds
    T = s X L1 as a hi/lo pair: T ~= T[:, :r] + T[:, r:] (see ``t_value``).
    With ``dropout_mask`` (keep bits, 32-bit words [M, K/32], element 32 w + b
    in bit b of word w) LoRA dropout acts on the adapter input:
    T = s (X * m / (1 - dropout_p)) L1; ``Xm`` ([M, K] bf16, optional)
    receives the masked input X * m for the backward.
    """
    M, K = X.shape
    r = L1.shape[1]
    N = q.n_out
    if K != q.k_in or L1.shape[0] != K or tuple(L2.shape) != (r, N):
        raise ValueError("qlora: shape mismatch")
    dev = X.device
    _check_out(Y, (M, N), torch.bfloat16, dev, "Y")
    if save_T:
        _check_out(T, (M, 2 * r), torch.bfloat16, dev, "T")
    _check_out(Xm, (M, K), torch.bfloat16, dev, "Xm")
    _check_device(dev, L1=L1, L2=L2, codes=q.codes, c2_fp8=q.c2_fp8, c1=q.c1, c2_mean=q.c2_mean, mask=dropout_mask)
    lib = _lib.load()
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    if save_T and T is None:
        T = torch.empty((M, 2 * r), dtype=torch.bfloat16, device=dev)
    if dropout_mask is not None:
        _mask_arg(dropout_mask, M, K, dev)
        ws = _WS.get(lib.qlora_linear_fwd_dropout_workspace_size(M, N, K, r), dev)
        _lib.check(lib.qlora_linear_fwd_dropout(_ptr(_bits(X)), M, q.as_struct(), _ptr(_bits(L1)), _ptr(_bits(L2)), r,
                                                float(s), _ptr(dropout_mask), float(dropout_p), _ptr(_bits(Y)),
                                                _ptr(T) if save_T else None, _ptr(Xm), _ptr(ws), ws.numel(),
                                                _stream(dev)),
                   "qlora_linear_fwd_dropout")
        return Y, (T if save_T else None)
    ws_bytes = lib.qlora_linear_fwd_workspace_size(M, N, K, r)
    ws = _WS.get(ws_bytes, dev)
    _lib.check(lib.qlora_linear_fwd(_ptr(_bits(X)), M, q.as_struct(), _ptr(_bits(L1)), _ptr(_bits(L2)), r, float(s),
                                    _ptr(_bits(Y)), _ptr(T) if save_T else None, _ptr(ws), ws.numel(),
                                    _stream(dev)), "qlora_linear_fwd")
    return Y, (T if save_T else None)


class FwdGroup:
    """A grouped forward whose arguments are marshalled once (see
    ``linear_fwd_group``).  Calling it runs the group again on the same
    tensors, which it keeps alive; only the C call is made per run."""

    def __init__(self, members, save_T: bool = True):
        if not 0 < len(members) <= _lib.QLORA_MAX_GROUP:
            raise ValueError(f"qlora: a group holds 1..{_lib.QLORA_MAX_GROUP} linears")
        M = members[0]["X"].shape[0]
        dev = members[0]["X"].device
        # every argument is checked before the library is loaded or a pointer taken
        for m in members:
            X, q, L1, L2 = m["X"], m["q"], m["L1"], m["L2"]
            K, r, N = X.shape[1], L1.shape[1], q.n_out
            if X.shape[0] != M or X.device != dev:
                raise ValueError("qlora: the members of a group share the token count and the device")
            if K != q.k_in or L1.shape[0] != K or tuple(L2.shape) != (r, N):
                raise ValueError("qlora: shape mismatch")
            _check_out(m.get("Y"), (M, N), torch.bfloat16, dev, "Y")
            if save_T:
                _check_out(m.get("T"), (M, 2 * r), torch.bfloat16, dev, "T")
            _check_device(dev, False, L1=L1, L2=L2, codes=q.codes, c2_fp8=q.c2_fp8, c1=q.c1, c2_mean=q.c2_mean)
        # caller-supplied outputs may not overlap any member's input X or output
        outs = [(i, name, _span(m.get(name))) for i, m in enumerate(members)
                for name in (("Y", "T") if save_T else ("Y",))]
        for i, name, sp in outs:
            for j, m in enumerate(members):
                if _overlap(sp, _span(m["X"])):
                    raise ValueError(f"qlora: member {i}'s {name} overlaps member {j}'s X")
            for j, name2, sp2 in outs:
                if (i, name) < (j, name2) and _overlap(sp, sp2):
                    raise ValueError(f"qlora: member {i}'s {name} overlaps member {j}'s {name2}")
        _check_device(dev)
        lib = _lib.load()
        arr = (_lib.FwdMember * len(members))()
        self._keep, self.outputs = [], []
        for i, m in enumerate(members):
            X, q, L1, L2 = m["X"], m["q"], m["L1"], m["L2"]
            r, N = L1.shape[1], q.n_out
            Y = m.get("Y")
            if Y is None:
                Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            T = m.get("T")
            if save_T and T is None:
                T = torch.empty((M, 2 * r), dtype=torch.bfloat16, device=dev)
            w = q.as_struct()
            self._keep += [w, X, q, L1, L2]
            arr[i] = _lib.FwdMember(_ptr(_bits(X)), ctypes.pointer(w), _ptr(_bits(L1)), _ptr(_bits(L2)), r,
                                    float(m["s"]), _ptr(_bits(Y)), _ptr(T) if save_T else None)
            self.outputs.append((Y, T if save_T else None))
        self._arr, self._n, self._M, self._dev = arr, len(members), M, dev
        self._ws_bytes = lib.qlora_linear_fwd_group_workspace_size(arr, len(members), M)
        self._fn = lib.qlora_linear_fwd_group

    def __call__(self) -> list:
        ws = _WS.get(self._ws_bytes, self._dev)
        _lib.check(self._fn(self._arr, self._n, self._M, ws.data_ptr(), ws.numel(), _stream(self._dev)),
                   "qlora_linear_fwd_group")
        return self.outputs


def linear_fwd_group(members, save_T: bool = True) -> list:
    """The forward of several linears that see the same tokens, in one call.

    ``members``: a sequence of dicts with keys ``X`` [M, K_i], ``q``
    (NF4Tensor), ``L1`` [K_i, r_i], ``L2`` [r_i, N_i], ``s`` and optionally the
    outputs ``Y`` [M, N_i] and ``T`` [M, 2 r_i].  Every member computes what
    ``linear_fwd`` computes; with at most 128 tokens the whole group runs as
    one launch chain.  Returns [(Y, T or None)] in member order.  For repeated
    calls on the same tensors, ``FwdGroup(members)`` marshals the arguments
    once.
    """
    return FwdGroup(members, save_T)()


def t_value(T: torch.Tensor) -> torch.Tensor:
    """The fp32 value of a hi/lo pair T [M, 2r] saved by ``linear_fwd``."""
    r = T.shape[1] // 2
    return T[:, :r].float() + T[:, r:].float()


def linear_bwd(dY: torch.Tensor, X: torch.Tensor, T: torch.Tensor | None, q: NF4Tensor, L1: torch.Tensor,
               L2: torch.Tensor, s: float, need_dX: bool = True, grad_dtype=torch.bfloat16,
               dX: torch.Tensor | None = None, dL1: torch.Tensor | None = None, dL2: torch.Tensor | None = None,
               dropout_mask: torch.Tensor | None = None, dropout_p: float = 0.0, Xm: torch.Tensor | None = None):
    """Adapter-only backward.  Returns (dX or None, dL1 [K, r], dL2 [r, N]).

    With ``dropout_mask`` (the forward's mask) the adapter path goes through
    the mask: dX = dY W_hat + (G L1^T) m / (1 - p), dL1 = drop(X)^T G.
    ``Xm`` is the forward's masked input (recomputed from X and the mask if None).
    """
    M, N = dY.shape
    K = q.k_in
    r = L1.shape[1]
    if N != q.n_out or tuple(X.shape) != (M, K) or tuple(L2.shape) != (r, N) or L1.shape[0] != K:
        raise ValueError("qlora: shape mismatch")
    if grad_dtype == torch.bfloat16:
        gdt = _lib.QLORA_DTYPE_BF16
    elif grad_dtype == torch.float32:
        gdt = _lib.QLORA_DTYPE_F32
    else:
        raise TypeError("qlora: grad_dtype must be bfloat16 or float32")
    dev = dY.device
    if T is not None and (tuple(T.shape) != (M, 2 * r) or T.dtype != torch.bfloat16):
        raise ValueError(f"qlora: T must be the forward's bf16 [M, 2r] = {(M, 2 * r)} hi/lo pair")
    if need_dX:
        _check_out(dX, (M, K), torch.bfloat16, dev, "dX")
    _check_out(dL1, (K, r), grad_dtype, dev, "dL1")
    _check_out(dL2, (r, N), grad_dtype, dev, "dL2")
    _check_device(dev, X=X, T=T, L1=L1, L2=L2, codes=q.codes, c2_fp8=q.c2_fp8, c1=q.c1, c2_mean=q.c2_mean,
                  mask=dropout_mask, Xm=Xm)
    lib = _lib.load()
    if need_dX and dX is None:
        dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    if dL1 is None:
        dL1 = torch.empty((K, r), dtype=grad_dtype, device=dev)
    if dL2 is None:
        dL2 = torch.empty((r, N), dtype=grad_dtype, device=dev)
    if dropout_mask is not None:
        _mask_arg(dropout_mask, M, K, dev)
        ws = _WS.get(lib.qlora_linear_bwd_dropout_workspace_size(M, N, K, r), dev)
        _lib.check(lib.qlora_linear_bwd_dropout(_ptr(_bits(dY)), _ptr(_bits(X)), _ptr(T), _ptr(Xm), M, q.as_struct(),
                                                _ptr(_bits(L1)), _ptr(_bits(L2)), r, float(s), _ptr(dropout_mask),
                                                float(dropout_p), _ptr(dX) if need_dX else None, _ptr(dL1),
                                                _ptr(dL2), gdt, _ptr(ws), ws.numel(), _stream(dev)),
                   "qlora_linear_bwd_dropout")
        return (dX if need_dX else None), dL1, dL2
    ws_bytes = lib.qlora_linear_bwd_workspace_size(M, N, K, r)
    ws = _WS.get(ws_bytes, dev)
    _lib.check(lib.qlora_linear_bwd(_ptr(_bits(dY)), _ptr(_bits(X)), _ptr(T), M, q.as_struct(), _ptr(_bits(L1)),
                                    _ptr(_bits(L2)), r, float(s), _ptr(dX) if need_dX else None, _ptr(dL1),
                                    _ptr(dL2), gdt, _ptr(ws), ws.numel(), _stream(dev)), "qlora_linear_bwd")
    return (dX if need_dX else None), dL1, dL2


class BwdGroup:
    """A grouped backward whose arguments are marshalled once (see
    ``linear_bwd_group``).  Calling it runs the group again on the same
    tensors, which it keeps alive; only the C call is made per run."""

    def __init__(self, members, need_dX: bool = True, grad_dtype=torch.bfloat16):
        if not 0 < len(members) <= _lib.QLORA_MAX_GROUP:
            raise ValueError(f"qlora: a group holds 1..{_lib.QLORA_MAX_GROUP} linears")
        if grad_dtype == torch.bfloat16:
            gdt = _lib.QLORA_DTYPE_BF16
        elif grad_dtype == torch.float32:
            gdt = _lib.QLORA_DTYPE_F32
        else:
            raise TypeError("qlora: grad_dtype must be bfloat16 or float32")
        M = members[0]["dY"].shape[0]
        dev = members[0]["dY"].device
        # every argument is checked before the library is loaded or a pointer taken
        for m in members:
            dY, X, T, q, L1, L2 = m["dY"], m["X"], m.get("T"), m["q"], m["L1"], m["L2"]
            K, r, N = q.k_in, L1.shape[1], q.n_out
            if dY.shape[0] != M or dY.device != dev:
                raise ValueError("qlora: the members of a group share the token count and the device")
            if tuple(dY.shape) != (M, N) or tuple(X.shape) != (M, K) or L1.shape[0] != K or tuple(L2.shape) != (r, N):
                raise ValueError("qlora: shape mismatch")
            if T is not None and (tuple(T.shape) != (M, 2 * r) or T.dtype != torch.bfloat16):
                raise ValueError(f"qlora: T must be the forward's bf16 [M, 2r] = {(M, 2 * r)} hi/lo pair")
            if need_dX:
                _check_out(m.get("dX"), (M, K), torch.bfloat16, dev, "dX")
            _check_out(m.get("dL1"), (K, r), grad_dtype, dev, "dL1")
            _check_out(m.get("dL2"), (r, N), grad_dtype, dev, "dL2")
            _check_device(dev, False, X=X, T=T, L1=L1, L2=L2, codes=q.codes, c2_fp8=q.c2_fp8, c1=q.c1,
                          c2_mean=q.c2_mean)
        # caller-supplied outputs may not overlap each other or any member's input
        names = ("dX", "dL1", "dL2") if need_dX else ("dL1", "dL2")
        outs = [(i, name, _span(m.get(name))) for i, m in enumerate(members) for name in names]
        for i, name, sp in outs:
            for j, m in enumerate(members):
                for inp in ("dY", "X", "T"):
                    if _overlap(sp, _span(m.get(inp))):
                        raise ValueError(f"qlora: member {i}'s {name} overlaps member {j}'s {inp}")
            for j, name2, sp2 in outs:
                if (i, name) < (j, name2) and _overlap(sp, sp2):
                    raise ValueError(f"qlora: member {i}'s {name} overlaps member {j}'s {name2}")
        _check_device(dev)
        lib = _lib.load()
        arr = (_lib.BwdMember * len(members))()
        self._keep, self.outputs = [], []
        for i, m in enumerate(members):
            dY, X, T, q, L1, L2 = m["dY"], m["X"], m.get("T"), m["q"], m["L1"], m["L2"]
            K, r, N = q.k_in, L1.shape[1], q.n_out
            dX = m.get("dX") if need_dX else None
            if need_dX and dX is None:
                dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
            dL1 = m.get("dL1")
            if dL1 is None:
                dL1 = torch.empty((K, r), dtype=grad_dtype, device=dev)
            dL2 = m.get("dL2")
            if dL2 is None:
                dL2 = torch.empty((r, N), dtype=grad_dtype, device=dev)
            w = q.as_struct()
            self._keep += [w, dY, X, T, q, L1, L2]
            arr[i] = _lib.BwdMember(_ptr(_bits(dY)), _ptr(_bits(X)), _ptr(T), ctypes.pointer(w), _ptr(_bits(L1)),
                                    _ptr(_bits(L2)), r, float(m["s"]), _ptr(dX) if need_dX else None, _ptr(dL1),
                                    _ptr(dL2))
            self.outputs.append((dX if need_dX else None, dL1, dL2))
        self._arr, self._n, self._M, self._dev, self._gdt = arr, len(members), M, dev, gdt
        self._ws_bytes = lib.qlora_linear_bwd_group_workspace_size(arr, len(members), M)
        self._fn = lib.qlora_linear_bwd_group

    def __call__(self) -> list:
        ws = _WS.get(self._ws_bytes, self._dev)
        _lib.check(self._fn(self._arr, self._n, self._M, self._gdt, ws.data_ptr(), ws.numel(), _stream(self._dev)),
                   "qlora_linear_bwd_group")
        return self.outputs


def linear_bwd_group(members, need_dX: bool = True, grad_dtype=torch.bfloat16) -> list:
    """The backward of several linears whose output gradients are available
    together, in one call.

    ``members``: a sequence of dicts with keys ``dY`` [M, N_i], ``X`` [M, K_i],
    ``T`` (the forward's [M, 2 r_i] pair, or None to recompute), ``q``
    (NF4Tensor), ``L1`` [K_i, r_i], ``L2`` [r_i, N_i], ``s`` and optionally the
    outputs ``dX``, ``dL1``, ``dL2``.  Every member computes what
    ``linear_bwd`` computes; the rank-r products of all members run as two
    launches, and members that read the same X share one pass over it for
    dL1.  Returns [(dX or None, dL1, dL2)] in member order.
    """
    return BwdGroup(members, need_dX, grad_dtype)()


def profile_start(capacity: int = 4096) -> None:
    """Start logging the library's kernel launches with CUDA events (diagnostics)."""
    _lib.check(_lib.load().qlora_profile_start(capacity), "qlora_profile_start")


def profile_stop() -> list:
    """Stop logging; returns [(kernel kind name, milliseconds), ...] in launch order.

    Waits for the logged launches to finish.
    """
    import ctypes
    lib = _lib.load()
    n = lib.qlora_profile_stop()
    out = []
    kind, ms = ctypes.c_int(), ctypes.c_float()
    for i in range(n):
        _lib.check(lib.qlora_profile_read(i, ctypes.byref(kind), ctypes.byref(ms)), "qlora_profile_read")
        out.append((_lib.KERNEL_KINDS.get(kind.value, str(kind.value)), ms.value))
    return out


def last_device_error(device=None) -> int:
    """Synchronize the current stream and return/clear the library's device error word."""
    lib = _lib.load()
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    return lib.qlora_get_last_device_error(_stream(dev))
