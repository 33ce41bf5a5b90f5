"""Host-side test of the decoder-stack driver's wiring.

The driver is run on the CPU with a stand-in for the library whose linears
are the oracle's (test infrastructure only), so the test checks the driver's
own logic: which tensor feeds which linear, forward and backward, and the
residual add and gradient sum against the oracle's wiring definitions, bit
for bit.
"""

import numpy as np
import torch

from bit_nf4_quantized_02_b200 import stack as qstack
from oracle import nf4dq, qlora_linear
from oracle import stack as ostack


def _np(t):
    return t.detach().float().numpy()


class OracleOps:
    """quantize_nf4_dq / linear_fwd / linear_bwd (and their grouped forms) on CPU tensors via the oracle."""

    def __init__(self):
        self.calls = []

    def quantize_nf4_dq(self, W, out=None):
        oq = nf4dq.quantize_nf4_dq(W.float().numpy())
        oq["w_hat"] = nf4dq.dequantize(oq)
        return oq

    def linear_fwd(self, X, q, L1, L2, s, Y=None, T=None):
        Yr, Tr = qlora_linear.forward(_np(X), q["w_hat"], _np(L1), _np(L2), s)
        Y.copy_(torch.from_numpy(Yr.astype(np.float32)))
        r = L1.shape[1]
        hi = torch.from_numpy(Tr.astype(np.float32)).bfloat16()
        T[:, :r] = hi
        T[:, r:] = torch.from_numpy((Tr - hi.double().numpy()).astype(np.float32)).bfloat16()
        self.calls.append(("fwd", X, Y.clone()))
        return Y, T

    def FwdGroup(self, members):
        """A grouped forward: each member as linear_fwd computes it, in member order."""
        def run():
            return [self.linear_fwd(m["X"], m["q"], m["L1"], m["L2"], m["s"], Y=m["Y"], T=m["T"])
                    for m in members]
        return run

    def BwdGroup(self, members, grad_dtype=None):
        """A grouped backward: each member as linear_bwd computes it, in member order."""
        def run():
            return [self.linear_bwd(m["dY"], m["X"], m["T"], m["q"], m["L1"], m["L2"], m["s"], dX=m["dX"],
                                    dL1=m["dL1"], dL2=m["dL2"]) for m in members]
        return run

    def linear_bwd(self, dY, X, T, q, L1, L2, s, grad_dtype=None, dX=None, dL1=None, dL2=None):
        dXr, dL1r, dL2r = qlora_linear.backward(_np(dY), _np(X), q["w_hat"], _np(L1), _np(L2), s)
        dX.copy_(torch.from_numpy(dXr.astype(np.float32)))
        dL1.copy_(torch.from_numpy(dL1r.astype(np.float32)))
        dL2.copy_(torch.from_numpy(dL2r.astype(np.float32)))
        self.calls.append(("bwd", dY.clone(), X, dX.clone()))
        return dX, dL1, dL2


def _make(shape, std, seed, dtype):
    t = torch.from_numpy(np.random.default_rng(seed).standard_normal(shape).astype(np.float32) * std)
    return t.to(dtype)


def test_stack_wiring_against_oracle_definitions():
    ops = OracleOps()
    hidden, mlp, layers, M, r = 64, 128, 3, 12, 4
    st = qstack.QLoRAStack(ops, hidden, mlp, layers, M, r, alpha=8.0, seed=7, device="cpu", make=_make)
    st.step()
    fwd = [c for c in ops.calls if c[0] == "fwd"]
    bwd = [c for c in ops.calls if c[0] == "bwd"]
    assert len(fwd) == 7 * layers and len(bwd) == 7 * layers
    for l in range(layers):
        f = fwd[7 * l:7 * l + 7]
        # q, k, v, o, gate, up read H[l]; down reads U[l], up's output
        for c in f[:6]:
            assert c[1] is st.H[l]
        assert torch.equal(f[5][2], st.U[l]) and f[6][1] is st.U[l]
        assert torch.equal(f[6][2], st.D[l])
        np.testing.assert_array_equal(_np(st.H[l + 1]), ostack.next_input(_np(st.D[l]), _np(st.R[l])))
    for i, l in enumerate(reversed(range(layers))):
        b = bwd[7 * i:7 * i + 7]
        # down first, from the gradient of the layer output; then q, k, v, o, gate, up
        assert torch.equal(b[0][1], st.dH[l + 1]) and b[0][2] is st.U[l]
        assert torch.equal(b[0][3], st.dU[l])
        for name, c in zip(qstack.READS_H, b[1:]):
            x = st.lin[l][name]
            assert c[2] is st.H[l]
            assert torch.equal(c[1], st.dU[l] if name == "up" else x.dY)
        dX = {name: _np(c[3]) for name, c in zip(qstack.READS_H, b[1:])}
        np.testing.assert_array_equal(_np(st.dH[l]), ostack.grad_sum(dX))
    # adapter gradients land in the flat buffer, one view per linear
    for x in st.linears():
        assert x.dL1.data_ptr() >= st.grads.flat.data_ptr()
        assert np.abs(_np(x.dL1)).sum() > 0 and np.abs(_np(x.dL2)).sum() > 0
