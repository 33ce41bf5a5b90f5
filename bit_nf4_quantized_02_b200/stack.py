"""A stack of decoder layers, each the seven QLoRA linears of a LLaMA layer.

Every linear is an NF4 + Double-Quantization weight with a LoRA adapter
(QLoRA, §3 Eq. 5), run forward and then backward in sequence through the
library (quantize_nf4_dq, FwdGroup, linear_fwd, BwdGroup, linear_bwd).

The pages give no model code, so the layer wiring is the plainest stack of the
seven LLaMA linears that carries activations from layer to layer:

* forward: q, k, v, o, gate and up all read the layer input H (one grouped
  call, which shares their adapter down-projection); down reads U = up(H);
  the layer output is D = down(U).  The next layer's input is
  H' = bf16(D + R), with R a fixed N(0, 1) bf16 residual per layer;
* backward, top to bottom: dD = dH'; dU = dX of down.  q, k, v, o and gate
  get fixed N(0, 1) bf16 output gradients; the six linears on H then run as
  one grouped backward (their adapter products in two launches).  dH = bf16
  of the fp32 sum of the six dX, taken in the order q, k, v, o, gate, up.

The residual add and the gradient sum are elementwise glue outside the QLoRA
linear, done here with torch; every linear's work runs in the library.  The
``ops`` argument takes any object with those library functions, so that the
wiring can be exercised on the host with a stand-in.
"""

from __future__ import annotations

from dataclasses import dataclass

import torch

from .dp import FlatGrads

NAMES = ("q", "k", "v", "o", "gate", "up", "down")
SEEDED_DY = ("q", "k", "v", "o", "gate")    # output gradients drawn, not propagated
READS_H = ("q", "k", "v", "o", "gate", "up")


def layer_shapes(hidden: int, mlp: int) -> dict:
    """(n_out, k_in) of each of the seven linears."""
    return {"q": (hidden, hidden), "k": (hidden, hidden), "v": (hidden, hidden), "o": (hidden, hidden),
            "gate": (mlp, hidden), "up": (mlp, hidden), "down": (hidden, mlp)}


@dataclass
class StackLinear:
    name: str
    W: torch.Tensor          # fp32 or bf16 [n_out, k_in], quantized every step
    L1: torch.Tensor         # bf16 [k_in, r]
    L2: torch.Tensor         # bf16 [r, n_out]
    T: torch.Tensor          # bf16 [M, 2r], saved by the forward
    q: object = None         # NF4Tensor
    dY: torch.Tensor | None = None   # seeded output gradient (q, k, v, o, gate)
    dL1: torch.Tensor | None = None
    dL2: torch.Tensor | None = None


class QLoRAStack:
    """``layers`` decoder layers of seven QLoRA linears over M tokens.

    ``make(shape, std, seed, dtype)`` draws the seeded tensors.  Activations
    kept for the backward and for inspection: H[l] (layer inputs, H[layers]
    the stack output), U[l], D[l], dU[l] and dH[l] (gradient of H[l]).
    """

    def __init__(self, ops, hidden: int, mlp: int, layers: int, M: int, r: int, alpha: float, seed: int,
                 device, make, grad_dtype=torch.float32):
        self.ops = ops
        self.hidden, self.mlp, self.layers, self.M, self.r = hidden, mlp, layers, M, r
        self.s = alpha / r
        self.grad_dtype = grad_dtype
        shapes = layer_shapes(hidden, mlp)
        bf = torch.bfloat16
        self.lin = []
        for l in range(layers):
            row = {}
            for i, name in enumerate(NAMES):
                n, k = shapes[name]
                base = seed + 1000 * l + 10 * i
                row[name] = StackLinear(
                    name, make((n, k), 0.02, base, torch.float32),
                    make((k, r), 1.0 / k ** 0.5, base + 1, bf), make((r, n), 0.01, base + 2, bf),
                    torch.empty(M, 2 * r, dtype=bf, device=device),
                    dY=make((M, n), 1.0, base + 3, bf) if name in SEEDED_DY else None)
            self.lin.append(row)
        self.R = [make((M, hidden), 1.0, seed + 1000 * l + 500, bf) for l in range(layers)]
        self.H = [make((M, hidden), 1.0, seed + 999_000, bf)] + \
                 [torch.empty(M, hidden, dtype=bf, device=device) for _ in range(layers)]
        self.U = [torch.empty(M, mlp, dtype=bf, device=device) for _ in range(layers)]
        self.D = [torch.empty(M, hidden, dtype=bf, device=device) for _ in range(layers)]
        self.dU = [torch.empty(M, mlp, dtype=bf, device=device) for _ in range(layers)]
        self.dH = [torch.empty(M, hidden, dtype=bf, device=device) for _ in range(layers)] + \
                  [make((M, hidden), 1.0, seed + 998_000, bf)]     # dH[layers]: gradient at the top
        # discarded outputs (q, k, v, o, gate): one buffer each, since a grouped
        # forward's members may not share an output
        self._y = {name: torch.empty(M, shapes[name][0], dtype=bf, device=device) for name in SEEDED_DY}
        self._groups, self._group_key = None, None
        self._bgroups, self._bgroup_key = None, None
        # the dX of the six linears on H: one buffer each (a grouped backward's
        # members may not share an output), summed into dH
        self._dx = {name: torch.empty(M, hidden, dtype=bf, device=device) for name in READS_H}
        self._acc = torch.empty(M, hidden, dtype=torch.float32, device=device)
        # adapter gradients: views of one flat buffer (one all-reduce per step)
        order = [self.lin[l][name] for l in range(layers) for name in NAMES]
        self.grads = FlatGrads([(x.L1.shape[0], x.L2.shape[1], r) for x in order], device,
                               dtype=grad_dtype)
        for x, (dl1, dl2) in zip(order, self.grads.views):
            x.dL1, x.dL2 = dl1, dl2

    def linears(self):
        return [self.lin[l][name] for l in range(self.layers) for name in NAMES]

    def quantize(self):
        for x in self.linears():
            x.q = self.ops.quantize_nf4_dq(x.W, out=x.q)

    def _fwd_groups(self):
        """One grouped forward per layer over the six linears that read H (built
        once per set of quantized weights)."""
        key = tuple(id(self.lin[l][name].q) for l in range(self.layers) for name in READS_H)
        if key != self._group_key:
            self._groups = [
                self.ops.FwdGroup([{"X": self.H[l], "q": row[name].q, "L1": row[name].L1, "L2": row[name].L2,
                                    "s": self.s, "Y": self.U[l] if name == "up" else self._y[name],
                                    "T": row[name].T} for name in READS_H])
                for l, row in enumerate(self.lin)]
            self._group_key = key
        return self._groups

    def _bwd_groups(self):
        """One grouped backward per layer over the six linears that read H."""
        key = tuple(id(self.lin[l][name].q) for l in range(self.layers) for name in READS_H)
        if key != self._bgroup_key:
            self._bgroups = [
                self.ops.BwdGroup([{"dY": self.dU[l] if name == "up" else row[name].dY, "X": self.H[l],
                                    "T": row[name].T, "q": row[name].q, "L1": row[name].L1, "L2": row[name].L2,
                                    "s": self.s, "dX": self._dx[name], "dL1": row[name].dL1,
                                    "dL2": row[name].dL2} for name in READS_H], grad_dtype=self.grad_dtype)
                for l, row in enumerate(self.lin)]
            self._bgroup_key = key
        return self._bgroups

    def forward(self):
        ops, s = self.ops, self.s
        groups = self._fwd_groups()
        for l in range(self.layers):
            row = self.lin[l]
            groups[l]()          # q, k, v, o, gate and up on H[l]
            d = row["down"]
            ops.linear_fwd(self.U[l], d.q, d.L1, d.L2, s, Y=self.D[l], T=d.T)
            torch.add(self.D[l].float(), self.R[l].float(), out=self._acc)
            self.H[l + 1].copy_(self._acc)          # round to nearest even into bf16

    def backward(self):
        ops, s = self.ops, self.s
        groups = self._bwd_groups()
        for l in reversed(range(self.layers)):
            d = self.lin[l]["down"]
            ops.linear_bwd(self.dH[l + 1], self.U[l], d.T, d.q, d.L1, d.L2, s, grad_dtype=self.grad_dtype,
                           dX=self.dU[l], dL1=d.dL1, dL2=d.dL2)
            groups[l]()          # q, k, v, o, gate and up on H[l]
            for j, name in enumerate(READS_H):
                if j == 0:
                    self._acc.copy_(self._dx[name])
                else:
                    self._acc.add_(self._dx[name].float())
            self.dH[l].copy_(self._acc)

    def step(self, group=None):
        """One pass: quantize every weight, forward, backward, adapter all-reduce."""
        self.quantize()
        self.forward()
        self.backward()
        self.grads.allreduce(group)
