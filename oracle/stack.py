"""Layer-to-layer wiring of a stack of QLoRA linears (oracle).

TEST INFRASTRUCTURE ONLY (see the package docstring).

The QLoRA paper ("QLoRA: Efficient Finetuning of Quantized LLMs",
aiingo.vercel.app/paper/paper-2305-14314) finetunes LLaMA models whose
layers each hold seven linears (§4 and Table 9 name the model sizes), but
it gives no model code.  The reading used for a stack of such layers, and
restated here as plain definitions:

* the layer output D is down(up(H)); the next layer's input is
  H' = bf16(fp32(D + R)) for a fixed bf16 residual R;
* the gradient of H is dH = bf16 of the fp32 sum of the six dX of the
  linears that read H, added one after another in the order
  q, k, v, o, gate, up.

Both are exact given their bf16 inputs (round to nearest even at each
fp32 add and at the final bf16 rounding), so the GPU's glue is checked
bit for bit against them.  Each linear of a layer is checked with
``qlora_linear`` on the GPU's own inputs to that layer ("teacher forcing"),
so errors do not compound across layers.

Parity of the chained stack beyond these per-layer checks is unpinned: the
pages fix no stack, so there is no value to pin the chain to.
"""

from __future__ import annotations

import numpy as np

from .nf4dq import bf16_bits_to_f32, bf16_rne_bits

READS_H = ("q", "k", "v", "o", "gate", "up")


def _bf16(x32: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(bf16_rne_bits(np.asarray(x32, np.float32)))


def next_input(D, R) -> np.ndarray:
    """H' = bf16(fp32(D + R)) for bf16-valued D, R (float32 arrays)."""
    return _bf16(np.asarray(D, np.float32) + np.asarray(R, np.float32))


def grad_sum(dX_by_name: dict) -> np.ndarray:
    """dH = bf16(((((dX_q + dX_k) + dX_v) + dX_o) + dX_gate) + dX_up) in fp32."""
    acc = np.asarray(dX_by_name[READS_H[0]], np.float32).copy()
    for name in READS_H[1:]:
        acc = (acc + np.asarray(dX_by_name[name], np.float32)).astype(np.float32)
    return _bf16(acc)
