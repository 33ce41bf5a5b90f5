"""CPU oracle for the QLoRA NF4 + Double Quantization linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product package imports, links or
executes this package; only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may call it.

It is a plain, slow, obviously-correct restatement of what the QLoRA paper
("QLoRA: Efficient Finetuning of Quantized LLMs", Dettmers et al., page
aiingo.vercel.app/paper/paper-2305-14314) defines:

* ``nf4dq``        -- blockwise absmax quantization (§2 "Block-wise k-bit
                      Quantization", Eqs. 1-2), the NF4 code (§3 "4-bit
                      NormalFloat Quantization", Eq. 4 and the exact values in
                      Appendix E), Double Quantization (§3 "Double
                      Quantization") and doubleDequant (§3, Eq. 6).
* ``qlora_linear`` -- the QLoRA linear layer forward (§2 Eq. 3, §3 Eq. 5) and
                      its backward with adapter-only gradients (§3, the
                      paragraph after Eq. 6), in float64.
* ``stack``        -- the wiring between the layers of a stack of such
                      linears (a reading: the pages give no model code).

Every function is pinned by ``tests/test_oracle_*.py`` against values the
paper prints, closed forms, library special cases or brute force.  It shares
no code, table or constant with the CUDA path.
"""

from . import nf4dq, qlora_linear, stack  # noqa: F401
