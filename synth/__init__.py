"""Seeded synthetic inputs and workload shapes.

This package holds only random-number generation and shape tables: none of the
quantization or linear-layer arithmetic.  Both the CPU oracle's tests and the
CUDA path's tests and benchmark draw their inputs from here.
"""
