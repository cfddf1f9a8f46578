"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This package holds the input recipe only (shapes, seeds, value distributions)
and none of the recurrence's arithmetic.  Both the tests and the benchmark draw
their inputs here, once, on the host; the oracle and the CUDA library then
receive the same (rounded) values.
"""
from .inputs import (CONFIGS, DECODE, DecodeProblem, Problem, decode_inputs, make_inputs,
                     problem)

__all__ = ["CONFIGS", "DECODE", "DecodeProblem", "Problem", "decode_inputs", "make_inputs",
           "problem"]
