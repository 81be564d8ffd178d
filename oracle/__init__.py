"""CPU oracle for the TokenGate gate layer and token-gated attention.

TEST INFRASTRUCTURE. Only the tests, the package smoke check and the benchmark's
CPU-baseline / reference legs may import this package.  The library's product path
never calls it, and this package never imports the library: the two share nothing
but the seeded tensors drawn by ``synthetic_inputs``.

Everything is plain NumPy in float64 (selection decisions in float32, the precision
the scores are handed over in), written step by step from the pages' description of
the method.  See ``oracle.tokengate`` for the functions and their citations.
"""
from .tokengate import *  # noqa: F401,F403
