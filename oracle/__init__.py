"""CPU oracle of the OneTrans hot path (fp64 NumPy).

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check and by the
benchmark's CPU-baseline leg.  The CUDA library never imports or calls it, and
it shares no code with the library.
"""
from . import onetrans, flops  # noqa: F401
