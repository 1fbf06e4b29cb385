"""CPU oracle for MXFP4 quantization and MXFP4 attention (UOS / OCP, PNQ).

TEST INFRASTRUCTURE ONLY: used by tests/, the package smoke check and the benchmark's
CPU-baseline leg. The library never imports it and shares no code with it.
"""
from . import mxfp4, attention, efq  # noqa: F401
