"""Seeded synthetic inputs shared by the CUDA path's tests, the bench and the oracle.

This package only draws random numbers and encodes them in the storage formats the
library reads (fp32, or bf16 bit patterns held as ``uint16``).  It holds none of the
method's arithmetic: no bucketing, no attention, no FFN.
"""
from .generate import (  # noqa: F401
    STCA_CONFIGS,
    bf16_bits,
    make_hyformer,
    make_pointwise,
    make_stca,
    make_stca_history,
)
