"""STCA forward on NVIDIA B200: libstca (CUDA, sm_100a) and its thin Python binding.

``binding`` mirrors the C ABI in include/stca.h and include/stca_kernels.h; ``device``
uploads workloads and owns handles.  The library must be built
(``python -m target_attention_b200.build``); nothing here computes on the CPU.
"""
from . import binding  # noqa: F401
from .binding import lib  # noqa: F401
