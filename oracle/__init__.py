"""CPU oracle for the STCA forward path: TEST INFRASTRUCTURE, not part of the library.

Only ``tests/``, ``__graft_entry__.smoke()`` and the bench's CPU-baseline leg may import
anything from this package.  The CUDA library never calls it, and it never calls the
library.
"""
