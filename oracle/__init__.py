"""CPU oracle for the T16 trellis-quantised MoE layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference arm of
``bench.py`` may import this package.  The product path (the CUDA library and its
Python binding) never imports it, and the two share no code.

``t16``      scalar C bit reader and T16 codebook (ctypes).
``layer``    fp64 Hadamard rotation, dequantisation, projections, routing, SwiGLU
             expert and combine, written from the pages' description.
"""
from . import t16, layer  # noqa: F401
