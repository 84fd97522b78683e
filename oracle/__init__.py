"""CPU oracle for the QLoRA NF4 + double-quantization linear layer.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``, never by the product path.  It shares
no code with the CUDA library (no kernels, headers, tables or helpers); the
only module both sides use is ``synth``, the seeded input generator.
"""
from . import nf4  # noqa: F401
