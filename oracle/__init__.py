"""CPU oracle for the tensor-parallel decoder block — TEST INFRASTRUCTURE ONLY.

Plain, slow, float64 NumPy statements of what the hot path computes, used by
``tests/``, by ``__graft_entry__.smoke()`` and by the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py``, and by nothing else. It shares no
code with the CUDA library and never imports it. See ``oracle/tp_block.py``.
"""
from .tp_block import *  # noqa: F401,F403
