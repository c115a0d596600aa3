"""CPU oracle for the paged-attention library — TEST INFRASTRUCTURE ONLY.

Plain NumPy fp64 restatements of what the paged-attention path computes,
written from the pages and pinned by the ``-m "not gpu"`` tests.  Only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may import
this package; the CUDA library never does.
"""
from . import arithmetic, fp8, paged_attention  # noqa: F401
from .paged_attention import *  # noqa: F401,F403
from .arithmetic import *  # noqa: F401,F403
