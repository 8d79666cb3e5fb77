"""CPU oracle for BigBird block-sparse attention.  TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously-correct fp64 reference: an independent layout builder
(``oracle.layout``), masked-dense attention (``oracle.attention``), its
gradients (``oracle.backward``) and the layer's two projections
(``oracle.projection``).  Only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import it; the CUDA library never does, and this package imports nothing from
the library.  Every function cites the page passage it follows.

Parity status: every function here is pinned by a ``-m "not gpu"`` test
against a closed form, a library routine, a published known-answer vector or
brute force (see ``tests/test_oracle_*.py``).
"""

from . import attention, backward, layout, projection  # noqa: F401
