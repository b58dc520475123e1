"""fp64 CPU oracle for the Lighthouse attention layer.

TEST INFRASTRUCTURE ONLY: imported by the tests, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``, never by the product package.
"""

from . import lighthouse_oracle  # noqa: F401
from . import gap_repair  # noqa: F401
