"""fp64 CPU oracles: the Lighthouse attention layer and PISA block selection.

TEST INFRASTRUCTURE ONLY: imported by the tests, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``, never by the product package.
"""

from . import lighthouse_oracle  # noqa: F401
from . import gap_repair  # noqa: F401
from . import pisa_oracle  # noqa: F401
