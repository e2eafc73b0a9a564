"""CPU oracle for SageSLA attention -- test infrastructure only.

Imported by tests/, by the package entry's smoke check and by the benchmark's
CPU-baseline leg; never by the library.  See sla_oracle.py.
"""

from . import sla_oracle  # noqa: F401
from .sla_oracle import *  # noqa: F401,F403
