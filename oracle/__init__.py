"""CPU oracle for SageSLA attention -- test infrastructure only.

Imported by tests/, by the package entry's smoke check and by the benchmark's
CPU-baseline leg; never by the library.  See sla_oracle.py (the operator),
w8a8_oracle.py (the W8A8 linear layer) and sla_backward_oracle.py (the
gradient of the fine-tune path), each with a plain C++ restatement (*.cpp,
loaded through cpp_oracle.py, w8a8_cpp.py and sla_backward_cpp.py).
"""

from . import sla_oracle  # noqa: F401
from .sla_oracle import *  # noqa: F401,F403
