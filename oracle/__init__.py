"""CPU oracle for the ConvRot W4A4 linear layer (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline arm of
``bench.py`` may import this package.  The CUDA library never does, and the
two share no code.
"""

from .convrot_oracle import *  # noqa: F401,F403
from .convrot_oracle import __all__  # noqa: F401
