"""CPU oracle for the two-level sparse decode step (test infrastructure only).

Plain, slow numpy code in float64.  Only the tests, the package's smoke entry
and the benchmark's CPU-baseline leg may import it; the product path never
does.  It shares no code with the CUDA library.
"""

from .two_level import *  # noqa: F401,F403
from .two_level import __all__  # noqa: F401
