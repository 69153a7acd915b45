"""Float64 CPU oracle of the HySparse hybrid-block hot path (test infrastructure only).

Only tests, the smoke check and the benchmark's CPU-baseline leg import this
package.  The CUDA library and its binding never call it."""
from .hysparse_oracle import *  # noqa: F401,F403
from . import hysparse_backward as backward  # noqa: F401,E402
