"""CPU oracle (test infrastructure only; see ``ds4sp_oracle``).

Only tests, the smoke check and the benchmark's CPU-baseline leg import this
package. The CUDA library never does.
"""
from .ds4sp_oracle import *  # noqa: F401,F403
