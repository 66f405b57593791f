"""CPU oracle of the gated block-sparse GQA decode step (test infrastructure only).

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
may import this package.  The library never does, and this package never
imports the library.
"""

from .seer_oracle import *  # noqa: F401,F403
