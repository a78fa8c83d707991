"""CPU oracle of the LoopKV decode path: test infrastructure only.

Imported by the tests, the smoke check and the benchmark's CPU-baseline leg;
never by the product package.
"""

from .loopkv_oracle import *  # noqa: F401,F403
