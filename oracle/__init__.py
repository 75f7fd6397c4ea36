"""CPU oracle of the LatentMoE layer forward (test infrastructure only).

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
import this package. See ``oracle.lmoe_oracle`` for what it computes.
"""
from . import lmoe_oracle  # noqa: F401
