"""CPU oracle of the LatentMoE layer (test infrastructure only).

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
import this package. ``oracle.lmoe_oracle`` is the layer forward;
``oracle.lmoe_backward`` its gradients and the NVFP4 training recipe's pieces.
"""
from . import lmoe_backward  # noqa: F401
from . import lmoe_oracle  # noqa: F401
