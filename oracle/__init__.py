"""CPU fp64 oracle of the Step-3.5-Flash MoE FFN layer forward.

Test infrastructure: only the tests, the smoke check and the CPU-baseline legs
of the benchmark use it.  The product library never imports it.
"""
from .moe_oracle import *  # noqa: F401,F403
from .moe_oracle import as_numpy  # noqa: F401
