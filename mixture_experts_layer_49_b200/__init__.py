"""B200-native forward pass of a Mixture-of-Experts FFN layer.

The layer runs in libmoe (hand-written CUDA for sm_100a behind the C ABI in
include/moe.h); ``native`` is its thin Python binding and ``synthetic`` draws
seeded inputs shaped like the layers the pages describe.
"""
from . import native, synthetic  # noqa: F401
from .native import MoEError, MoeConfig, Outputs, config_from_workload, make_config  # noqa: F401
