"""Seeded synthetic inputs for BitDelta compress / apply workloads.

This package produces input *data* only (weights, deltas, activations, tenant ids,
tenant sign words and scales). It holds none of the method's arithmetic: no delta,
no clip, no scale, no sign, no packing, no product. Both the oracle-based tests and
the CUDA path take their inputs from here, so both see identical bytes.
"""

from .gen import *  # noqa: F401,F403
