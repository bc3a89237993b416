"""CPU oracle (fp64 NumPy) of the Zebra3D global-attention hot path.

TEST INFRASTRUCTURE: imported only by the tests, the smoke check and the
benchmark's CPU-baseline leg. The library never imports it.
"""
from .zebra_oracle import *  # noqa: F401,F403
from .zebra_oracle import Geom, NEAR_TIE_REL_GAP  # noqa: F401
