"""B200-native bidirectional Video Delta Attention (VDA) branch.

The compute lives in the C-ABI library ``libvda.so`` (hand-written CUDA for
sm_100a); ``frame_wise_delta_vda_b200.api`` marshals torch tensors into it.
Importing the package does not load the library, so the seeded input
generator (``frame_wise_delta_vda_b200.inputs``) works on machines without it.
"""

import importlib

__all__ = ["api", "inputs"]


def __getattr__(name):
    if name in ("api", "inputs", "build"):
        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)
