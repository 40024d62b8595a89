"""B200-native bidirectional Video Delta Attention (VDA) branch.

The compute lives in the C-ABI library ``libvda.so`` (hand-written CUDA for
sm_100a); ``frame_wise_delta_vda_b200.api`` marshals torch tensors into it.
Importing the package does not load the library, so the seeded input
generator (``frame_wise_delta_vda_b200.inputs``) works on machines without it.
"""

__all__ = ["api", "inputs"]


def __getattr__(name):
    if name == "api":
        from . import api
        return api
    raise AttributeError(name)
