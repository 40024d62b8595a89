"""B200-native bidirectional Video Delta Attention (VDA) branch.

The compute lives in the C-ABI library ``libvda.so`` (hand-written CUDA for
sm_100a); ``frame_wise_delta_vda_b200.api`` marshals torch tensors into it.
Importing the package does not load the library, so the seeded input
generator (``frame_wise_delta_vda_b200.inputs``) works on machines without it.
``frame_wise_delta_vda_b200.ulysses`` runs the op head-sharded over the ranks
of a ``torch.distributed`` job (all-to-all exchanges around the forward).
"""

import importlib

__all__ = ["api", "inputs", "ulysses"]


def __getattr__(name):
    if name in ("api", "inputs", "build", "ulysses", "ranks"):
        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)
