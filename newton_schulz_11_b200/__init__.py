"""B200-native Muon optimizer step (momentum, Newton-Schulz orthogonalisation, update).

The compute path is the C-ABI library ``libmuon_b200.so`` (hand-written sm_100a
kernels); this package only marshals arguments to it.  The library is loaded on
first use, and a missing or unloadable library raises ``MuonLibraryError``:
there is no other implementation to fall back to.
"""
from .inputs import WORKLOADS  # noqa: F401


def __getattr__(name):
    # Lazy: importing the package (e.g. for the input generators) must not need torch/CUDA.
    if name in ("muon_step", "newton_schulz", "workspace_size", "scratch_view", "device_status",
                "Workspace", "default_workspace", "QUINTIC", "quintic_table", "MuonError",
                "MuonLibraryError"):
        from . import api

        return getattr(api, name)
    raise AttributeError(name)
