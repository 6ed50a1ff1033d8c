"""B200-native Muon optimizer step (momentum, Newton-Schulz orthogonalisation, update).

The compute path is the C-ABI library ``libmuon_b200.so`` (hand-written sm_100a
kernels); this package only marshals arguments to it.  The library is loaded on
first use and a missing or unloadable library raises ``MuonLibraryError``.
"""
from .inputs import WORKLOADS  # noqa: F401
