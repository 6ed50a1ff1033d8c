"""fp64 CPU oracle for the Muon step.  Test infrastructure: imported only by tests,
the smoke check and the benchmark's CPU-baseline leg, never by the product path."""
from .muon_oracle import (  # noqa: F401
    NS_EPS,
    QUINTIC,
    apply_step,
    default_shape_scale,
    frobenius_norm,
    gram,
    momentum_update,
    muon_step,
    nesterov_input,
    newton_schulz,
    parameter_update,
    polynomial,
)
