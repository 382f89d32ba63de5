"""fp64 CPU oracle for the Muon step.  Test infrastructure only: never imported
by the product path (see muon_oracle's header)."""
from .muon_oracle import (  # noqa: F401
    CLASSIC_COEFFS,
    DEFAULT_EPS,
    DEFAULT_RESTARTS,
    TUNED_COEFFS,
    adamw_step,
    frobenius_normalize,
    momentum_update,
    muon_step,
    ns_flops,
    ns_gram,
    ns_standard,
    orthogonalize,
)
