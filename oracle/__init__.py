"""fp64 CPU oracle (test infrastructure only; see ``muon_oracle``)."""
from .muon_oracle import *  # noqa: F401,F403
from .muon_oracle import (KJ_COEFFS, TEXTBOOK_COEFFS, NS_EPS, SCALE_MODES,  # noqa: F401
                          fixed_schedule, hybrid_schedule, round_to_bf16, round_to_f32,
                          momentum, ns_input, frobenius_prescale, newton_schulz, msign_svd,
                          scale_factor, muon_update, muon_step, project_tangent,
                          cayley_dense, cayley_woodbury, stiefel_cayley_step,
                          orthogonality_error)
