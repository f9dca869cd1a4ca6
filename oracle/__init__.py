"""Float64 CPU oracle (test infrastructure only; see la_oracle.py)."""

from .la_oracle import (  # noqa: F401
    FEATURE_MAPS,
    brute_force,
    brute_force_head,
    brute_force_rows,
    e4m3_decode,
    feature_map,
    forward,
    forward_e4m3,
    landmark_count,
    landmark_head,
    landmark_positions,
    linear_causal_head,
    linear_noncausal_head,
    phi_elu1,
    phi_relu,
    phi_softmax,
    rows,
    sigmoid,
    ttr_forward,
)
