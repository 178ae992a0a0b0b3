"""Float64 CPU oracle for the KDA layer (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU baseline /
reference leg may import this package.
"""
from .kda_oracle import (  # noqa: F401
    GATE_LOWER_BOUND, L2_EPS, NORM_EPS, sigmoid, softplus, silu, l2_normalize, log_decay,
    apply_key_decay, causal_depthwise_conv, prep, recurrence, gated_rmsnorm,
    layer, projections, verify, rollback, chunked_recurrence,
)
