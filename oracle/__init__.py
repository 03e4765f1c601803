"""Float64 CPU oracle (test infrastructure only; see ``la2_oracle``)."""

from .la2_oracle import (  # noqa: F401
    backward,
    backward_gqa,
    backward_rows,
    blocked_forward,
    decode_step,
    forward,
    forward_gqa,
    forward_rows,
    kv_state,
    recurrent_forward,
    relative_frobenius,
)
