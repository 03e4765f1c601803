"""Float64 CPU oracle (test infrastructure only; see ``la2_oracle``)."""

from .la2_oracle import (  # noqa: F401
    backward,
    backward_decay,
    backward_gqa,
    backward_rows,
    blocked_forward,
    decode_step,
    backward_from_states,
    forward,
    forward_decay,
    forward_from_state,
    forward_gqa,
    forward_rows,
    kv_state,
    recurrent_forward,
    recurrent_forward_decay,
    relative_frobenius,
)
