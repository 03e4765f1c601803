"""Bounded device-side waits: a wait that runs out reports LA2_ERR_TIMEOUT
through la2_check() and leaves the context usable.

The fault is made on purpose with a spin limit far below what any wait needs
(la2_set_spin_limit), never with a trap, a bad address or an endless loop.
"""

import pytest
import torch

from linear_attention_la2_b200 import inputs as la2_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def la2():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_la2_b200 import build

    build.build()
    from linear_attention_la2_b200 import la2 as lib

    yield lib
    lib.la2_set_spin_limit(0)
    lib.la2_set_chunk_len(0)


def test_wait_limit_reports_timeout_and_recovers(la2):
    ins = la2_inputs.make_custom(1, 4, 4096, 128, 128, "bf16", seed=3)
    q, k, v = (ins[n].cuda() for n in "qkv")
    ref = la2.forward(q, k, v, block=64)
    la2.check()
    assert la2.la2_set_spin_limit(1) == la2.LA2_OK
    try:
        out = torch.zeros_like(ref)
        la2.forward(q, k, v, block=64, out=out)  # launch succeeds; waits give up on the device
        assert la2.la2_check(la2._stream_handle(None)) == la2.LA2_ERR_TIMEOUT
    finally:
        la2.la2_set_spin_limit(0)
    # the error word is cleared and the next call runs normally
    assert la2.la2_check(la2._stream_handle(None)) == la2.LA2_OK
    again = la2.forward(q, k, v, block=64)
    la2.check()
    assert torch.equal(again, ref)
