"""la2_forward_noalloc: the forward for callers that cannot allocate device
memory when they call the op (its chunk states live in a fixed 32 MiB array
inside the library instead of a caller workspace).

Checked through the C ABI against la2_forward (the regular entry point with a
caller workspace), within the bf16 / fp32 bars of the parity tests, on two
calls in a row with different inputs so that a result left in the shared array
by the first call cannot pass for the second. This file sorts last so that a
run stopping at the first failure has run every other test before it.
"""

import ctypes

import pytest
import torch

from linear_attention_la2_b200 import inputs as la2_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 1e-2}


@pytest.fixture(scope="module")
def la2():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_la2_b200 import build

    build.build()
    from linear_attention_la2_b200 import la2 as lib

    lib.la2_set_chunk_len(0)
    yield lib
    lib.la2_set_chunk_len(0)


def _rel(x, ref):
    x, ref = x.double(), ref.double()
    return float(torch.linalg.vector_norm(x - ref) / torch.linalg.vector_norm(ref))


def _noalloc(la2, q, k, v, o, causal, block, dt):
    B, H, N, d = q.shape
    return la2.la2_forward_noalloc(la2._ptr(q), la2._ptr(k), la2._ptr(v), la2._ptr(o), B, H, N, d,
                                   v.shape[-1], int(causal), block, dt, la2._stream_handle(None))


@pytest.mark.parametrize("case", [
    # dtype, B, H, N, block, causal, chunk_len   (chunk_len > 0 forces chunk states)
    ("bf16", 1, 2, 4096, 64, True, 512),
    ("bf16", 2, 2, 3000, 128, True, 1024),
    ("bf16", 1, 3, 777, 64, False, 0),
    ("f32", 1, 2, 1000, 64, True, 256),
])
def test_noalloc_matches_workspace_forward(la2, case):
    dt_name, B, H, N, block, causal, chunk = case
    d = 128 if dt_name == "bf16" else 64
    dt = la2.LA2_BF16 if dt_name == "bf16" else la2.LA2_F32
    la2.la2_set_chunk_len(chunk)
    try:
        need = la2.workspace_bytes(B, H, N, d, d, causal, block, dt, False)
        assert 0 < need <= la2.NOALLOC_SCRATCH_BYTES  # the scratch array is really used
        for call in range(2):
            ins = la2_inputs.make_custom(B, H, N, d, d, dt_name, seed=100 + call)
            q, k, v = (ins[n].cuda() for n in "qkv")
            ref = la2.forward(q, k, v, causal=causal, block=block)
            out = torch.full_like(ref, float("nan"))
            assert _noalloc(la2, q, k, v, out, causal, block, dt) == la2.LA2_OK
            assert la2.la2_check(la2._stream_handle(None)) == la2.LA2_OK
            assert _rel(out, ref) <= TOL[dt_name], f"call {call}"
    finally:
        la2.la2_set_chunk_len(0)


def test_noalloc_rejects_problems_beyond_the_array(la2):
    # non-causal always needs one 64 KiB state per (b, h): 1024 heads need 64 MiB
    dt = la2.LA2_BF16
    need = la2.workspace_bytes(1, 1024, 128, 128, 128, False, 64, dt, False)
    assert need > la2.NOALLOC_SCRATCH_BYTES
    null = ctypes.c_void_p(0)
    rc = la2.la2_forward_noalloc(null, null, null, null, 1, 1024, 128, 128, 128, 0, 64, dt,
                                 la2._stream_handle(None))
    assert rc == la2.LA2_ERR_WORKSPACE
    # invalid arguments are reported as by la2_forward
    assert la2.la2_forward_noalloc(null, null, null, null, 1, 1, 16, 128, 128, 3, 64, dt,
                                   la2._stream_handle(None)) == la2.LA2_ERR_INVALID_ARG
