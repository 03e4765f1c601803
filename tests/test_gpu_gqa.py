"""GPU parity of grouped K/V heads (GQA; MQA with one K/V head) through the C
ABI (la2_forward_gqa / la2_backward_gqa) against the float64 oracle.

Source: cccbook long-context chapter, section on MQA/GQA, and mhpn.cn blog,
section 3 (query heads share a key/value head); each query head computes the
op of "Lightning Attention-2简介", point 1, with its group's K and V.

Expected values: oracle.forward_gqa / backward_gqa at small N; at larger N the
plain oracle on K/V heads repeated per query head (forward) and its per-head
gradients summed over each group (dK, dV) - the identities tests/test_oracle_gqa.py
pins forward_gqa / backward_gqa to. Bars as in the other parity tests.
"""

import numpy as np
import pytest
import torch

import oracle
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


def make(B, H, Hkv, N, d, dt, seed, grad=False):
    """Query-side tensors [B,H,N,.] and K/V [B,Hkv,N,.], drawn with the input
    recipe (q, k, v, dO of a [B,H,N,.] draw; K/V keep their first Hkv heads)."""
    ins = la2_inputs.make_custom(B, H, N, d, d, dt, seed=seed, with_grad_out=grad)
    ins["k"] = ins["k"][:, :Hkv].contiguous()
    ins["v"] = ins["v"][:, :Hkv].contiguous()
    return ins


def rep(x, H):
    """K/V heads repeated per query head: head h <- K/V head h // (H // Hkv)."""
    return x.repeat_interleave(H // x.shape[1], dim=1)


def ref_forward(ins, causal):
    H = ins["q"].shape[1]
    if ins["q"].shape[2] <= 2048:
        return oracle.forward_gqa(ins["q"], ins["k"], ins["v"], causal)
    return oracle.forward(ins["q"], rep(ins["k"], H), rep(ins["v"], H), causal)


def ref_backward(ins, causal):
    q, k, v, do = ins["q"], ins["k"], ins["v"], ins["do"]
    H, Hkv = q.shape[1], k.shape[1]
    if q.shape[2] <= 2048:
        return oracle.backward_gqa(q, k, v, do, causal)
    dq, dk, dv = oracle.backward(q, rep(k, H), rep(v, H), do, causal)
    B, N = q.shape[0], q.shape[2]
    g = H // Hkv
    return (dq, dk.reshape(B, Hkv, g, N, -1).sum(axis=2), dv.reshape(B, Hkv, g, N, -1).sum(axis=2))


def run(la2, ins, causal, block, chunk=0, grad=False):
    la2.la2_set_chunk_len(chunk)
    try:
        q, k, v = (ins[n].cuda() for n in "qkv")
        o = torch.full(q.shape[:3] + (v.shape[-1],), float("nan"), dtype=q.dtype, device="cuda")
        la2.forward(q, k, v, causal=causal, block=block, out=o)
        la2.check()
        if not grad:
            return o.cpu()
        do = ins["do"].cuda()
        outs = tuple(torch.full_like(t, float("nan")) for t in (q, k, v))
        la2.backward(q, k, v, do, causal=causal, block=block, outs=outs)
        la2.check()
        return o.cpu(), tuple(t.cpu() for t in outs)
    finally:
        la2.la2_set_chunk_len(0)


def rel(x, ref):
    return oracle.relative_frobenius(x, ref)


CASES = [
    # dtype, B, H, Hkv, N, d, block, chunk_len
    ("bf16", 1, 32, 8, 1024, 128, 64, 0),     # GQA, tensor cores, pre-pass split
    ("bf16", 1, 8, 1, 2000, 128, 128, 0),     # MQA, Bk=128 (dK/dV in 64-row tiles)
    ("bf16", 2, 8, 2, 777, 128, 64, 0),       # ragged tail, ranges across sequences
    ("bf16", 1, 8, 2, 4096, 128, 64, 128),    # forced split beyond the range table: chunk path
    ("bf16", 1, 4, 1, 8192, 128, 64, 0),      # one K/V head, many chunk states in the backward
    ("bf16", 1, 6, 3, 500, 64, 64, 0),        # CUDA-core path (d = 64)
    ("f32", 1, 4, 2, 300, 64, 64, 0),         # fp32, CUDA cores
    ("f32", 2, 6, 1, 200, 32, 32, 64),        # fp32 MQA, forced chunk split
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
@pytest.mark.parametrize("causal", [True, False])
def test_gqa_forward_backward(la2, case, causal):
    dt, B, H, Hkv, N, d, block, chunk = case
    ins = make(B, H, Hkv, N, d, dt, seed=N + H + Hkv, grad=True)
    o, (dq, dk, dv) = run(la2, ins, causal, block, chunk, grad=True)
    assert rel(o, ref_forward(ins, causal)) <= TOL[dt]
    rq, rk, rv = ref_backward(ins, causal)
    assert rel(dq, rq) <= TOL[dt]
    assert rel(dk, rk) <= TOL[dt]
    assert rel(dv, rv) <= TOL[dt]


def test_gqa_with_range_states(la2):
    """Long sequences at small B*H: the range split sums per-range states of
    the query sequences, whose K/V come from the group's K/V head. Sampled rows
    against the left product, two whole heads against the block algorithm."""
    B, H, Hkv, N, block = 1, 4, 1, 65536, 128
    starts = la2.plan_ranges(B, H, N, 128, 128, True, block, la2.LA2_BF16)
    assert len(starts) - 1 > B * H  # sequences are split
    ins = make(B, H, Hkv, N, 128, "bf16", seed=91)
    got = run(la2, ins, True, block)
    rows = la2_inputs.sample_rows(N, block, 91, count=64)
    kr, vr = rep(ins["k"], H), rep(ins["v"], H)
    ref_rows = oracle.forward_rows(ins["q"], kr, vr, rows, True)
    assert rel(got[:, :, rows], ref_rows) <= TOL["bf16"]
    for h in (0, 3):
        sl = (slice(0, 1), slice(h, h + 1))
        ref = oracle.blocked_forward(ins["q"][sl], kr[sl], vr[sl], 256, True)
        assert rel(got[sl], ref) <= TOL["bf16"]


def test_gqa_with_one_group_is_the_plain_op(la2):
    """Hkv = H runs the same kernels as la2_forward / la2_backward: identical bits."""
    ins = la2_inputs.make_custom(1, 4, 512, 128, 128, "bf16", seed=5, with_grad_out=True)
    q, k, v, do = (ins[n].cuda() for n in ("q", "k", "v", "do"))
    o1 = la2.forward(q, k, v, block=64)
    g1 = la2.backward(q, k, v, do, block=64)
    B, H, N, d = q.shape
    o2 = torch.empty_like(o1)
    ws = torch.empty(max(1, la2.workspace_bytes(B, H, N, d, d, True, 64, la2.LA2_BF16, False)),
                     dtype=torch.uint8, device="cuda")
    assert la2.la2_forward(la2._ptr(q), la2._ptr(k), la2._ptr(v), la2._ptr(o2), B, H, N, d, d, 1, 64,
                           la2.LA2_BF16, la2._ptr(ws), ws.numel(), la2._stream_handle(None)) == 0
    la2.check()
    assert torch.equal(o1, o2)
    ref = oracle.backward(ins["q"], ins["k"], ins["v"], ins["do"], True)
    for g, r in zip(g1, ref):
        assert rel(g.cpu(), r) <= TOL["bf16"]
