"""GPU parity: libla2 (through its C ABI) against the float64 CPU oracle.

Bars (relative Frobenius error over the compared elements): 1e-5 for fp32
inputs, 1e-2 for bf16 inputs with fp32 accumulation; the same for O, dQ, dK
and dV. Outputs are pre-filled with NaN so an unwritten row fails the check.
"""

import math

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


def _dev(t):
    return t.to("cuda").contiguous()


def _nan_like(t, last=None):
    shape = t.shape if last is None else t.shape[:-1] + (last,)
    return torch.full(shape, float("nan"), dtype=t.dtype, device="cuda")


def run_forward(la2, ins, causal, block, chunk_len=0):
    la2.la2_set_chunk_len(chunk_len)
    try:
        q, k, v = (_dev(ins[n]) for n in "qkv")
        o = _nan_like(q, v.shape[-1])
        la2.forward(q, k, v, causal=causal, block=block, out=o)
        la2.check()
        return o.cpu()
    finally:
        la2.la2_set_chunk_len(0)


def run_backward(la2, ins, causal, block, chunk_len=0):
    la2.la2_set_chunk_len(chunk_len)
    try:
        q, k, v, do = (_dev(ins[n]) for n in ("q", "k", "v", "do"))
        outs = (_nan_like(q), _nan_like(k), _nan_like(v))
        la2.backward(q, k, v, do, causal=causal, block=block, outs=outs)
        la2.check()
        return tuple(t.cpu() for t in outs)
    finally:
        la2.la2_set_chunk_len(0)


def rel(x, ref):
    return oracle.relative_frobenius(x, ref)


# ------------------------------------------------------- fp32, 1 x 1 x 256 x 64


@pytest.mark.parametrize("causal", [True, False])
def test_fp32_small_forward(la2, causal):
    w = la2_inputs.WORKLOADS["fp32_small"]
    ins = la2_inputs.make_inputs(w)
    got = run_forward(la2, ins, causal, w.block)
    ref = oracle.forward(ins["q"], ins["k"], ins["v"], causal)
    assert rel(got, ref) <= TOL["f32"]


@pytest.mark.parametrize("causal", [True, False])
def test_fp32_small_backward(la2, causal):
    w = la2_inputs.WORKLOADS["fp32_small"]
    ins = la2_inputs.make_inputs(w, with_grad_out=True)
    got = run_backward(la2, ins, causal, w.block)
    ref = oracle.backward(ins["q"], ins["k"], ins["v"], ins["do"], causal)
    for g, r in zip(got, ref):
        assert rel(g, r) <= TOL["f32"]


# ---------------------------------------------------------------- edge cases

EDGE = [
    # dtype, B, H, N, d, dv, block, chunk_len
    ("f32", 1, 1, 1, 64, 64, 64, 0),          # one token
    ("f32", 1, 2, 37, 16, 24, 16, 0),         # N < 3 blocks, ragged, odd dims
    ("f32", 2, 3, 200, 32, 48, 32, 64),       # forced chunk split, ragged tail
    ("f32", 1, 1, 513, 64, 64, 64, 128),      # tail of one row in the last chunk
    ("f32", 1, 1, 300, 128, 128, 16, 0),
    ("f32", 1, 1, 257, 32, 32, 128, 0),       # block 128 at small d
    ("bf16", 1, 1, 1, 128, 128, 64, 0),
    ("bf16", 1, 1, 63, 128, 128, 64, 0),      # N < block
    ("bf16", 1, 2, 65, 128, 128, 64, 0),      # one full block + one row
    ("bf16", 2, 2, 1000, 128, 128, 128, 0),
    ("bf16", 1, 1, 4095, 128, 128, 64, 512),  # chunk split with ragged last block
    ("bf16", 1, 3, 777, 64, 64, 64, 128),
    ("bf16", 1, 2, 640, 64, 128, 128, 256),
    ("bf16", 1, 2, 384, 128, 64, 64, 0),
]


@pytest.mark.parametrize("case", EDGE, ids=lambda c: "-".join(map(str, c)))
@pytest.mark.parametrize("causal", [True, False])
def test_edge_forward(la2, case, causal):
    dt, B, H, N, d, dv, block, chunk = case
    ins = la2_inputs.make_custom(B, H, N, d, dv, dt, seed=N + d + block)
    got = run_forward(la2, ins, causal, block, chunk)
    ref = oracle.forward(ins["q"], ins["k"], ins["v"], causal)
    assert rel(got, ref) <= TOL[dt]
    # boundary rows of every block and chunk, each on its own
    step = chunk if chunk else block
    rows = sorted({r for s in range(0, N, block) for r in (s, min(N, s + block) - 1)}
                  | {r for s in range(0, N, step) for r in (s, min(N, s + step) - 1)})
    for r in rows:
        assert rel(got[:, :, r], ref[:, :, r]) <= 4 * TOL[dt]


@pytest.mark.parametrize("case", EDGE, ids=lambda c: "-".join(map(str, c)))
@pytest.mark.parametrize("causal", [True, False])
def test_edge_backward(la2, case, causal):
    dt, B, H, N, d, dv, block, chunk = case
    ins = la2_inputs.make_custom(B, H, N, d, dv, dt, seed=N + d + block + 1, with_grad_out=True)
    got = run_backward(la2, ins, causal, block, chunk)
    ref = oracle.backward(ins["q"], ins["k"], ins["v"], ins["do"], causal)
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        assert rel(g, r) <= TOL[dt], name


def test_empty_problem(la2):
    q = torch.empty((0, 2, 16, 64), device="cuda")
    o = la2.forward(q, q, q, block=64)
    assert o.shape == (0, 2, 16, 64)
    la2.check()


# ------------------------------------------------------ full-size workloads


def test_bf16_b4h16_n2k_forward(la2):
    w = la2_inputs.WORKLOADS["bf16_b4h16_n2k"]
    ins = la2_inputs.make_inputs(w)
    got = run_forward(la2, ins, True, w.block)
    ref = oracle.forward(ins["q"], ins["k"], ins["v"], True)
    assert rel(got, ref) <= TOL["bf16"]


@pytest.mark.parametrize("block", la2_inputs.SWEEP_BLOCKS)
@pytest.mark.parametrize("N", [1024, 4096, 16384])
def test_bf16_sweep_full(la2, N, block):
    w = la2_inputs.sweep_workload(N, block)
    ins = la2_inputs.make_inputs(w)
    got = run_forward(la2, ins, True, block)
    ref = oracle.forward(ins["q"], ins["k"], ins["v"], True)
    assert rel(got, ref) <= TOL["bf16"]


def _sampled_and_blocked(la2, w, heads_full=None):
    """Large sizes: sampled rows against the left product, and every row
    against the float64 block algorithm (pinned to the left product)."""
    ins = la2_inputs.make_inputs(w)
    got = run_forward(la2, ins, True, w.block)
    T = -(-w.N // w.block)
    starts = la2.plan_ranges(w.B, w.H, w.N, w.d, w.dv, True, w.block, la2.LA2_BF16)
    # rows on both sides of every range boundary inside a sequence
    edges = {r for f in starts[1:-1] if f % T for r in ((f % T) * w.block - 1, (f % T) * w.block)}
    rows = sorted(set(la2_inputs.sample_rows(w.N, w.block, w.seed)) | edges)
    ref_rows = oracle.forward_rows(ins["q"], ins["k"], ins["v"], rows, True)
    assert rel(got[:, :, rows], ref_rows) <= TOL["bf16"]
    for r_i, r in enumerate(rows[:: max(1, len(rows) // 64)]):
        idx = rows.index(r)
        assert rel(got[:, :, r], ref_rows[:, :, idx]) <= 4 * TOL["bf16"]
    num = den = 0.0
    for b in range(w.B):
        for h in range(w.H) if heads_full is None else heads_full:
            sl = (slice(b, b + 1), slice(h, h + 1))
            ref = oracle.blocked_forward(ins["q"][sl], ins["k"][sl], ins["v"][sl], 256, True)
            diff = got[sl].double().numpy() - ref
            num += float(np.sum(diff * diff))
            den += float(np.sum(ref * ref))
    assert math.sqrt(num / den) <= TOL["bf16"]


@pytest.mark.parametrize("block", la2_inputs.SWEEP_BLOCKS)
def test_bf16_sweep_64k(la2, block):
    _sampled_and_blocked(la2, la2_inputs.sweep_workload(65536, block), heads_full=range(0, 32, 4))


def test_bf16_long_512k(la2):
    _sampled_and_blocked(la2, la2_inputs.WORKLOADS["bf16_long_512k"], heads_full=[0, 7])


def test_bf16_fwdbwd_b2h32_n8k(la2):
    """The forward + backward workload, every element of O, dQ, dK and dV of all
    64 sequences against the float64 closed forms (article, "Lightning
    Attention-2简介", point 1; the backward's gradients of <dO, O>), and the
    first and last row of every block of every sequence on their own (chunk and
    range boundaries are block boundaries)."""
    w = la2_inputs.WORKLOADS["bf16_fwdbwd_b2h32_n8k"]
    ins = la2_inputs.make_inputs(w)
    o = run_forward(la2, ins, True, w.block)
    g = run_backward(la2, ins, True, w.block)
    ref_o = oracle.forward(ins["q"], ins["k"], ins["v"], True)
    assert rel(o, ref_o) <= TOL["bf16"]
    ref_g = oracle.backward(ins["q"], ins["k"], ins["v"], ins["do"], True)
    for name, gg, rr in zip(("dq", "dk", "dv"), g, ref_g):
        assert rel(gg, rr) <= TOL["bf16"], name
    rows = sorted({r for s0 in range(0, w.N, w.block) for r in (s0, s0 + w.block - 1)})
    got = (o,) + tuple(g)
    refs = (ref_o,) + tuple(ref_g)
    for name, x, r in zip(("o", "dq", "dk", "dv"), got, refs):
        xr = x[:, :, rows].double().numpy()
        rr = r[:, :, rows]
        num = np.sqrt(np.sum((xr - rr) ** 2, axis=-1))
        den = np.sqrt(np.sum(rr ** 2, axis=-1))
        assert np.all(num <= 4 * TOL["bf16"] * den), name


# ------------------------------------------- branches reached by forced splits


def test_noncausal_many_chunk_states(la2):
    """Tensor-core non-causal forward and backward with 16 chunk states per
    sequence: more than the map pass adds up itself, so the total is scanned
    into slot 0 first (article, point 1: without the mask O = Q (K^T V))."""
    B, H, N, block, chunk = 1, 2, 4096, 64, 256
    la2.la2_set_chunk_len(chunk)
    try:
        starts = la2.plan_ranges(B, H, N, 128, 128, False, block, la2.LA2_BF16)
    finally:
        la2.la2_set_chunk_len(0)
    assert len(starts) - 1 == B * H * (N // chunk)  # 16 chunk states per sequence
    ins = la2_inputs.make_custom(B, H, N, 128, 128, "bf16", seed=41, with_grad_out=True)
    got = run_forward(la2, ins, False, block, chunk)
    assert rel(got, oracle.forward(ins["q"], ins["k"], ins["v"], False)) <= TOL["bf16"]
    g = run_backward(la2, ins, False, block, chunk)
    ref = oracle.backward(ins["q"], ins["k"], ins["v"], ins["do"], False)
    for name, gg, rr in zip(("dq", "dk", "dv"), g, ref):
        assert rel(gg, rr) <= TOL["bf16"], name


@pytest.mark.parametrize("block", [64, 128])
def test_causal_split_beyond_range_table(la2, block):
    """A forced split into 256 chunks (more than the 160 ranges the persistent
    kernel's table holds): the forward and the backward's dQ pass run on the
    chunk kernels from scanned chunk prefixes (article, point 2: the state an
    inner block starts from is the sum over the earlier blocks)."""
    B, H, N, chunk = 1, 4, 16384, 256
    la2.la2_set_chunk_len(chunk)
    try:
        starts = la2.plan_ranges(B, H, N, 128, 128, True, block, la2.LA2_BF16)
    finally:
        la2.la2_set_chunk_len(0)
    assert len(starts) - 1 == B * H * N // chunk  # chunk boundaries, one per chunk
    ins = la2_inputs.make_custom(B, H, N, 128, 128, "bf16", seed=43 + block, with_grad_out=True)
    got = run_forward(la2, ins, True, block, chunk)
    ref = oracle.forward(ins["q"], ins["k"], ins["v"], True)
    assert rel(got, ref) <= TOL["bf16"]
    for r in sorted({r for s0 in range(0, N, chunk) for r in (s0, s0 + chunk - 1)}):
        assert rel(got[:, :, r], ref[:, :, r]) <= 4 * TOL["bf16"]
    g = run_backward(la2, ins, True, block, chunk)
    refg = oracle.backward(ins["q"], ins["k"], ins["v"], ins["do"], True)
    for name, gg, rr in zip(("dq", "dk", "dv"), g, refg):
        assert rel(gg, rr) <= TOL["bf16"], name


def test_ragged_tail_inside_a_range(la2):
    """Several sequences per persistent range with N mod 64 in 1..48 at Bk=64:
    the last block of a sequence leaves whole 16-row store groups past N, and
    the range runs on into the next sequence with the same staging tiles."""
    B, H, N = 2, 40, 777
    starts = la2.plan_ranges(B, H, N, 128, 128, True, 64, la2.LA2_BF16)
    T = -(-N // 64)
    # some range holds the end of one sequence and the start of the next
    assert any(starts[i] // T != (starts[i + 1] - 1) // T for i in range(len(starts) - 1))
    ins = la2_inputs.make_custom(B, H, N, 128, 128, "bf16", seed=47)
    got = run_forward(la2, ins, True, 64)
    ref = oracle.forward(ins["q"], ins["k"], ins["v"], True)
    assert rel(got, ref) <= TOL["bf16"]
    tail = list(range((T - 1) * 64, N))
    assert rel(got[:, :, tail], ref[:, :, tail]) <= TOL["bf16"]
