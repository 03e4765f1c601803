"""GPU parity of the decayed causal form (la2_forward_decay / la2_backward_decay)
with the float64 oracle.

The decayed form is a reading (the article gives no decay): per head a rate lam,
``KV_t = lam KV_{t-1} + k_t^T v_t``; the oracle's ``forward_decay`` /
``backward_decay`` are pinned in tests/test_oracle_decay.py. Cases cover one and
several chunks a sequence (the decayed chunk states and their decayed prefix /
suffix scans), ragged tails, per-head rates, lam = 0 and lam = 1, fp32 and bf16.
Tolerances: relative Frobenius 1e-5 (fp32) and 1e-2 (bf16), as for the plain op.
"""

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


def rel(x, ref):
    return oracle.relative_frobenius(x, ref)


def run(la2, ins, lam, block, chunk=0, grad=False):
    la2.la2_set_chunk_len(chunk)
    try:
        q, k, v = (ins[n].cuda() for n in "qkv")
        rates = torch.tensor(lam, dtype=torch.float32, device="cuda")
        o = torch.full(q.shape[:3] + (v.shape[-1],), float("nan"), dtype=q.dtype, device="cuda")
        la2.forward_decay(q, k, v, rates, block=block, out=o)
        la2.check()
        if not grad:
            return o.cpu()
        do = ins["do"].cuda()
        outs = tuple(torch.full_like(t, float("nan")) for t in (q, k, v))
        la2.backward_decay(q, k, v, do, rates, block=block, outs=outs)
        la2.check()
        return o.cpu(), tuple(t.cpu() for t in outs)
    finally:
        la2.la2_set_chunk_len(0)


CASES = [
    # dtype, B, H, N, d, dv, block, chunk_len, rates
    ("f32", 1, 2, 200, 32, 48, 32, 0, [0.9, 0.5]),
    ("f32", 2, 3, 777, 64, 64, 64, 128, [0.99, 0.7, 1.0]),     # several chunks, ragged tail
    ("f32", 1, 1, 300, 16, 24, 16, 64, [0.0]),                 # lam = 0: the diagonal only
    ("f32", 1, 2, 513, 64, 32, 64, 0, [1.0, 1.0]),             # lam = 1: the plain op
    ("bf16", 1, 2, 1000, 128, 128, 64, 0, [0.995, 0.9]),       # tensor cores both ways
    ("bf16", 2, 2, 4096, 64, 64, 64, 512, [0.999, 0.98]),      # eight chunks a sequence
    ("bf16", 1, 3, 650, 128, 64, 64, 256, [0.5, 0.97, 1.0]),
    ("bf16", 2, 2, 1537, 128, 128, 128, 0, [0.99, 0.7]),       # tensor cores, block 128, odd N
    ("bf16", 1, 2, 3001, 128, 128, 128, 256, [0.999, 0.95]),   # twelve chunks: the decayed scan
    ("bf16", 1, 2, 2100, 128, 128, 64, 512, [0.0, 1.0]),       # five chunks summed in the kernel
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c[:8])))
def test_decay_forward_backward(la2, case):
    dt, B, H, N, d, dv, block, chunk, lam = case
    ins = la2_inputs.make_custom(B, H, N, d, dv, dt, seed=N + d + H, with_grad_out=True)
    o, (dq, dk, dv_) = run(la2, ins, lam, block, chunk, grad=True)
    assert rel(o, oracle.forward_decay(ins["q"], ins["k"], ins["v"], lam)) <= TOL[dt]
    rq, rk, rv = oracle.backward_decay(ins["q"], ins["k"], ins["v"], ins["do"], lam)
    assert rel(dq, rq) <= TOL[dt]
    assert rel(dk, rk) <= TOL[dt]
    assert rel(dv_, rv) <= TOL[dt]
    # rows on both sides of every chunk and block edge, each on its own
    step = chunk if chunk else block
    rows = sorted({r for s in range(0, N, step) for r in (max(0, s - 1), s)} | {N - 1})
    ref = oracle.forward_decay(ins["q"], ins["k"], ins["v"], lam)
    for r in rows:
        assert rel(o[:, :, r], ref[:, :, r]) <= 4 * TOL[dt]


@pytest.mark.parametrize("block,chunk,lam", [(128, 0, [0.99, 0.8]), (128, 512, [0.0, 0.999]),
                                             (64, 256, [0.5, 1.0]), (64, 0, [0.97, 0.9])])
def test_decay_forward_tensor_cores(la2, block, chunk, lam):
    """bf16 d = dv = 128: the decayed forward on the tensor-core chunk kernels
    (decayed chunk states, their decayed prefix, scaled Q and K rows, the
    state decayed in TMEM), one and several chunks, lam = 0 and 1."""
    B, H, N = 2, 2, 3000
    ins = la2_inputs.make_custom(B, H, N, 128, 128, "bf16", seed=block + chunk)
    o = run(la2, ins, lam, block, chunk)
    ref = oracle.forward_decay(ins["q"], ins["k"], ins["v"], lam)
    assert rel(o, ref) <= TOL["bf16"]
    step = chunk if chunk else block
    for r in sorted({r for s in range(0, N, step) for r in (max(0, s - 1), s)} | {N - 1}):
        assert rel(o[:, :, r], ref[:, :, r]) <= 4 * TOL["bf16"]


def test_decay_rates_are_per_head(la2):
    """The same inputs under rates permuted between heads: each head follows its
    own rate (a wrong head index would mix them)."""
    ins = la2_inputs.make_custom(2, 2, 300, 32, 32, "f32", seed=11)
    same = {n: torch.cat([ins[n][:, :1], ins[n][:, :1]], dim=1).contiguous() for n in "qkv"}
    o = run(la2, same, [0.3, 0.95], 32, 64)
    assert rel(o[:, 0], oracle.forward_decay(same["q"], same["k"], same["v"], [0.3, 0.95])[:, 0]) <= 1e-5
    assert rel(o[:, 1], oracle.forward_decay(same["q"], same["k"], same["v"], [0.3, 0.95])[:, 1]) <= 1e-5
    assert rel(o[:, 0], o[:, 1]) > 1e-2


@pytest.mark.parametrize("N,block", [(1, 64), (63, 64), (65, 64), (130, 128), (1, 128), (257, 128)])
def test_decay_forward_tensor_cores_edges(la2, N, block):
    """The tensor-core decayed forward on one token, fewer rows than a block, a
    block plus a row and ragged tails (rows past N are zero in the tiles; the
    scaled Q and K rows there stay zero)."""
    lam = [0.9, 0.6]
    ins = la2_inputs.make_custom(1, 2, N, 128, 128, "bf16", seed=N + block)
    o = run(la2, ins, lam, block)
    assert rel(o, oracle.forward_decay(ins["q"], ins["k"], ins["v"], lam)) <= TOL["bf16"]


@pytest.mark.parametrize("N,block", [(1, 64), (2, 128), (63, 64), (129, 128), (200, 64)])
def test_decay_backward_tensor_cores_edges(la2, N, block):
    """The tensor-core decayed backward (three decayed forwards, two of them on
    the time-reversed rows) on one and two tokens, under a block, a block plus a
    row and a ragged tail: the in-place reversal of dK and dV leaves an odd N's
    middle row where it is."""
    lam = [0.8, 0.97]
    ins = la2_inputs.make_custom(1, 2, N, 128, 128, "bf16", seed=3 * N + block, with_grad_out=True)
    _, (dq, dk, dv_) = run(la2, ins, lam, block, grad=True)
    rq, rk, rv = oracle.backward_decay(ins["q"], ins["k"], ins["v"], ins["do"], lam)
    assert rel(dq, rq) <= TOL["bf16"]
    assert rel(dk, rk) <= TOL["bf16"]
    assert rel(dv_, rv) <= TOL["bf16"]


def test_decay_backward_runs_on_tensor_cores(la2):
    """bf16 d = dv = 128: the backward launches the tensor-core chunk kernels and
    the row reversal, and no CUDA-core attention kernel."""
    ins = la2_inputs.make_custom(1, 2, 700, 128, 128, "bf16", seed=5, with_grad_out=True)
    torch.cuda.synchronize()
    assert la2.la2_profile_enable(1) == la2.LA2_OK
    try:
        run(la2, ins, [0.9, 0.99], 64, 256, grad=True)
        torch.cuda.synchronize()
        ran = {}
        for kid in range(la2.la2_profile_num_kernels()):
            n, _ = la2.la2_profile_collect(kid)
            if n:
                ran[la2.la2_profile_kernel_name(kid)] = n
    finally:
        la2.la2_profile_enable(0)
    assert ran.get("la2_reverse_rows") == 2
    assert ran.get("la2_fwd_sm100", 0) >= 4  # the forward, then dQ, dV, dK
    assert not any(name.endswith("_simt") for name in ran), ran
