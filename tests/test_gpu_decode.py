"""Parity of the inference form (la2_kv_state + la2_decode_step) with the oracle.

A prefill of P tokens through la2_kv_state, then T single-token steps through
la2_decode_step, must give the rows P..P+T-1 of the causal left product of the
whole sequence (article "Lightning Attention-2 新一代注意力机制", speed section:
the lossless RNN form), and the state must equal sum_t k_t^T v_t.
Tolerances: the bf16 and fp32 bounds of the forward (relative Frobenius 1e-2 /
1e-5); the fp32 state of bf16 inputs is held to 1e-5 (products of bf16 values
are exact in fp32, only the order of the adds differs).
"""

import numpy as np
import pytest
import torch

import oracle
from linear_attention_la2_b200 import inputs as la2_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def la2():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_la2_b200 import build

    build.build()
    from linear_attention_la2_b200 import la2 as lib

    return lib


CASES = [
    # dtype, B, H, P (prefill), d, dv, T (decode steps)
    ("bf16", 2, 3, 200, 128, 128, 17),   # tensor-core chunk states
    ("bf16", 1, 2, 4100, 128, 128, 3),   # several chunks per sequence
    ("bf16", 1, 4, 1000, 64, 64, 9),     # CUDA-core chunk states
    ("f32", 2, 2, 300, 64, 32, 11),
    ("f32", 1, 3, 0, 32, 40, 5),         # no prefill; dv not a multiple of 32
    ("f32", 1, 2, 50, 16, 30, 4),        # dv not a multiple of 4: one column per lane
    ("bf16", 3, 1, 64, 64, 128, 6),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_prefill_then_decode_matches_causal_forward(la2, case):
    dt, B, H, P, d, dv, T = case
    ins = la2_inputs.make_custom(B, H, P + T, d, dv, dt, seed=P + T + d)
    q, k, v = ins["q"], ins["k"], ins["v"]
    ref = oracle.forward(q, k, v, True)[:, :, P:]
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    state = torch.zeros((B, H, d, dv), dtype=torch.float32, device="cuda")
    la2.kv_state(kd[:, :, :P].contiguous(), vd[:, :, :P].contiguous(), state)
    torch.cuda.synchronize()
    la2.check()
    if P:
        ref_state = oracle.kv_state(k[:, :, :P], v[:, :, :P])
        assert oracle.relative_frobenius(state.cpu().double().numpy(), ref_state) <= 1e-5
    outs = []
    for t in range(P, P + T):
        outs.append(la2.decode_step(qd[:, :, t].contiguous(), kd[:, :, t].contiguous(),
                                    vd[:, :, t].contiguous(), state))
    torch.cuda.synchronize()
    la2.check()
    got = torch.stack(outs, dim=2).cpu().double().numpy()
    tol = 1e-2 if dt == "bf16" else 1e-5
    assert oracle.relative_frobenius(got, ref) <= tol
    assert oracle.relative_frobenius(state.cpu().double().numpy(), oracle.kv_state(k, v)) <= 1e-5


def test_kv_state_accumulates_and_repeats_bitwise(la2):
    ins = la2_inputs.make_custom(2, 2, 3000, 128, 128, "bf16", seed=7)
    k, v = ins["k"].cuda(), ins["v"].cuda()
    first = la2.kv_state(k[:, :, :1700].contiguous(), v[:, :, :1700].contiguous())
    both = la2.kv_state(k[:, :, 1700:].contiguous(), v[:, :, 1700:].contiguous(), first.clone())
    again = la2.kv_state(k[:, :, 1700:].contiguous(), v[:, :, 1700:].contiguous(), first.clone())
    torch.cuda.synchronize()
    la2.check()
    assert torch.equal(both, again)  # fixed summation order
    ref = oracle.kv_state(ins["k"], ins["v"])
    assert oracle.relative_frobenius(both.cpu().double().numpy(), ref) <= 1e-5


def test_decode_step_full_workload(la2):
    """One step at the decode benchmark's size (B=64, H=32, d=dv=128, bf16) from a
    random fp32 state, every head against the oracle's step."""
    B, H, d, dv = 64, 32, 128, 128
    g = torch.Generator().manual_seed(11)
    q, k, v = ((torch.randn((B, H, n), generator=g) / np.sqrt(d)).to(torch.bfloat16)
               for n in (d, d, dv))
    s0 = torch.randn((B, H, d, dv), generator=g) * 0.1
    state = s0.cuda()
    o = la2.decode_step(q.cuda(), k.cuda(), v.cuda(), state)
    torch.cuda.synchronize()
    la2.check()
    ref_o, ref_s = oracle.decode_step(q, k, v, s0)
    assert oracle.relative_frobenius(o.cpu().double().numpy(), ref_o) <= 1e-2
    assert oracle.relative_frobenius(state.cpu().double().numpy(), ref_s) <= 1e-6


@pytest.mark.parametrize("dt,d,dv", [("f32", 160, 36), ("f32", 128, 64), ("bf16", 96, 128),
                                     ("bf16", 200, 128)])
def test_decode_step_from_random_state(la2, dt, d, dv):
    """Decode steps from a random fp32 state, without a prefill: d above 128 runs
    the one-column-per-lane kernel, d <= 128 with dv % 4 == 0 the kernel that holds
    all of a thread's state rows in registers."""
    B, H, T = 3, 2, 4
    g = torch.Generator().manual_seed(d + dv)
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    q, k, v = ((torch.randn((B, H, T, n), generator=g) / np.sqrt(d)).to(tdt) for n in (d, d, dv))
    s = torch.randn((B, H, d, dv), generator=g) * 0.1
    state = s.cuda()
    outs = [la2.decode_step(q[:, :, t].cuda(), k[:, :, t].cuda(), v[:, :, t].cuda(), state)
            for t in range(T)]
    torch.cuda.synchronize()
    la2.check()
    tol = 1e-2 if dt == "bf16" else 1e-5
    for t in range(T):
        ref_o, s = oracle.decode_step(q[:, :, t], k[:, :, t], v[:, :, t], s)
        assert oracle.relative_frobenius(outs[t].cpu().double().numpy(), ref_o) <= tol
    assert oracle.relative_frobenius(state.cpu().double().numpy(), s) <= 1e-6
