"""Sequence parallelism on one GPU: a sequence cut into parts that run as if on
different ranks (each part from the summed states of the others, through the C
ABI calls la2_kv_state, la2_forward_sp, la2_backward_sp), compared with the
float64 oracle of the whole sequence. The exchange between ranks is tested on
CPU ranks (tests/test_multirank_cpu.py); here the gathered states are stacked
on one device, which is what the all-gather produces on each rank.
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


CASES = [
    # dtype, B, H, N (whole), d, block, parts
    ("bf16", 1, 8, 8192, 128, 64, 2),
    ("bf16", 2, 4, 3000, 128, 128, 3),     # ragged parts
    ("bf16", 1, 2, 20000, 128, 64, 4),     # several chunks per part
    ("bf16", 1, 3, 777, 64, 64, 2),        # CUDA-core path
    ("f32", 1, 2, 600, 64, 64, 3),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_parts_reproduce_the_whole_sequence(la2, case):
    dt, B, H, N, d, block, parts = case
    ins = la2_inputs.make_custom(B, H, N, d, d, dt, seed=N + parts, with_grad_out=True)
    cuts = [N * i // parts for i in range(parts + 1)]
    dev = {n: t.cuda() for n, t in ins.items()}
    sl = [(slice(None), slice(None), slice(a, b)) for a, b in zip(cuts, cuts[1:])]
    part = [{n: t[s].contiguous() for n, t in dev.items()} for s in sl]
    # what each rank contributes to the exchange
    kv = torch.stack([la2.kv_state(p["k"], p["v"]) for p in part])
    qdo = torch.stack([la2.kv_state(p["q"], p["do"]) for p in part])
    outs, grads = [], []
    for r, p in enumerate(part):
        outs.append(la2.forward_sp(p["q"], p["k"], p["v"], kv[:r], block=block))
        grads.append(la2.backward_sp(p["q"], p["k"], p["v"], p["do"], kv[:r], qdo[r + 1:],
                                     block=block))
    la2.check()
    o = torch.cat([x.cpu() for x in outs], dim=2)
    assert oracle.relative_frobenius(o, oracle.forward(ins["q"], ins["k"], ins["v"], True)) <= TOL[dt]
    ref = oracle.backward(ins["q"], ins["k"], ins["v"], ins["do"], True)
    for i, name in enumerate(("dq", "dk", "dv")):
        g = torch.cat([x[i].cpu() for x in grads], dim=2)
        assert oracle.relative_frobenius(g, ref[i]) <= TOL[dt], name
    # every part on its own against the oracle of one part (first and last rows)
    for r, (a, b) in enumerate(zip(cuts, cuts[1:])):
        before = oracle.kv_state(ins["k"][:, :, :a], ins["v"][:, :, :a])
        ref_r = oracle.forward_from_state(ins["q"][sl[r]], ins["k"][sl[r]], ins["v"][sl[r]], before)
        assert oracle.relative_frobenius(outs[r].cpu()[:, :, [0, -1]], ref_r[:, :, [0, -1]]) <= 4 * TOL[dt]


def test_first_part_without_states_is_the_plain_forward(la2):
    ins = la2_inputs.make_custom(1, 4, 1024, 128, 128, "bf16", seed=3)
    q, k, v = (ins[n].cuda() for n in "qkv")
    o = la2.forward_sp(q, k, v, None, block=64)
    la2.check()
    ref = oracle.forward(ins["q"], ins["k"], ins["v"], True)
    assert oracle.relative_frobenius(o.cpu(), ref) <= TOL["bf16"]
