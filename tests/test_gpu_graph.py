"""CUDA-graph capture of the library's launches.

Every call of the C ABI enqueues plain kernel launches on the caller's stream
with caller-owned workspace, so a captured sequence of calls replays exactly:
the test captures forward and backward calls of the range-split forward
(pre-pass and range-state plans) and of the backward (split dK/dV with the
in-kernel suffix state), replays the graph on new inputs copied into the same
buffers, and compares bit for bit with direct calls on those inputs.
"""

import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def la2():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_la2_b200 import build

    build.build()
    from linear_attention_la2_b200 import la2 as lib

    return lib


@pytest.mark.parametrize("B,H,N,block", [(4, 16, 2048, 64), (1, 4, 65536, 128), (2, 8, 3000, 64)])
def test_graph_replay_matches_direct_calls(la2, B, H, N, block):
    g = torch.Generator(device="cuda").manual_seed(N + H)

    def draw():
        return tuple((torch.randn(B, H, N, 128, device="cuda", generator=g) * 0.088).to(torch.bfloat16)
                     for _ in range(4))

    q, k, v, do = draw()
    o = torch.empty_like(q)
    grads = tuple(torch.empty_like(q) for _ in range(3))
    wsf = torch.empty(max(la2.workspace_bytes(B, H, N, 128, 128, True, block, la2.LA2_BF16, False), 1),
                      dtype=torch.uint8, device="cuda")
    wsb = torch.empty(max(la2.workspace_bytes(B, H, N, 128, 128, True, block, la2.LA2_BF16, True), 1),
                      dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()

    def calls():
        la2.forward(q, k, v, causal=True, block=block, out=o, workspace=wsf, stream=s)
        la2.backward(q, k, v, do, causal=True, block=block, outs=grads, workspace=wsb, stream=s)

    with torch.cuda.stream(s):
        calls()  # warm-up: kernel attributes set outside the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        calls()
    new = draw()
    for dst, src in zip((q, k, v, do), new):
        dst.copy_(src)
    torch.cuda.synchronize()
    graph.replay()
    torch.cuda.synchronize()
    la2.check()
    got = (o.clone(),) + tuple(t.clone() for t in grads)
    with torch.cuda.stream(s):
        calls()
    torch.cuda.synchronize()
    la2.check()
    for a, b in zip(got, (o,) + grads):
        assert torch.equal(a, b)
