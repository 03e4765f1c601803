"""Pins of the oracle for grouped K/V heads (GQA/MQA): a layout of the same op
(article "Lightning Attention-2 新一代注意力机制", section "Lightning Attention-2简介",
point 1: O = ((Q K^T) ⊙ M) V per head). Each query head h reads K/V head
h // (H / Hkv). Pinned by replicating K/V heads through the plain forward, by
torch float64 autograd, and by a hand-worked example."""

import numpy as np
import pytest
import torch

import oracle
from oracle import la2_oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("H,Hkv", [(4, 4), (4, 2), (6, 1)])
@pytest.mark.parametrize("causal", [True, False])
def test_gqa_equals_forward_on_replicated_kv(H, Hkv, causal):
    B, N, d, dv = 2, 13, 4, 3
    q, k, v = _rand((B, H, N, d), 1), _rand((B, Hkv, N, d), 2), _rand((B, Hkv, N, dv), 3)
    rep = H // Hkv
    ref = oracle.forward(q, np.repeat(k, rep, axis=1), np.repeat(v, rep, axis=1), causal)
    assert oracle.relative_frobenius(oracle.forward_gqa(q, k, v, causal), ref) < 1e-14


def test_gqa_hand_example():
    # two query heads share one K/V head; N = 2, d = dv = 1
    q = np.array([[[[1.0], [2.0]], [[3.0], [-1.0]]]])      # [1, 2, 2, 1]
    k = np.array([[[[2.0], [5.0]]]])                         # [1, 1, 2, 1]
    v = np.array([[[[1.0], [10.0]]]])
    # head 0: o0 = 1*2*1 = 2, o1 = 2*2*1 + 2*5*10 = 104
    # head 1: o0 = 3*2*1 = 6, o1 = -1*2*1 + -1*5*10 = -52
    expect = np.array([[[[2.0], [104.0]], [[6.0], [-52.0]]]])
    assert np.array_equal(oracle.forward_gqa(q, k, v, True), expect)


@pytest.mark.parametrize("causal", [True, False])
def test_gqa_gradients_match_autograd(causal):
    B, H, Hkv, N, d, dv = 1, 4, 2, 9, 3, 2
    q, k, v = _rand((B, H, N, d), 10), _rand((B, Hkv, N, d), 11), _rand((B, Hkv, N, dv), 12)
    do = _rand((B, H, N, dv), 13)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    rep = H // Hkv
    kk, vv = tk.repeat_interleave(rep, dim=1), tv.repeat_interleave(rep, dim=1)
    S = tq @ kk.transpose(-1, -2)
    if causal:
        S = S * torch.tril(torch.ones(N, N, dtype=torch.float64))
    (S @ vv * torch.tensor(do)).sum().backward()
    got = oracle.backward_gqa(q, k, v, do, causal)
    for g, t in zip(got, (tq, tk, tv)):
        assert oracle.relative_frobenius(g, t.grad.numpy()) < 1e-12


def test_gqa_rejects_a_head_count_that_does_not_divide():
    with pytest.raises(ValueError):
        oracle.forward_gqa(_rand((1, 3, 4, 2), 0), _rand((1, 2, 4, 2), 1), _rand((1, 2, 4, 2), 2))


def test_pins_reject_a_wrong_head_map():
    """Mapping query head h to K/V head h % Hkv (interleaved) instead of h // g
    fails the replication pin."""
    B, H, Hkv, N, d, dv = 1, 4, 2, 7, 3, 2
    q, k, v = _rand((B, H, N, d), 20), _rand((B, Hkv, N, d), 21), _rand((B, Hkv, N, dv), 22)
    wrong = np.stack([la2_oracle.forward(q[:, h:h + 1], k[:, h % Hkv:h % Hkv + 1],
                                         v[:, h % Hkv:h % Hkv + 1], True)[:, 0] for h in range(H)], 1)
    ref = oracle.forward(q, np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1), True)
    assert oracle.relative_frobenius(wrong, ref) > 1e-3
