"""Pins of the float64 oracle against what the article and the mathematics fix.

The article ("Lightning Attention-2 新一代注意力机制", section
"Lightning Attention-2简介") gives the left product O = ((Q K^T) ⊙ M) V (point 1),
the right product Q (K^T V) in the unmasked case (point 1, Fig. 2), the block
split with an accumulated KV state (point 2, Fig. 3) and, in its speed section,
the lossless RNN form. None of these pins calls the oracle to check itself:
each compares it with an independent computation or a value fixed by hand.
"""

import json
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import la2_oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _brute_force(q, k, v, causal):
    """Pure-Python loops: build the full N x N score matrix, mask it, multiply."""
    N, d = len(q), len(q[0])
    dv = len(v[0])
    A = [[sum(q[t][c] * k[s][c] for c in range(d)) for s in range(N)] for t in range(N)]
    if causal:
        A = [[A[t][s] if s <= t else 0 for s in range(N)] for t in range(N)]
    return [[sum(A[t][s] * v[s][e] for s in range(N)) for e in range(dv)] for t in range(N)]


# ---------------------------------------------------------------- fixed values


def test_hand_worked_examples(golden_dir):
    with open(os.path.join(golden_dir, "hand_examples.json")) as f:
        data = json.load(f)
    for ex in data["examples"]:
        q = np.array(ex["q"], float)[None, None]
        k = np.array(ex["k"], float)[None, None]
        v = np.array(ex["v"], float)[None, None]
        assert np.array_equal(oracle.forward(q, k, v, True)[0, 0], np.array(ex["o_causal"], float))
        assert np.array_equal(oracle.forward(q, k, v, False)[0, 0], np.array(ex["o_noncausal"], float))
        if "do" in ex:
            do = np.array(ex["do"], float)[None, None]
            dq, dk, dv = oracle.backward(q, k, v, do, True)
            assert np.array_equal(dq[0, 0], np.array(ex["dq_causal"], float))
            assert np.array_equal(dk[0, 0], np.array(ex["dk_causal"], float))
            assert np.array_equal(dv[0, 0], np.array(ex["dv_causal"], float))


@pytest.mark.parametrize("N,d,dv", [(1, 1, 1), (2, 3, 2), (5, 2, 4), (8, 4, 3), (7, 4, 4)])
@pytest.mark.parametrize("causal", [True, False])
def test_brute_force_integer_inputs(N, d, dv, causal):
    rng = np.random.default_rng(N * 100 + d * 10 + dv)
    q = rng.integers(-3, 4, (1, 2, N, d)).astype(float)
    k = rng.integers(-3, 4, (1, 2, N, d)).astype(float)
    v = rng.integers(-3, 4, (1, 2, N, dv)).astype(float)
    got = oracle.forward(q, k, v, causal)
    for h in range(2):
        ref = _brute_force(q[0, h].tolist(), k[0, h].tolist(), v[0, h].tolist(), causal)
        assert np.array_equal(got[0, h], np.array(ref, float))  # exact: integer sums


@pytest.mark.parametrize("N,d,dv", [(1, 8, 4), (9, 3, 5), (130, 16, 8)])
def test_all_ones_closed_form(N, d, dv):
    q = np.ones((1, 1, N, d))
    k = np.ones((1, 1, N, d))
    v = np.ones((1, 1, N, dv))
    t = np.arange(N, dtype=float)[:, None]
    assert np.array_equal(oracle.forward(q, k, v, True)[0, 0], np.broadcast_to((t + 1) * d, (N, dv)))
    assert np.array_equal(oracle.forward(q, k, v, False)[0, 0], np.full((N, dv), float(N * d)))


def test_single_token():
    q, k, v = _rand((2, 3, 1, 5), 1), _rand((2, 3, 1, 5), 2), _rand((2, 3, 1, 7), 3)
    ref = np.einsum("bhnc,bhnc->bhn", q, k)[..., None] * v
    np.testing.assert_allclose(oracle.forward(q, k, v, True), ref, rtol=1e-14, atol=0)


# ------------------------------------------------------------ identities


@pytest.mark.parametrize("N", [1, 17, 200])
def test_equals_rnn_form(N):
    q, k, v = _rand((2, 2, N, 8), 4), _rand((2, 2, N, 8), 5), _rand((2, 2, N, 6), 6)
    err = oracle.relative_frobenius(oracle.forward(q, k, v, True), oracle.recurrent_forward(q, k, v))
    assert err <= 1e-12


@pytest.mark.parametrize("block", [1, 7, 64, 128, 300])
def test_block_size_invariance(block):
    N = 300
    q, k, v = _rand((1, 2, N, 16), 7), _rand((1, 2, N, 16), 8), _rand((1, 2, N, 12), 9)
    ref = oracle.forward(q, k, v, True)
    assert oracle.relative_frobenius(oracle.blocked_forward(q, k, v, block, True), ref) <= 1e-12


def test_noncausal_associativity():
    q, k, v = _rand((2, 2, 150, 16), 10), _rand((2, 2, 150, 16), 11), _rand((2, 2, 150, 8), 12)
    right = np.einsum("bhnc,bhce->bhne", q, np.einsum("bhnc,bhne->bhce", k, v))
    assert oracle.relative_frobenius(oracle.forward(q, k, v, False), right) <= 1e-12
    assert oracle.relative_frobenius(oracle.blocked_forward(q, k, v, 32, False), right) <= 1e-12


def test_rows_match_full():
    q, k, v, do = (_rand((1, 2, 600, 8), s) for s in (13, 14, 15, 16))
    rows = [0, 1, 63, 64, 511, 512, 599]
    for causal in (True, False):
        full = oracle.forward(q, k, v, causal)
        np.testing.assert_allclose(oracle.forward_rows(q, k, v, rows, causal), full[:, :, rows],
                                   rtol=1e-12, atol=1e-12)
        gq, gk, gv = oracle.backward(q, k, v, do, causal)
        rq, rk, rv = oracle.backward_rows(q, k, v, do, rows, causal)
        for a, b in ((rq, gq), (rk, gk), (rv, gv)):
            np.testing.assert_allclose(a, b[:, :, rows], rtol=1e-10, atol=1e-10)


# ------------------------------------------------------------- gradients


def _loss(q, k, v, do, causal):
    return float(np.sum(oracle.forward(q, k, v, causal) * do))


@pytest.mark.parametrize("causal", [True, False])
def test_gradient_exact_directional(causal):
    """O is linear in each of Q, K, V, so L(X+E) - L(X) = <dX, E> exactly."""
    shp = (1, 2, 40, 6)
    q, k, v, do = (_rand(shp, s) for s in (20, 21, 22, 23))
    dq, dk, dv = oracle.backward(q, k, v, do, causal)
    base = _loss(q, k, v, do, causal)
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        E = _rand(shp, 30 + len(name))
        args = {"q": q, "k": k, "v": v}
        args[name] = args[name] + E
        delta = _loss(args["q"], args["k"], args["v"], do, causal) - base
        assert abs(delta - float(np.sum(grad * E))) <= 1e-9 * max(1.0, abs(delta))


@pytest.mark.parametrize("causal", [True, False])
def test_gradient_euler_identity(causal):
    """L is linear in each input, so <dQ,Q> = <dK,K> = <dV,V> = <dO,O> = L."""
    q, k, v, do = (_rand((2, 1, 70, 5), s) for s in (40, 41, 42, 43))
    dq, dk, dv = oracle.backward(q, k, v, do, causal)
    L = np.sum(oracle.forward(q, k, v, causal) * do)
    for g, x in ((dq, q), (dk, k), (dv, v)):
        assert abs(np.sum(g * x) - L) <= 1e-10 * abs(L)


@pytest.mark.parametrize("causal", [True, False])
def test_gradient_matches_autograd(causal):
    """torch autograd (float64) differentiates a plain masked product."""
    q, k, v, do = (_rand((1, 2, 50, 8), s) for s in (50, 51, 52, 53))
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    S = tq @ tk.transpose(-1, -2)
    if causal:
        S = S * torch.tril(torch.ones(50, 50, dtype=torch.float64))
    (S @ tv).backward(torch.tensor(do))
    dq, dk, dv = oracle.backward(q, k, v, do, causal)
    for a, b in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert oracle.relative_frobenius(a, b) <= 1e-12


# ------------------------------------------------- planted mistakes are caught


def _mutant_forward_strict_mask(q, k, v, causal=True):
    """A plausible mistake: the mask drops the diagonal."""
    S = q @ np.swapaxes(k, -1, -2)
    N = q.shape[2]
    return np.where(np.tri(N, k=-1, dtype=bool), S, 0.0) @ v


def _mutant_forward_transposed(q, k, v, causal=True):
    """A plausible mistake: the mask is applied to (K Q^T)."""
    S = k @ np.swapaxes(q, -1, -2)
    N = q.shape[2]
    return np.where(np.tri(N, dtype=bool), S, 0.0) @ v


@pytest.mark.parametrize("mutant", [_mutant_forward_strict_mask, _mutant_forward_transposed])
def test_pins_reject_planted_forward_mistakes(mutant, monkeypatch):
    q, k, v = _rand((1, 1, 20, 4), 60), _rand((1, 1, 20, 4), 61), _rand((1, 1, 20, 3), 62)
    monkeypatch.setattr(la2_oracle, "forward", mutant)
    rnn_err = oracle.relative_frobenius(la2_oracle.forward(q, k, v, True),
                                        oracle.recurrent_forward(q, k, v))
    ones = np.ones((1, 1, 6, 2))
    t = np.arange(6, dtype=float)[:, None]
    ones_ok = np.array_equal(la2_oracle.forward(ones, ones, ones, True)[0, 0],
                             np.broadcast_to((t + 1) * 2, (6, 2)))
    qi = np.array([[1.0, 0.0], [0.0, 1.0]])[None, None]
    ki = np.array([[2.0, 3.0], [5.0, 7.0]])[None, None]
    vi = np.array([[1.0], [10.0]])[None, None]
    hand_ok = np.array_equal(la2_oracle.forward(qi, ki, vi, True)[0, 0], np.array([[2.0], [73.0]]))
    assert rnn_err > 1e-3 or not ones_ok or not hand_ok
    assert not hand_ok  # the hand-worked example alone catches both mistakes


def test_pins_reject_planted_gradient_mistake():
    """dK taken as dP Q instead of dP^T Q fails the exact directional pin."""
    shp = (1, 1, 12, 3)
    q, k, v, do = (_rand(shp, s) for s in (70, 71, 72, 73))
    N = shp[2]
    keep = np.tri(N, dtype=bool)
    dP = np.where(keep, do[0, 0] @ v[0, 0].T, 0.0)
    wrong_dk = (dP @ q[0, 0])[None, None]
    E = _rand(shp, 74)
    delta = _loss(q, k + E, v, do, True) - _loss(q, k, v, do, True)
    assert abs(delta - float(np.sum(wrong_dk * E))) > 1e-6


def test_relative_frobenius_basic():
    a = np.array([3.0, 4.0])
    assert oracle.relative_frobenius(a, a) == 0.0
    assert abs(oracle.relative_frobenius(a * 1.01, a) - 0.01) < 1e-12
    assert oracle.relative_frobenius(np.zeros(2), np.zeros(2)) == 0.0


def test_seeded_inputs_recipe():
    """The shared generator: fixed seed -> fixed values, scaled by 1/sqrt(d)."""
    from linear_attention_la2_b200.inputs import WORKLOADS, make_inputs

    w = WORKLOADS["fp32_small"]
    a = make_inputs(w)
    b = make_inputs(w)
    assert all(torch.equal(a[n], b[n]) for n in "qkv")
    assert a["q"].shape == (1, 1, 256, 64) and a["q"].dtype == torch.float32
    g = torch.Generator().manual_seed(0)
    first = torch.randn((1, 1, 256, 64), generator=g) / 8.0
    assert torch.equal(a["q"], first)
    bf = make_inputs(WORKLOADS["bf16_b4h16_n2k"])
    assert bf["v"].dtype == torch.bfloat16 and bf["v"].shape == (4, 16, 2048, 128)
    assert 0.05 < float(bf["k"].float().std()) < 0.12  # N(0,1)/sqrt(128) ~ 0.088
