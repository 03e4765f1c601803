"""Pins of the decayed form in the float64 oracle.

The decayed form is a reading (the article gives no decay): per head h a rate
lam in [0, 1], ``KV_t = lam KV_{t-1} + k_t^T v_t`` and ``o_t = q_t KV_t``, i.e. the
causal mask of the left product ``O = ((Q K^T) ⊙ M) V`` (article "Lightning
Attention-2 新一代注意力机制", section "Lightning Attention-2简介", point 1)
becomes ``D[t, s] = lam^(t-s)``. Every pin compares the oracle with an independent
computation or a value fixed by the mathematics: the recurrence, the article's op
at lam = 1, the diagonal-only closed form at lam = 0, exact rational brute force
at lam = 1/2, a hand example, and exact directional derivatives of a product that
is linear in each of q, k and v.
"""

from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _inputs(B, H, N, d, dv, seed):
    return _rand((B, H, N, d), seed), _rand((B, H, N, d), seed + 1), _rand((B, H, N, dv), seed + 2)


def test_hand_example():
    # d = dv = 1, lam = 1/2, q = (1, 2, 3), k = (1, 1, 1), v = (1, 2, 4):
    # o_0 = 1*1*1 = 1; o_1 = 2*(1/2*1 + 2) = 5; o_2 = 3*(1/4*1 + 1/2*2 + 4) = 15.75
    q = np.array([1.0, 2.0, 3.0]).reshape(1, 1, 3, 1)
    k = np.ones((1, 1, 3, 1))
    v = np.array([1.0, 2.0, 4.0]).reshape(1, 1, 3, 1)
    assert np.array_equal(oracle.forward_decay(q, k, v, [0.5])[0, 0, :, 0], [1.0, 5.0, 15.75])
    # dO = ones: dv_s = sum_{t>=s} lam^(t-s) q_t k_s -> (1 + 1 + 0.75, 2 + 1.5, 3) = (2.75, 3.5, 3)
    _, _, dv = oracle.backward_decay(q, k, v, np.ones((1, 1, 3, 1)), [0.5])
    assert np.array_equal(dv[0, 0, :, 0], [2.75, 3.5, 3.0])


@pytest.mark.parametrize("N,d,dv", [(1, 1, 1), (4, 2, 3), (7, 3, 2)])
def test_brute_force_rationals_half(N, d, dv):
    """lam = 1/2 and integer inputs: every term is a dyadic rational, so the
    float64 oracle must equal exact rational arithmetic bit for bit."""
    rng = np.random.default_rng(N * 10 + d)
    q = rng.integers(-3, 4, (1, 1, N, d)).astype(float)
    k = rng.integers(-3, 4, (1, 1, N, d)).astype(float)
    v = rng.integers(-3, 4, (1, 1, N, dv)).astype(float)
    got = oracle.forward_decay(q, k, v, [0.5])[0, 0]
    half = Fraction(1, 2)
    for t in range(N):
        for e in range(dv):
            ref = sum(half ** (t - s) * sum(Fraction(int(q[0, 0, t, c])) * int(k[0, 0, s, c]) for c in range(d))
                      * int(v[0, 0, s, e]) for s in range(t + 1))
            assert got[t, e] == float(ref)


@pytest.mark.parametrize("lam", [0.0, 0.3, 0.9, 0.999, 1.0])
def test_left_product_equals_recurrence(lam):
    q, k, v = _inputs(2, 2, 67, 5, 3, 11)
    lams = [lam, 0.5]
    a = oracle.forward_decay(q, k, v, lams)
    b = oracle.recurrent_forward_decay(q, k, v, lams)
    assert oracle.relative_frobenius(a, b) <= 1e-12


def test_rate_one_is_the_article_op():
    q, k, v = _inputs(1, 3, 90, 4, 6, 21)
    a = oracle.forward_decay(q, k, v, [1.0, 1.0, 1.0])
    assert oracle.relative_frobenius(a, oracle.forward(q, k, v, True)) <= 1e-13
    do = _rand((1, 3, 90, 6), 24)
    for g, r in zip(oracle.backward_decay(q, k, v, do, [1.0] * 3), oracle.backward(q, k, v, do, True)):
        assert oracle.relative_frobenius(g, r) <= 1e-13


def test_rate_zero_keeps_the_diagonal():
    q, k, v = _inputs(1, 1, 20, 4, 3, 31)
    got = oracle.forward_decay(q, k, v, [0.0])[0, 0]
    ref = np.sum(q[0, 0] * k[0, 0], axis=1)[:, None] * v[0, 0]  # o_t = (q_t . k_t) v_t
    assert np.allclose(got, ref, rtol=0, atol=1e-13)


def test_rates_are_per_head():
    q, k, v = _inputs(1, 2, 30, 3, 3, 41)
    both = oracle.forward_decay(q, k, v, [0.2, 0.8])
    h0 = oracle.forward_decay(q[:, :1], k[:, :1], v[:, :1], [0.2])
    h1 = oracle.forward_decay(q[:, 1:], k[:, 1:], v[:, 1:], [0.8])
    assert np.array_equal(both[:, :1], h0) and np.array_equal(both[:, 1:], h1)


@pytest.mark.parametrize("which", ["q", "k", "v"])
def test_directional_derivatives_are_exact(which):
    """O is linear in each of q, k, v: <dO, O(x + dx) - O(x)> = <grad_x, dx>."""
    q, k, v = _inputs(1, 2, 40, 4, 3, 51)
    do = _rand((1, 2, 40, 3), 55)
    lams = [0.7, 0.95]
    grads = dict(zip("qkv", oracle.backward_decay(q, k, v, do, lams)))
    args = {"q": q, "k": k, "v": v}
    dx = _rand(args[which].shape, 57)
    moved = dict(args)
    moved[which] = args[which] + dx
    lhs = np.sum(do * (oracle.forward_decay(moved["q"], moved["k"], moved["v"], lams)
                       - oracle.forward_decay(q, k, v, lams)))
    rhs = np.sum(grads[which] * dx)
    assert abs(lhs - rhs) <= 1e-10 * max(1.0, abs(rhs))


def test_gradients_against_autograd():
    q, k, v = (torch.tensor(x, requires_grad=True) for x in _inputs(1, 2, 25, 3, 4, 61))
    do = torch.tensor(_rand((1, 2, 25, 4), 65))
    lam = torch.tensor([0.6, 0.85], dtype=torch.float64)
    N = 25
    gap = torch.arange(N)[:, None] - torch.arange(N)[None, :]
    D = torch.where(gap >= 0, lam[:, None, None] ** gap.clamp(min=0), torch.zeros(()))  # [H, N, N]
    o = ((q @ k.transpose(-1, -2)) * D[None]) @ v
    (o * do).sum().backward()
    got = oracle.backward_decay(q.detach(), k.detach(), v.detach(), do, lam.numpy())
    for g, ref in zip(got, (q.grad, k.grad, v.grad)):
        assert oracle.relative_frobenius(g, ref.numpy()) <= 1e-12


def test_pins_reject_a_shifted_exponent():
    """A plausible mistake (lam^(t-s+1): the own token decayed once) fails the
    recurrence pin."""
    q, k, v = _inputs(1, 1, 30, 3, 3, 71)
    lam = 0.8
    N = 30
    gap = np.arange(N)[:, None] - np.arange(N)[None, :]
    D1 = np.where(gap >= 0, lam ** (np.maximum(gap, 0) + 1), 0.0)
    wrong = ((q[0, 0] @ k[0, 0].T) * D1) @ v[0, 0]
    ref = oracle.recurrent_forward_decay(q, k, v, [lam])[0, 0]
    assert oracle.relative_frobenius(wrong, ref) > 1e-3


def test_rejects_wrong_rate_count():
    q, k, v = _inputs(1, 2, 5, 2, 2, 81)
    with pytest.raises(ValueError):
        oracle.forward_decay(q, k, v, [0.5])


@pytest.mark.parametrize("N,lams", [(1, [0.5]), (9, [0.0, 1.0]), (40, [0.7, 0.95])])
def test_backward_as_forwards_on_reversed_rows(N, lams):
    """The gradients are decayed forwards: dQ = F(dO, V, K), and with row t moved
    to N-1-t (R), dV = R F(R K, R Q, R dO) and dK = R F(R V, R dO, R Q) (the
    sums over later rows become sums over earlier ones with the same gaps). The
    tensor-core backward is built on this identity; here both sides are the
    oracle's own, independently written forward and backward."""
    H = len(lams)
    q, k, v = _inputs(1, H, N, 4, 3, 91)
    do = _rand((1, H, N, 3), 95)
    gq, gk, gv = oracle.backward_decay(q, k, v, do, lams)
    rev = lambda x: x[:, :, ::-1]
    assert oracle.relative_frobenius(oracle.forward_decay(do, v, k, lams), gq) <= 1e-12
    assert oracle.relative_frobenius(rev(oracle.forward_decay(rev(k), rev(q), rev(do), lams)), gv) <= 1e-12
    assert oracle.relative_frobenius(rev(oracle.forward_decay(rev(v), rev(do), rev(q), lams)), gk) <= 1e-12
