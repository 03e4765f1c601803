"""Pins of the sequence-parallel oracle (one part of a sequence whose other
parts are summarised by KV states): forward_from_state, backward_from_states.

They are checked against the already pinned full-sequence definition (forward,
backward, kv_state) by cutting a sequence into parts, against exact directional
derivatives (the loss is linear in each input), and on a hand-worked example.
Article, "Lightning Attention-2简介", point 2: the inter-block term is the
queries times the KV state of everything earlier.
"""

import numpy as np
import pytest
import torch

import oracle


def _rand(shape, g):
    return torch.randn(shape, generator=g, dtype=torch.float64)


@pytest.mark.parametrize("cut", [1, 17, 40])
def test_forward_of_the_second_part_matches_the_whole(cut):
    g = torch.Generator().manual_seed(cut)
    B, H, N, d, dv = 2, 3, 57, 5, 6
    q, k, v = _rand((B, H, N, d), g), _rand((B, H, N, d), g), _rand((B, H, N, dv), g)
    whole = oracle.forward(q, k, v, True)
    state = oracle.kv_state(k[:, :, :cut], v[:, :, :cut])
    tail = oracle.forward_from_state(q[:, :, cut:], k[:, :, cut:], v[:, :, cut:], state)
    assert np.allclose(tail, whole[:, :, cut:], rtol=0, atol=1e-11)
    # a zero state is the plain forward
    zero = np.zeros((B, H, d, dv))
    assert np.allclose(oracle.forward_from_state(q, k, v, zero), whole, rtol=0, atol=0)


def test_three_parts_chain_through_summed_states():
    g = torch.Generator().manual_seed(3)
    B, H, N, d, dv = 1, 2, 90, 4, 4
    q, k, v = _rand((B, H, N, d), g), _rand((B, H, N, d), g), _rand((B, H, N, dv), g)
    whole = oracle.forward(q, k, v, True)
    cuts = [0, 30, 60, 90]
    states = [oracle.kv_state(k[:, :, a:b], v[:, :, a:b]) for a, b in zip(cuts, cuts[1:])]
    for i, (a, b) in enumerate(zip(cuts, cuts[1:])):
        prefix = sum(states[:i]) if i else np.zeros((B, H, d, dv))
        part = oracle.forward_from_state(q[:, :, a:b], k[:, :, a:b], v[:, :, a:b], prefix)
        assert np.allclose(part, whole[:, :, a:b], rtol=0, atol=1e-11)


@pytest.mark.parametrize("cuts", [(0, 25, 70), (0, 1, 70), (0, 69, 70)])
def test_backward_of_each_part_matches_the_whole(cuts):
    g = torch.Generator().manual_seed(sum(cuts))
    B, H, N, d, dv = 1, 2, 70, 5, 3
    q, k, v = _rand((B, H, N, d), g), _rand((B, H, N, d), g), _rand((B, H, N, dv), g)
    do = _rand((B, H, N, dv), g)
    dq, dk, dvv = oracle.backward(q, k, v, do, True)
    bounds = list(cuts) + [N] if cuts[-1] != N else list(cuts)
    parts = list(zip(bounds, bounds[1:]))
    for a, b in parts:
        prefix = oracle.kv_state(k[:, :, :a], v[:, :, :a])
        suffix = oracle.kv_state(q[:, :, b:], do[:, :, b:])  # sum_t q_t^T dO_t after the part
        sl = (slice(None), slice(None), slice(a, b))
        gq, gk, gv = oracle.backward_from_states(q[sl], k[sl], v[sl], do[sl], prefix, suffix)
        assert np.allclose(gq, dq[sl], rtol=0, atol=1e-10)
        assert np.allclose(gk, dk[sl], rtol=0, atol=1e-10)
        assert np.allclose(gv, dvv[sl], rtol=0, atol=1e-10)


def test_backward_from_states_exact_directional_derivatives():
    """L = sum_t <dO_t, O_t> over the part with its outside summarised by states;
    L is linear in each of q, k, v, so L(x + E) - L(x) = <dX, E> exactly."""
    g = torch.Generator().manual_seed(11)
    B, H, N, d, dv = 1, 1, 9, 3, 2
    q, k, v = _rand((B, H, N, d), g), _rand((B, H, N, d), g), _rand((B, H, N, dv), g)
    do = _rand((B, H, N, dv), g)
    P, U = _rand((B, H, d, dv), g), _rand((B, H, d, dv), g)

    def loss(q_, k_, v_):
        # the part's own output from prefix P, plus what later queries (summed
        # into U = sum q^T dO) read from this part's keys and values
        o = oracle.forward_from_state(q_, k_, v_, P)
        later = float(np.einsum("bhnd,bhne,bhde->", k_.numpy(), v_.numpy(), U.numpy()))
        return float(np.sum(o * do.numpy())) + later

    gq, gk, gv = oracle.backward_from_states(q, k, v, do, P, U)
    for which, grad in ((0, gq), (1, gk), (2, gv)):
        args = [q, k, v]
        E = _rand(args[which].shape, g)
        moved = list(args)
        moved[which] = args[which] + E
        delta = loss(*moved) - loss(*args)
        assert abs(delta - float(np.sum(grad * E.numpy()))) <= 1e-9 * (1 + abs(delta))


def test_hand_worked_forward_from_state():
    # one token: o = q P + (q . k) v with q = [1, 2], k = [3, 0], v = [1, -1],
    # P = [[1, 0], [0, 2]]: q P = [1, 4], q . k = 3 -> o = [1 + 3, 4 - 3] = [4, 1]
    q = torch.tensor([[[[1.0, 2.0]]]], dtype=torch.float64)
    k = torch.tensor([[[[3.0, 0.0]]]], dtype=torch.float64)
    v = torch.tensor([[[[1.0, -1.0]]]], dtype=torch.float64)
    P = np.array([[[[1.0, 0.0], [0.0, 2.0]]]])
    assert oracle.forward_from_state(q, k, v, P).tolist() == [[[[4.0, 1.0]]]]


def test_planted_mistake_is_caught():
    """A prefix applied as P^T (a transposed state) breaks the part identity."""
    g = torch.Generator().manual_seed(5)
    q, k, v = _rand((1, 1, 20, 4), g), _rand((1, 1, 20, 4), g), _rand((1, 1, 20, 4), g)
    whole = oracle.forward(q, k, v, True)
    state = oracle.kv_state(k[:, :, :8], v[:, :, :8])
    wrong = oracle.forward_from_state(q[:, :, 8:], k[:, :, 8:], v[:, :, 8:],
                                      np.swapaxes(state, -1, -2))
    assert not np.allclose(wrong, whole[:, :, 8:], atol=1e-6)
