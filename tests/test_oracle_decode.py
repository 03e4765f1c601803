"""Pins of the oracle's inference form: the state after a prefill and one
RNN-mode step (article "Lightning Attention-2 新一代注意力机制", speed section:
linear attention converts losslessly to an RNN; section "Lightning Attention-2简介",
point 2: the KV state accumulated block after block).

Each pin compares the oracle with an independent computation: pure-Python loops
over integer inputs (exact), the masked or unmasked left product, or values worked
by hand.
"""

import numpy as np
import pytest

import oracle
from oracle import la2_oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _ints(shape, seed):
    return np.random.default_rng(seed).integers(-3, 4, size=shape).astype(np.float64)


def _left_product_rows(q, k, v):
    """Pure-Python causal left product of one sequence (lists of lists)."""
    N, d, dv = len(q), len(q[0]), len(v[0])
    out = []
    for t in range(N):
        row = []
        for e in range(dv):
            row.append(sum(sum(q[t][c] * k[s][c] for c in range(d)) * v[s][e] for s in range(t + 1)))
        out.append(row)
    return out


def _decode_all(step, q, k, v, state):
    """Run `step` token by token over [B,H,N,*] inputs from `state`."""
    outs = []
    for t in range(q.shape[2]):
        o, state = step(q[:, :, t], k[:, :, t], v[:, :, t], state)
        outs.append(o)
    if not outs:
        return np.zeros(q.shape[:2] + (0, v.shape[3])), state
    return np.stack(outs, axis=2), state


def _decode_error_vs_loops(step):
    q, k, v = _ints((1, 1, 9, 3), 1), _ints((1, 1, 9, 3), 2), _ints((1, 1, 9, 2), 3)
    got, _ = _decode_all(step, q, k, v, np.zeros((1, 1, 3, 2)))
    ref = np.array(_left_product_rows(q[0, 0].tolist(), k[0, 0].tolist(), v[0, 0].tolist()))
    return float(np.max(np.abs(got[0, 0] - ref)))


def test_decode_hand_example():
    q, k, v = np.array([[[1.0, 1.0]]]), np.array([[[1.0, 0.0]]]), np.array([[[2.0]]])
    state = np.array([[[[1.0], [3.0]]]])
    o, new = oracle.decode_step(q, k, v, state)
    # new = state + k^T v = [[1+2], [3+0]]; o = q new = 3 + 3
    assert np.array_equal(new, np.array([[[[3.0], [3.0]]]]))
    assert np.array_equal(o, np.array([[[6.0]]]))


def test_kv_state_hand_example():
    k = np.array([[[[1.0, 2.0], [3.0, 4.0]]]])
    v = np.array([[[[5.0], [6.0]]]])
    # sum_t k_t^T v_t = [[1*5 + 3*6], [2*5 + 4*6]]
    assert np.array_equal(oracle.kv_state(k, v), np.array([[[[23.0], [34.0]]]]))
    assert np.array_equal(oracle.kv_state(k, v, np.ones((1, 1, 2, 1))), np.array([[[[24.0], [35.0]]]]))


def test_decode_steps_equal_left_product_exactly():
    assert _decode_error_vs_loops(oracle.decode_step) == 0.0


@pytest.mark.parametrize("P", [0, 1, 17, 40])
def test_decode_continues_from_prefill_state(P):
    shp = (2, 3, 40, 5)
    q, k, v = _rand(shp, 10), _rand(shp, 11), _rand((2, 3, 40, 4), 12)
    state = oracle.kv_state(k[:, :, :P], v[:, :, :P])
    got, final = _decode_all(oracle.decode_step, q[:, :, P:], k[:, :, P:], v[:, :, P:], state)
    ref = oracle.forward(q, k, v, True)[:, :, P:]
    if P < 40:
        assert oracle.relative_frobenius(got, ref) < 1e-12
    # the state after the last step is the state of the whole sequence
    assert oracle.relative_frobenius(final, oracle.kv_state(k, v)) < 1e-12


def test_kv_state_is_the_unmasked_right_factor():
    """Unit-vector queries through the unmasked left product read K^T V row by row."""
    N, d, dv = 11, 4, 3
    k, v = _rand((1, 2, N, d), 20), _rand((1, 2, N, dv), 21)
    q = np.zeros((1, 2, N, d))
    for i in range(d):
        q[:, :, i, i] = 1.0
    rows = oracle.forward(q, k, v, causal=False)[:, :, :d]
    assert oracle.relative_frobenius(oracle.kv_state(k, v), rows) < 1e-13


def _mutant_decode_old_state(q, k, v, state):
    """A plausible mistake: the output reads the state before the token's own pair."""
    o = np.einsum("bhd,bhde->bhe", q, state)
    return o, state + k[..., :, None] * v[..., None, :]


def test_pins_reject_decode_without_own_pair():
    assert _decode_error_vs_loops(_mutant_decode_old_state) > 0.0
