"""CPU float64 oracle for Lightning Attention-2 causal linear attention.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or run
this module. The CUDA library never calls it, and it shares no code, table or
helper with the CUDA path.

Source of every formula: the news article "Lightning Attention-2 新一代注意力机制"
(youleyou.com), section "Lightning Attention-2简介":

* point 1 (with Fig. 2): with softmax removed, the output is the *left product*
  ``O = ((Q K^T) ⊙ M) V``; ``M`` is the lower-triangular all-ones mask in the
  unidirectional (GPT) case and is dropped in the bidirectional case, where
  associativity gives the *right product* ``O = Q (K^T V)``;
* point 2 (with Fig. 3): Q, K, V are cut into the same number of blocks; inside a
  block the masked left product is kept, across blocks the right product is used
  with a KV state that is accumulated for the next block, and the two partial
  outputs are added to give ``O_i``;
* section "Lightning Attention-2速度对比": linear attention converts losslessly
  to an RNN at inference (one token at a time with a constant-size state).

Readings where the article is silent (each is listed in the design notes):

* ``M`` includes the diagonal (token t attends to itself);
* no normalisation, no ``1/sqrt(d)`` inside the op, no feature map, no decay;
* tensors are ``[B, H, N, d]`` (``dv`` for V and O), each (b, h) independent;
* gradients are those of ``L = <dO, O>`` for the closed form above.

All arithmetic is float64 on the exact (already rounded) input values.
``forward`` / ``backward`` / ``*_rows`` are the plain definition. ``recurrent_*``
is the RNN form and ``blocked_forward`` the block algorithm of point 2; those two
exist to pin the definition (and to check very long sequences where the O(N^2)
definition is too slow on a CPU), never the other way round. ``kv_state`` (the
state after a prefill) and ``decode_step`` (one RNN-mode step) are the oracle of
the inference form; ``forward_gqa`` / ``backward_gqa`` the oracle of grouped K/V
heads (a layout of the same op: each query head reads the K/V head of its group);
``forward_from_state`` / ``backward_from_states`` the oracle of one part of a
sequence whose other parts are summarised by KV states (sequence parallelism).

Decay (``forward_decay``, ``backward_decay``, ``recurrent_forward_decay``) is a
reading, not an article formula: the article has no decay, and the only nearby
text on the pages is a one-line mention of data-dependent gating (gated linear
attention). The reading is the plainest decayed form of the same op: per head h
a rate ``lam_h`` in [0, 1] multiplies the KV state before each token,
``KV_t = lam KV_{t-1} + k_t^T v_t``, i.e. the causal mask becomes
``D[t, s] = lam^(t - s)`` for ``s <= t``. It reduces to the article's op at
``lam = 1``. Its pins are mathematical (``tests/test_oracle_decay.py``): equality
of the left product and the recurrence, ``lam = 1`` against ``forward``,
``lam = 0`` against its closed form, brute force on integers at ``lam = 1/2``,
exact directional derivatives.

Parity status: every function here is pinned by ``tests/test_oracle.py``
(brute force on tiny integer inputs, closed forms, RNN-form equality, block-size
invariance, associativity, exact directional derivatives, autograd).
"""

from __future__ import annotations

import numpy as np

# Rows of scores held at once by the row-group loops below. It only bounds
# memory (ROW_GROUP x N float64); every output row is still its own sum.
ROW_GROUP = 512


def _f64(x) -> np.ndarray:
    """Upcast a torch tensor or array to a float64 numpy array."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover - torch is always present here
        pass
    return np.asarray(x, dtype=np.float64)


def _check(q, k, v):
    if q.ndim != 4 or k.shape != q.shape or v.shape[:3] != q.shape[:3]:
        raise ValueError("expected q,k [B,H,N,d] and v [B,H,N,dv]")


def forward(q, k, v, causal: bool = True) -> np.ndarray:
    """Left product ``O = ((Q K^T) ⊙ M) V`` for every (b, h).

    Row t of O is ``sum_{s in mask(t)} (q_t . k_s) v_s`` with ``mask(t) = {0..t}``
    when ``causal`` and ``{0..N-1}`` otherwise (article, point 1).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    _check(q, k, v)
    B, H, N, _ = q.shape
    out = np.empty(q.shape[:3] + (v.shape[3],), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            K, V = k[b, h], v[b, h]
            for r0 in range(0, N, ROW_GROUP):
                r1 = min(N, r0 + ROW_GROUP)
                S = q[b, h, r0:r1] @ K.T  # scores q_t . k_s, shape [rows, N]
                if causal:
                    t = np.arange(r0, r1)[:, None]
                    s = np.arange(N)[None, :]
                    S = np.where(s <= t, S, 0.0)  # M: lower-triangular ones, diagonal kept
                out[b, h, r0:r1] = S @ V
    return out


def forward_rows(q, k, v, rows, causal: bool = True) -> np.ndarray:
    """The same definition evaluated only at the given output rows.

    Returns ``[B, H, len(rows), dv]``. Used at sizes where the full O(N^2)
    product is too slow on a CPU.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    _check(q, k, v)
    rows = np.asarray(rows, dtype=np.int64)
    B, H, N, _ = q.shape
    out = np.empty((B, H, len(rows), v.shape[3]), dtype=np.float64)
    group = max(1, min(64, (1 << 27) // max(1, N * 8)))
    for b in range(B):
        for h in range(H):
            K, V = k[b, h], v[b, h]
            for g0 in range(0, len(rows), group):
                rr = rows[g0:g0 + group]
                S = q[b, h, rr] @ K.T
                if causal:
                    S = np.where(np.arange(N)[None, :] <= rr[:, None], S, 0.0)
                out[b, h, g0:g0 + len(rr)] = S @ V
    return out


def backward(q, k, v, do, causal: bool = True):
    """Closed-form gradients of ``L = <dO, O>`` with ``O = ((Q K^T) ⊙ M) V``.

    With ``P = (Q K^T) ⊙ M`` and ``dP = (dO V^T) ⊙ M``:
    ``dQ = dP K``, ``dK = dP^T Q``, ``dV = P^T dO``.
    Returns ``(dq, dk, dv)`` as float64 arrays.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    _check(q, k, v)
    B, H, N, _ = q.shape
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dvv = np.empty_like(v)
    for b in range(B):
        for h in range(H):
            Q, K, V, dO = q[b, h], k[b, h], v[b, h], do[b, h]
            dk_acc = np.zeros_like(K)
            dv_acc = np.zeros_like(V)
            for r0 in range(0, N, ROW_GROUP):
                r1 = min(N, r0 + ROW_GROUP)
                P = Q[r0:r1] @ K.T
                dP = dO[r0:r1] @ V.T
                if causal:
                    keep = np.arange(N)[None, :] <= np.arange(r0, r1)[:, None]
                    P = np.where(keep, P, 0.0)
                    dP = np.where(keep, dP, 0.0)
                dq[b, h, r0:r1] = dP @ K
                dk_acc += dP.T @ Q[r0:r1]
                dv_acc += P.T @ dO[r0:r1]
            dk[b, h] = dk_acc
            dvv[b, h] = dv_acc
    return dq, dk, dvv


def backward_rows(q, k, v, do, rows, causal: bool = True):
    """Rows of the closed-form gradients, one output row at a time.

    ``dq_t = sum_{s<=t} (do_t . v_s) k_s``;
    ``dk_s = sum_{t>=s} (do_t . v_s) q_t``;
    ``dv_s = sum_{t>=s} (q_t . k_s) do_t`` (all s, t for the non-causal case).
    Returns three ``[B, H, len(rows), .]`` arrays.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    rows = np.asarray(rows, dtype=np.int64)
    B, H, N, d = q.shape
    dvd = v.shape[3]
    dq = np.empty((B, H, len(rows), d))
    dk = np.empty((B, H, len(rows), d))
    dvv = np.empty((B, H, len(rows), dvd))
    group = max(1, min(64, (1 << 27) // max(1, N * 8)))
    cols = np.arange(N)[None, :]
    for b in range(B):
        for h in range(H):
            Q, K, V, dO = q[b, h], k[b, h], v[b, h], do[b, h]
            for g0 in range(0, len(rows), group):
                rr = rows[g0:g0 + group]
                sl = slice(g0, g0 + len(rr))
                a = dO[rr] @ V.T  # (do_t . v_s) for t in rr
                if causal:
                    a = np.where(cols <= rr[:, None], a, 0.0)
                dq[b, h, sl] = a @ K
                c = V[rr] @ dO.T  # (do_t . v_s) for s in rr, all t
                e = K[rr] @ Q.T   # (q_t . k_s) for s in rr, all t
                if causal:
                    later = cols >= rr[:, None]
                    c = np.where(later, c, 0.0)
                    e = np.where(later, e, 0.0)
                dk[b, h, sl] = c @ Q
                dvv[b, h, sl] = e @ dO
    return dq, dk, dvv


def recurrent_forward(q, k, v) -> np.ndarray:
    """RNN form of the causal op: ``KV_t = KV_{t-1} + k_t^T v_t``, ``o_t = q_t KV_t``.

    The state is d x dv and starts at zero (article, speed section: lossless
    conversion to an RNN). One token at a time; a pin for ``forward`` only.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    _check(q, k, v)
    B, H, N, d = q.shape
    out = np.empty(q.shape[:3] + (v.shape[3],))
    for b in range(B):
        for h in range(H):
            kv = np.zeros((d, v.shape[3]))
            for t in range(N):
                kv += np.outer(k[b, h, t], v[b, h, t])
                out[b, h, t] = q[b, h, t] @ kv
    return out


def _decay_rates(lam, H: int) -> np.ndarray:
    lam = np.asarray(_f64(lam), dtype=np.float64).reshape(-1)
    if lam.shape != (H,):
        raise ValueError("one decay rate per head expected")
    return lam


def _decay_matrix(lam: float, rows: np.ndarray, N: int) -> np.ndarray:
    """``D[t, s] = lam^(t - s)`` for ``s <= t``, else 0 (rows t given, all s)."""
    gap = rows[:, None] - np.arange(N)[None, :]
    return np.where(gap >= 0, lam ** np.maximum(gap, 0), 0.0)


def forward_decay(q, k, v, lam) -> np.ndarray:
    """Decayed causal left product ``O = ((Q K^T) ⊙ D) V`` for every (b, h).

    Row t of O is ``sum_{s<=t} lam_h^(t-s) (q_t . k_s) v_s`` with one rate
    ``lam_h`` per head (a reading: see the module notes).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    _check(q, k, v)
    B, H, N, _ = q.shape
    lam = _decay_rates(lam, H)
    out = np.empty(q.shape[:3] + (v.shape[3],), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            K, V = k[b, h], v[b, h]
            for r0 in range(0, N, ROW_GROUP):
                r1 = min(N, r0 + ROW_GROUP)
                S = (q[b, h, r0:r1] @ K.T) * _decay_matrix(lam[h], np.arange(r0, r1), N)
                out[b, h, r0:r1] = S @ V
    return out


def backward_decay(q, k, v, do, lam):
    """Closed-form gradients of ``L = <dO, O>`` for ``O = ((Q K^T) ⊙ D) V``.

    With ``P = (Q K^T) ⊙ D`` and ``dP = (dO V^T) ⊙ D``:
    ``dQ = dP K``, ``dK = dP^T Q``, ``dV = P^T dO``.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    _check(q, k, v)
    B, H, N, _ = q.shape
    lam = _decay_rates(lam, H)
    dq, dk, dvv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    for b in range(B):
        for h in range(H):
            Q, K, V, dO = q[b, h], k[b, h], v[b, h], do[b, h]
            dk_acc, dv_acc = np.zeros_like(K), np.zeros_like(V)
            for r0 in range(0, N, ROW_GROUP):
                r1 = min(N, r0 + ROW_GROUP)
                D = _decay_matrix(lam[h], np.arange(r0, r1), N)
                P = (Q[r0:r1] @ K.T) * D
                dP = (dO[r0:r1] @ V.T) * D
                dq[b, h, r0:r1] = dP @ K
                dk_acc += dP.T @ Q[r0:r1]
                dv_acc += P.T @ dO[r0:r1]
            dk[b, h] = dk_acc
            dvv[b, h] = dv_acc
    return dq, dk, dvv


def recurrent_forward_decay(q, k, v, lam) -> np.ndarray:
    """RNN form of the decayed op: ``KV_t = lam KV_{t-1} + k_t^T v_t``, ``o_t = q_t KV_t``.

    A pin for ``forward_decay`` only (one token at a time, zero initial state).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    _check(q, k, v)
    B, H, N, d = q.shape
    lam = _decay_rates(lam, H)
    out = np.empty(q.shape[:3] + (v.shape[3],))
    for b in range(B):
        for h in range(H):
            kv = np.zeros((d, v.shape[3]))
            for t in range(N):
                kv = lam[h] * kv + np.outer(k[b, h, t], v[b, h, t])
                out[b, h, t] = q[b, h, t] @ kv
    return out


def _group(H: int, Hkv: int) -> int:
    if Hkv < 1 or H % Hkv:
        raise ValueError("H must be a multiple of the number of K/V heads")
    return H // Hkv


def forward_gqa(q, k, v, causal: bool = True) -> np.ndarray:
    """Grouped K/V heads (GQA; MQA when there is one K/V head): ``q [B,H,N,d]``,
    ``k [B,Hkv,N,d]``, ``v [B,Hkv,N,dv]``; query head h attends through K/V head
    ``h // (H // Hkv)`` with the left product of point 1, one (b, h) at a time.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    if q.ndim != 4 or k.shape[:3] != (q.shape[0], k.shape[1], q.shape[2]) or v.shape[:3] != k.shape[:3]:
        raise ValueError("q [B,H,N,d], k [B,Hkv,N,d], v [B,Hkv,N,dv] expected")
    B, H, N, _ = q.shape
    g = _group(H, k.shape[1])
    out = np.empty((B, H, N, v.shape[3]))
    keep = np.tri(N, dtype=bool) if causal else np.ones((N, N), dtype=bool)
    for b in range(B):
        for h in range(H):
            S = q[b, h] @ k[b, h // g].T
            out[b, h] = np.where(keep, S, 0.0) @ v[b, h // g]
    return out


def backward_gqa(q, k, v, do, causal: bool = True):
    """Gradients of ``L = <dO, O>`` for ``forward_gqa``: per query head the closed
    forms of ``backward``; a K/V head's dK and dV add up over the query heads of
    its group (each of them reads that K/V head).
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, N, _ = q.shape
    g = _group(H, k.shape[1])
    keep = np.tri(N, dtype=bool) if causal else np.ones((N, N), dtype=bool)
    dq = np.empty_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(H):
            kv = h // g
            dP = np.where(keep, do[b, h] @ v[b, kv].T, 0.0)
            P = np.where(keep, q[b, h] @ k[b, kv].T, 0.0)
            dq[b, h] = dP @ k[b, kv]
            dk[b, kv] += dP.T @ q[b, h]
            dv[b, kv] += P.T @ do[b, h]
    return dq, dk, dv


def kv_state(k, v, state=None) -> np.ndarray:
    """The KV state a causal pass leaves behind: ``state + sum_t k_t^T v_t``.

    Shapes ``k [B,H,N,d]``, ``v [B,H,N,dv]``, ``state [B,H,d,dv]`` (zero when
    omitted). This is the state the block algorithm of point 2 carries past a
    sequence's last block, and the state an RNN-mode step (speed section)
    continues from. Defined as a plain sum of outer products.
    """
    k, v = _f64(k), _f64(v)
    if k.ndim != 4 or v.ndim != 4 or k.shape[:3] != v.shape[:3]:
        raise ValueError("k [B,H,N,d] and v [B,H,N,dv] expected")
    out = np.zeros(k.shape[:2] + (k.shape[3], v.shape[3])) if state is None else _f64(state).copy()
    for b in range(k.shape[0]):
        for h in range(k.shape[1]):
            for t in range(k.shape[2]):
                out[b, h] += np.outer(k[b, h, t], v[b, h, t])
    return out


def decode_step(q, k, v, state):
    """One RNN-mode step for one new token per (b, h) (article, speed section).

    ``q, k [B,H,d]``, ``v [B,H,dv]``, ``state [B,H,d,dv]``. Returns
    ``(o, new_state)`` with ``new_state = state + k^T v`` and
    ``o = q new_state``: the token's own pair is included, as the diagonal of
    the causal mask is in the left product.
    """
    q, k, v, s = _f64(q), _f64(k), _f64(v), _f64(state)
    if q.ndim != 3 or k.shape != q.shape or v.shape[:2] != q.shape[:2]:
        raise ValueError("q, k [B,H,d] and v [B,H,dv] expected")
    if s.shape != q.shape[:2] + (q.shape[2], v.shape[2]):
        raise ValueError("state [B,H,d,dv] expected")
    new = s + k[..., :, None] * v[..., None, :]
    o = np.einsum("bhd,bhde->bhe", q, new)
    return o, new


def forward_from_state(q, k, v, state) -> np.ndarray:
    """Causal output of a sequence whose earlier tokens are summarised by a KV
    state ``state [B,H,d,dv]`` (article, point 2: a block's inter-block part is
    its queries times the state accumulated over everything before it):
    ``o_t = q_t state + sum_{s <= t} (q_t . k_s) v_s``. With the state of a
    sequence's first part this is the output of its second part (sequence
    parallelism: each shard starts from the sum of the earlier shards' states).
    """
    st = _f64(state)
    out = forward(q, k, v, True)
    return out + np.einsum("bhnd,bhde->bhne", _f64(q), st)


def backward_from_states(q, k, v, do, prefix, suffix):
    """Gradients, for one part of a longer causal sequence, of the loss
    ``sum_t <dO_t, O_t>`` over the whole sequence: the part's closed forms
    (``backward``) plus the terms that cross its ends. ``prefix [B,H,d,dv]`` is
    the KV state of the tokens before the part (its queries read it:
    ``dq_t += dO_t prefix^T``); ``suffix [B,H,d,dv]`` is ``sum q_t^T dO_t`` over
    the tokens after it (their queries read this part's keys and values:
    ``dk_s += v_s suffix^T``, ``dv_s += k_s suffix``).
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    P, U = _f64(prefix), _f64(suffix)
    dq, dk, dvv = backward(q, k, v, do, True)
    dq = dq + np.einsum("bhne,bhde->bhnd", do, P)
    dk = dk + np.einsum("bhne,bhde->bhnd", v, U)
    dvv = dvv + np.einsum("bhnd,bhde->bhne", k, U)
    return dq, dk, dvv


def blocked_forward(q, k, v, block: int, causal: bool = True) -> np.ndarray:
    """The block algorithm of the article's point 2, in float64.

    Blocks of ``block`` rows. For block i: intra part ``((Q_i K_i^T) ⊙ M_B) V_i``
    (left product), inter part ``Q_i KV`` with ``KV = sum_{j<i} K_j^T V_j`` (right
    product); the two are added to give ``O_i``, then ``KV += K_i^T V_i``.
    Without the mask it is ``Q (K^T V)``. A cross-check of ``forward`` (block-size
    invariance) and the full-tensor reference for very long sequences.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    _check(q, k, v)
    B, H, N, d = q.shape
    dvd = v.shape[3]
    out = np.empty(q.shape[:3] + (dvd,))
    for b in range(B):
        for h in range(H):
            Q, K, V = q[b, h], k[b, h], v[b, h]
            if not causal:
                out[b, h] = Q @ (K.T @ V)
                continue
            kv = np.zeros((d, dvd))
            for i0 in range(0, N, block):
                i1 = min(N, i0 + block)
                S = Q[i0:i1] @ K[i0:i1].T
                S = np.tril(S)  # M_B, diagonal kept
                out[b, h, i0:i1] = S @ V[i0:i1] + Q[i0:i1] @ kv
                kv += K[i0:i1].T @ V[i0:i1]
    return out


def relative_frobenius(x, ref) -> float:
    """``||x - ref||_F / ||ref||_F`` in float64 (0 if both are zero)."""
    x = _f64(x)
    ref = _f64(ref)
    num = float(np.linalg.norm((x - ref).ravel()))
    den = float(np.linalg.norm(ref.ravel()))
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return num / den
