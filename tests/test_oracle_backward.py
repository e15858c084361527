"""Pins of the oracle's backward passes (route score and sparse attention): central finite
differences of the oracle's own forward, on small random inputs away from ties, and the closed
forms they must reduce to.  A wrong sign, a dropped norm term, a transposed rotation or a
missing softmax-centring term each fails one of them."""
import numpy as np
import pytest

import oracle


def _fd(f, x, idx, h):
    x0 = x[idx]
    x[idx] = x0 + h
    fp = f()
    x[idx] = x0 - h
    fm = f()
    x[idx] = x0
    return (fp - fm) / (2 * h)


def _route_problem(seed):
    rng = np.random.default_rng(seed)
    B, T, H_r, d_r = 2, 3, 2, 8
    off = np.array([0, 3, 5, 9], dtype=np.int64)  # 3 documents of 3, 2, 4 chunks
    Qr = rng.standard_normal((B, T, H_r, d_r))
    Kb = rng.standard_normal((int(off[-1]), H_r, d_r)) * rng.uniform(0.5, 2.0, (int(off[-1]), 1, 1))
    G = rng.standard_normal((B, 3))
    return Qr, Kb, off, G


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_route_backward_matches_finite_differences(seed):
    Qr, Kb, off, G = _route_problem(seed)
    dQ, dK = oracle.route_backward(Qr, Kb, off, G)

    def loss():
        return float(np.sum(G * oracle.route(Qr, Kb, off)))

    rng = np.random.default_rng(seed + 10)
    for arr, grad in ((Qr, dQ), (Kb, dK)):
        for _ in range(25):
            idx = tuple(rng.integers(0, n) for n in arr.shape)
            assert abs(_fd(loss, arr, idx, 1e-6) - grad[idx]) <= 1e-7 + 1e-6 * abs(grad[idx])


def test_route_backward_reaches_only_the_maximising_pair():
    Qr, Kb, off, G = _route_problem(3)
    G[:] = 0.0
    G[1, 2] = 1.0                                       # query 1, document 2 (chunks 5..8)
    dQ, dK = oracle.route_backward(Qr, Kb, off, G)
    assert np.count_nonzero(np.abs(dQ).sum(axis=(2, 3))) == 1   # one token of query 1
    assert np.all(dQ[0] == 0)
    rows = np.nonzero(np.abs(dK).sum(axis=(1, 2)))[0]
    assert rows.size == 1 and 5 <= rows[0] < 9
    # the cosine gradient is orthogonal to its own vector (scale invariance)
    t = int(np.nonzero(np.abs(dQ[1]).sum(axis=(1, 2)))[0][0])
    for h in range(Qr.shape[2]):
        assert abs(np.dot(dQ[1, t, h], Qr[1, t, h])) <= 1e-12
        assert abs(np.dot(dK[rows[0], h], Kb[rows[0], h])) <= 1e-12


def _attend_problem(seed, k=2, T=3, q_start=2, H_q=4, H_kv=2, D=8):
    rng = np.random.default_rng(seed)
    B = 2
    off = np.array([0, 2, 3, 6, 8], dtype=np.int64)   # 4 documents of 2, 1, 3, 2 chunks
    C = int(off[-1])
    L = q_start + T
    Q = rng.standard_normal((B, T, H_q, D))
    Kl = rng.standard_normal((B, L, H_kv, D))
    Vl = rng.standard_normal((B, L, H_kv, D))
    Kb = rng.standard_normal((C, H_kv, D))
    Vb = rng.standard_normal((C, H_kv, D))
    ids = np.stack([rng.choice(4, size=k, replace=False) for _ in range(B)]).astype(np.int32)
    dO = rng.standard_normal((B, T, H_q, D))
    return Q, Kl, Vl, Kb, Vb, off, ids, dO, q_start


@pytest.mark.parametrize("seed,k", [(0, 2), (1, 0), (2, 4)])
def test_attend_backward_matches_finite_differences(seed, k):
    Q, Kl, Vl, Kb, Vb, off, ids, dO, q0 = _attend_problem(seed, k=k)
    theta, pos = 1e4, k
    grads = oracle.attend_backward(Q, Kl, Vl, q0, Kb, Vb, off, ids, pos, theta, dO)

    def loss():
        O, _, _ = oracle.attend(Q, Kl, Vl, q0, Kb, Vb, off, ids, pos, theta)
        return float(np.sum(dO * O))

    rng = np.random.default_rng(seed + 20)
    for arr, grad in zip((Q, Kl, Vl, Kb, Vb), grads):
        for _ in range(20):
            idx = tuple(rng.integers(0, n) for n in arr.shape)
            assert abs(_fd(loss, arr, idx, 1e-5) - grad[idx]) <= 1e-8 + 1e-6 * abs(grad[idx])


def test_attend_backward_closed_forms():
    Q, Kl, Vl, Kb, Vb, off, ids, dO, q0 = _attend_problem(4, k=1)
    theta, pos = 1e4, 1
    dQ, dK, dV, dKb, dVb = oracle.attend_backward(Q, Kl, Vl, q0, Kb, Vb, off, ids, pos, theta, dO)
    # values: dV summed over every row = sum over (query, token, head) of dO (softmax rows sum to 1)
    group = Q.shape[2] // Kl.shape[2]
    for g in range(Kl.shape[2]):
        tot = dV[:, :, g].sum(axis=(0, 1)) + dVb[:, g].sum(axis=0)
        want = dO[:, :, g * group:(g + 1) * group].sum(axis=(0, 1, 2))
        assert np.allclose(tot, want, atol=1e-12)
    # keys: the softmax is invariant to a common shift of a row's logits (sum_y dz_y = 0), so
    # for one (query, token, head) the gradients of the keys as the logits see them -- dKbar
    # and the local keys' gradients rotated back to their RoPE positions -- sum to zero
    B, T, H_q, D = Q.shape
    one = np.zeros_like(dO)
    one[0, 0, 0] = dO[0, 0, 0]
    _, dK1, _, dKb1, _ = oracle.attend_backward(Q, Kl, Vl, q0, Kb, Vb, off, ids, pos, theta, one)
    rot = np.stack([oracle.rope_rows(dK1[0, :, None, 0], pos + np.arange(Kl.shape[1]),
                                     theta)[:, 0]])[0]
    total = rot.sum(axis=0) + dKb1[:, 0].sum(axis=0)
    assert np.allclose(total, 0.0, atol=1e-12)
    # rows the token cannot see get nothing
    assert np.all(dK1[0, q0 + 1:] == 0) and np.all(dK1[1] == 0)
