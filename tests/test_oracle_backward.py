"""Pins of the float64 backward oracle (CPU): the routing gradient against
central finite differences of the forward oracle, the pooling backward as
the adjoint of the forward pooling, and special cases."""

import numpy as np
import pytest

import oracle
from oracle import msa_backward as bwd


def _routing_case(seed, B=2, T=3, H=2, D=8, lengths=(64, 180, 100, 250, 64, 130)):
    rng = np.random.default_rng(seed)
    coff = oracle.chunk_offsets_from_lengths(np.array(lengths))
    C = int(coff[-1])
    q = rng.standard_normal((B, T, H, D))
    k = rng.standard_normal((C, H, D))
    g = rng.standard_normal((B, len(lengths)))
    return q, k, coff, g


def _loss(q, k, coff, g):
    ds, _ = oracle.route_scores(q, k, coff)
    return float((g * ds).sum())


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_route_backward_matches_finite_differences(seed):
    """dL/dQ_r and dL/dK_r of L = sum g * doc_score, against central
    differences of the forward oracle (random inputs: no ties)."""
    q, k, coff, g = _routing_case(seed)
    dq, dk = bwd.route_scores_backward(q, k, coff, g)
    h = 1e-6
    for x, dx in ((q, dq), (k, dk)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            old = x[i]
            x[i] = old + h
            lp = _loss(q, k, coff, g)
            x[i] = old - h
            lm = _loss(q, k, coff, g)
            x[i] = old
            num[i] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(dx, num, atol=2e-7, rtol=1e-5)


def test_route_argmax_is_the_forward_score():
    q, k, coff, _ = _routing_case(5)
    s, c, t = bwd.route_argmax(q, k, coff)
    ds, cs = oracle.route_scores(q, k, coff)
    np.testing.assert_allclose(s, ds, rtol=0, atol=1e-12)
    # the chosen chunk is in its document and carries the document's score
    for b in range(q.shape[0]):
        for d in range(len(coff) - 1):
            assert coff[d] <= c[b, d] < coff[d + 1]
            assert abs(cs[b, c[b, d]] - ds[b, d]) < 1e-12


def test_route_backward_ties_go_to_the_first_maximiser():
    """Two identical chunks and two identical query tokens: the whole
    gradient goes to the lower chunk and the lower token."""
    rng = np.random.default_rng(9)
    q = rng.standard_normal((1, 2, 1, 4))
    q[0, 1] = q[0, 0]
    k = np.repeat(q[0, 0][None], 2, axis=0) + 0.0  # chunks 0 and 1 equal, parallel to q
    coff = np.array([0, 2])
    _, c, t = bwd.route_argmax(q, k, coff)
    assert (c[0, 0], t[0, 0]) == (0, 0)
    dq, dk = bwd.route_scores_backward(q, k, coff, np.array([[1.0]]))
    assert np.all(dk[1] == 0) and np.all(dq[0, 1] == 0)


def test_route_backward_linear_in_g_and_zero_without_gradient():
    q, k, coff, g = _routing_case(3)
    dq1, dk1 = bwd.route_scores_backward(q, k, coff, g)
    dq2, dk2 = bwd.route_scores_backward(q, k, coff, 3.0 * g)
    np.testing.assert_allclose(dq2, 3.0 * dq1, rtol=1e-12)
    np.testing.assert_allclose(dk2, 3.0 * dk1, rtol=1e-12)
    dq0, dk0 = bwd.route_scores_backward(q, k, coff, 0.0 * g)
    assert not dq0.any() and not dk0.any()


def test_cosine_grad_closed_forms():
    """Orthogonality to the vector (scale invariance of the cosine); the
    gradient at q = k is 0 in q; a zero vector (norm below eps) gives
    k / (eps |k|) with no norm term."""
    rng = np.random.default_rng(4)
    q, k = rng.standard_normal(16), rng.standard_normal(16)
    dq, dk = oracle.cosine_grad(q, k)
    assert abs(dq @ q) < 1e-12 and abs(dk @ k) < 1e-12
    dq_same, _ = oracle.cosine_grad(k, k)
    assert np.max(np.abs(dq_same)) < 1e-12
    dq0, dk0 = oracle.cosine_grad(np.zeros(16), k)
    np.testing.assert_allclose(dq0, k / (oracle.EPS * np.linalg.norm(k)), rtol=1e-12)
    assert not dk0.any()


@pytest.mark.parametrize("L,lengths,D", [(1, [180, 64, 1, 130], 8), (2, [100, 300], 16)])
def test_pool_backward_is_the_adjoint_of_pooling(L, lengths, D):
    """<pool(x), y> = <x, pool_backward(y)> for random x (K, V, K_r token
    tensors) and y (pooled gradients): pooling with rotation is linear."""
    rng = np.random.default_rng(L * 100 + D)
    toff = np.concatenate([[0], np.cumsum(lengths)])
    N, H = int(toff[-1]), 2
    x = [rng.standard_normal((L, N, H, D)) for _ in range(3)]
    kb, vb, rb, coff = oracle.encode_pool(x[0], x[1], x[2], toff)
    y = [rng.standard_normal(t.shape) for t in (kb, vb, rb)]
    dx = bwd.encode_pool_backward(y[0], y[1], y[2], toff)
    lhs = sum(float((a * b).sum()) for a, b in zip((kb, vb, rb), y))
    rhs = sum(float((a * b).sum()) for a, b in zip(x, dx))
    assert abs(lhs - rhs) <= 1e-10 * max(1.0, abs(lhs))


def test_pool_backward_planted_rotation_sign_fails_the_adjoint():
    """A plausible mistake -- rotating the gradient forward by +p instead of
    back -- breaks the adjoint identity the test above pins."""
    rng = np.random.default_rng(2)
    toff = np.array([0, 150])
    x = rng.standard_normal((1, 150, 1, 8))
    kb, _, _, coff = oracle.encode_pool(x, x, x, toff)
    y = rng.standard_normal(kb.shape)
    dk, _, _ = bwd.encode_pool_backward(y, 0 * y, 0 * y, toff)
    # the wrong version
    wrong = np.zeros_like(dk)
    for j, (a, b) in enumerate(oracle.msa_oracle.chunk_token_ranges(150)):
        rows = np.repeat(y[0, j][None] / (b - a), b - a, axis=0)
        wrong[0, a:b] = oracle.rope_rotate(rows, np.arange(a, b), 10000.0)
    lhs = float((kb * y).sum())
    assert abs(lhs - float((x * dk).sum())) < 1e-10 * max(1, abs(lhs))
    assert abs(lhs - float((x * wrong).sum())) > 1e-3
