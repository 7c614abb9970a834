"""Pins for the oracle's load-balancing loss and router variants (CPU only).

The pages ask for a load-balancing auxiliary loss and for balancing over the
global batch but print no formula (discosf.com article on Olmo-core 3,
sections 2.2 and 4.3; Olmo-core 3 introduction page, section 4).  The
reading is the Switch-Transformer loss over the k routed slots; these tests
fix it by properties that do not reuse the oracle's own arithmetic:
its two textbook end points, central finite differences of the loss, the
additivity of the statistics over a split batch, and the identity between
renormalised gate weights and a softmax over the k chosen logits.
"""
import numpy as np
import pytest

from oracle import moe_ref as R


def _route(L, k):
    idx = R.topk_select(L, k)
    E = L.shape[1]
    counts = np.bincount(idx.reshape(-1), minlength=E)
    return idx, counts


def test_balanced_routing_gives_alpha():
    # equal logits: p = 1/E everywhere; every expert gets T k / E slots
    T, E, k, alpha = 64, 8, 2, 0.01
    p = np.full((T, E), 1.0 / E)
    counts = np.full(E, T * k // E)
    loss, dprob = R.router_aux_loss(R.router_load_stats(p, counts), T, k, alpha)
    assert loss == pytest.approx(alpha, rel=1e-14)
    np.testing.assert_allclose(dprob, alpha * E * (1.0 / E) / T, rtol=1e-14)


def test_collapsed_routing_gives_alpha_times_e():
    # k = 1 and every token on expert 0 with probability one: f_0 = P_0 = 1
    T, E, k, alpha = 32, 16, 1, 0.5
    p = np.zeros((T, E))
    p[:, 0] = 1.0
    counts = np.zeros(E)
    counts[0] = T
    loss, _ = R.router_aux_loss(R.router_load_stats(p, counts), T, k, alpha)
    assert loss == pytest.approx(alpha * E, rel=1e-14)


def _aux_of_logits(L, counts, k, alpha):
    return R.router_aux_loss(R.router_load_stats(R.softmax(L), counts), L.shape[0], k, alpha)[0]


@pytest.mark.parametrize("renorm", [False, True])
def test_gradient_matches_finite_differences(renorm):
    """loss(L) = sum_tj dw[t,j] w[t,j](L) + aux(L) with the top-k choice and
    the counts held fixed; router_bwd's dL must equal the numerical
    gradient of that loss."""
    rng = np.random.default_rng(5)
    T, E, k, alpha, d = 12, 6, 2, 0.3, 4
    L = rng.normal(size=(T, E))
    idx, counts = _route(L, k)
    dw = rng.normal(size=(T, k))

    def total(Lv):
        p = R.softmax(Lv)
        w = R.gate_weights(p, idx, renorm)
        return float(np.sum(dw * w)) + _aux_of_logits(Lv, counts, k, alpha)

    p = R.softmax(L)
    _, dprob = R.router_aux_loss(R.router_load_stats(p, counts), T, k, alpha)
    x = rng.normal(size=(T, d))
    w_r = rng.normal(size=(E, d))
    dL = R.router_bwd(dw, p, idx, x, w_r, renorm, rnd=None, dprob_aux=dprob)["dL"]
    h = 1e-6
    num = np.zeros_like(L)
    for t in range(T):
        for e in range(E):
            Lp, Lm = L.copy(), L.copy()
            Lp[t, e] += h
            Lm[t, e] -= h
            num[t, e] = (total(Lp) - total(Lm)) / (2 * h)
    np.testing.assert_allclose(dL, num, rtol=1e-6, atol=1e-9)


def test_aux_gradient_alone_matches_finite_differences():
    rng = np.random.default_rng(9)
    T, E, k, alpha = 10, 5, 3, 0.07
    L = rng.normal(size=(T, E)) * 2
    idx, counts = _route(L, k)
    p = R.softmax(L)
    _, dprob = R.router_aux_loss(R.router_load_stats(p, counts), T, k, alpha)
    dL = R.router_bwd(np.zeros((T, k)), p, idx, np.zeros((T, 1)), np.zeros((E, 1)), rnd=None,
                      dprob_aux=dprob)["dL"]
    h = 1e-6
    for t, e in [(0, 0), (3, 4), (9, 2), (5, 1)]:
        Lp, Lm = L.copy(), L.copy()
        Lp[t, e] += h
        Lm[t, e] -= h
        num = (_aux_of_logits(Lp, counts, k, alpha) - _aux_of_logits(Lm, counts, k, alpha)) / (2 * h)
        assert dL[t, e] == pytest.approx(num, rel=1e-6, abs=1e-12)


def test_statistics_add_over_a_split_batch():
    """Global-batch balancing: the statistics of two halves, added, are the
    statistics of the whole batch, so the loss of the summed statistics is
    the loss of the whole batch."""
    rng = np.random.default_rng(2)
    T, E, k, alpha = 40, 8, 2, 0.01
    L = rng.normal(size=(T, E))
    idx, counts = _route(L, k)
    p = R.softmax(L)
    whole = R.router_load_stats(p, counts)
    a = R.router_load_stats(p[:17], np.bincount(idx[:17].reshape(-1), minlength=E))
    b = R.router_load_stats(p[17:], np.bincount(idx[17:].reshape(-1), minlength=E))
    np.testing.assert_allclose(a + b, whole, rtol=1e-14)
    assert R.router_aux_loss(a + b, T, k, alpha)[0] == pytest.approx(
        R.router_aux_loss(whole, T, k, alpha)[0], rel=1e-14)


def test_renormalised_weights_equal_top_k_then_softmax():
    """A softmax over the k chosen logits gives the renormalised probabilities
    (exp(l_j) / sum_chosen exp(l)), so the two router variants coincide."""
    rng = np.random.default_rng(4)
    T, E, k = 50, 16, 4
    L = rng.normal(size=(T, E)) * 3
    idx = R.topk_select(L, k)
    chosen = np.take_along_axis(L, idx, axis=1)
    direct = np.exp(chosen - chosen.max(axis=1, keepdims=True))
    direct /= direct.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(R.gate_weights(R.softmax(L), idx, renorm=True), direct, rtol=1e-12)
