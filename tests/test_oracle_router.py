"""Pins for the oracle's router and routing metadata (CPU only).

Each check ties the oracle to something other than itself: brute-force
enumeration, a library routine, or an invariant that the pages' "dropless
top-k routing" fixes (each token goes to exactly k experts, nothing is
dropped, the restore step inverts the regrouping)."""
import itertools

import numpy as np
import pytest
import scipy.special
import torch

from oracle import moe_ref as R


def _brute_topk(row, k):
    """Best k-subset by sum of logits, ties to the lexicographically
    smallest index set; slots ordered by (-logit, index)."""
    E = len(row)
    best, best_key = None, None
    for S in itertools.combinations(range(E), k):
        key = (sum(row[i] for i in S), tuple(-i for i in S))
        if best_key is None or key > best_key:
            best, best_key = S, key
    return sorted(best, key=lambda i: (-row[i], i))


@pytest.mark.parametrize("E,k", [(1, 1), (3, 1), (4, 2), (5, 3), (6, 3), (6, 1)])
def test_topk_matches_brute_force(E, k):
    rng = np.random.default_rng(E * 10 + k)
    # integer logits make ties common, which exercises the tie rule
    L = rng.integers(-2, 3, size=(8, E)).astype(np.float64)
    got = R.topk_select(L, k)
    for t in range(L.shape[0]):
        assert list(got[t]) == _brute_topk(list(L[t]), k)


def test_topk_continuous_values_brute_force():
    rng = np.random.default_rng(1)
    L = rng.standard_normal((8, 6))
    got = R.topk_select(L, 3)
    for t in range(8):
        assert list(got[t]) == _brute_topk(list(L[t]), 3)


def test_softmax_matches_scipy():
    rng = np.random.default_rng(2)
    L = rng.standard_normal((16, 7)) * 5
    np.testing.assert_allclose(R.softmax(L), scipy.special.softmax(L, axis=1),
                               rtol=1e-14, atol=1e-16)


def test_single_expert_gate_is_one():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((5, 8))
    w_r = rng.standard_normal((1, 8))
    r = R.router_topk(x, w_r, 1)
    assert np.all(r["idx"] == 0)
    np.testing.assert_allclose(r["w"], 1.0)


def test_renorm_weights_sum_to_one():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((9, 8))
    w_r = rng.standard_normal((6, 8))
    r = R.router_topk(x, w_r, 3, renorm=True)
    np.testing.assert_allclose(r["w"].sum(axis=1), 1.0, rtol=1e-14)
    r0 = R.router_topk(x, w_r, 3)
    assert np.all(r0["w"].sum(axis=1) < 1.0)


def test_forced_route_uses_router_probabilities():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((4, 8))
    w_r = rng.standard_normal((5, 8))
    route = np.array([[4, 0], [1, 2], [3, 4], [0, 1]])
    r = R.router_topk(x, w_r, 2, route=route)
    p = scipy.special.softmax(x @ w_r.T, axis=1)
    for t in range(4):
        for j in range(2):
            assert r["w"][t, j] == pytest.approx(p[t, route[t, j]], rel=1e-14)


def test_bias_shifts_logits():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((4, 8))
    w_r = rng.standard_normal((5, 8))
    b = np.array([0.0, -1.0, 2.0, 0.5, -3.0])
    L = R.router_logits(x, w_r, b)
    np.testing.assert_allclose(L - R.router_logits(x, w_r), np.tile(b, (4, 1)), atol=1e-14)


def _brute_metadata(idx, E, align=32):
    T, k = len(idx), len(idx[0])
    counts = [0] * E
    for t in range(T):
        for j in range(k):
            counts[idx[t][j]] += 1
    offsets = [0]
    for e in range(E):
        offsets.append(offsets[-1] + (counts[e] + align - 1) // align * align)
    row_map = [[0] * k for _ in range(T)]
    for t in range(T):
        for j in range(k):
            e = idx[t][j]
            earlier = sum(1 for t2 in range(T) for j2 in range(k)
                          if (t2 * k + j2) < (t * k + j) and idx[t2][j2] == e)
            row_map[t][j] = offsets[e] + earlier
    return counts, offsets, row_map


@pytest.mark.parametrize("T,E,k,seed", [(7, 3, 2, 0), (12, 5, 3, 1), (40, 4, 1, 2),
                                        (33, 6, 4, 3), (5, 8, 2, 4)])
def test_metadata_brute_force(T, E, k, seed):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)])
    m = R.routing_metadata(idx, E)
    c, o, rm = _brute_metadata(idx.tolist(), E)
    assert m["counts"].tolist() == c
    assert m["offsets"].tolist() == o
    assert m["row_map"].tolist() == rm


@pytest.mark.parametrize("T,E,k,seed", [(512, 8, 4, 0), (300, 128, 4, 1), (64, 3, 3, 2),
                                        (1, 4, 2, 3)])
def test_metadata_invariants(T, E, k, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, 16))
    w_r = rng.standard_normal((E, 16))
    r = R.router_topk(x, w_r, k)
    idx = r["idx"]
    # exactly k distinct experts per token
    assert all(len(set(row)) == k for row in idx.tolist())
    m = R.routing_metadata(idx, E)
    counts, off, rm = m["counts"], m["offsets"], m["row_map"]
    assert counts.sum() == T * k                       # dropless
    pad = (counts + 31) // 32 * 32
    assert off[0] == 0 and np.all(np.diff(off) == pad)
    assert np.all(off % 32 == 0)
    flat = rm.reshape(-1)
    assert len(set(flat.tolist())) == T * k            # injective
    for e in range(E):                                 # onto the non-pad rows
        rows = sorted(flat[idx.reshape(-1) == e].tolist())
        assert rows == list(range(off[e], off[e] + counts[e]))
    # ascending token order inside a segment
    for e in range(E):
        sel = np.nonzero(idx.reshape(-1) == e)[0]
        assert np.all(np.diff(flat[sel]) == 1)
    # permute then restore
    xp = R.permute(x, rm, m["M_pad"], rnd=None)
    for j in range(k):
        np.testing.assert_array_equal(xp[rm[:, j]], x)
    mask = np.ones(m["M_pad"], bool)
    mask[flat] = False
    assert np.all(xp[mask] == 0)


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(7)
    v = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
                        [0.0, -0.0, 1.0, 3.0e38, -3.0e38, 1e-40]])
    ours = R.bf16_round(v)
    ref = torch.tensor(v.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(ours, ref)


def test_bf16_round_exact_ties_go_to_even():
    """fp32 words whose dropped half is exactly 0x8000 lie halfway between
    two bf16 values (random values almost never do). They must round to the
    neighbour with an even upper half, as torch's cast does. Words one below
    and one above the tie round down and up."""
    rng = np.random.default_rng(8)
    hi = rng.integers(0, 0x7F80, 4000).astype(np.uint32)    # finite upper halves
    hi = np.concatenate([hi, hi | 0x8000, [0, 1, 2, 3, 0x7F7E, 0x7F7F]]).astype(np.uint32)
    for low in (0x8000, 0x7FFF, 0x8001):
        v = ((hi << 16) | low).view(np.float32).astype(np.float64)
        ours = R.bf16_round(v)
        ref = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
        np.testing.assert_array_equal(ours, ref)
        up = ours.astype(np.float32).view(np.uint32) >> 16
        mag = (hi & 0x7FFF).astype(np.int64)
        got = (up & 0x7FFF).astype(np.int64)
        if low == 0x8000:
            want = np.where(mag % 2 == 0, mag, mag + 1)        # ties to the even neighbour
        else:
            want = mag + (1 if low == 0x8001 else 0)
        np.testing.assert_array_equal(got, want)
