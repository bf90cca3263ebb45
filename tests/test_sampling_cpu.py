"""The stratified token sample of the full-size parity tests reaches every tile case.

Host logic only: given a routing, the sample must hold, for every expert, its
first and last segment row, the rows on both sides of its first and last
128-row m-tile boundary, and rows of its last m-tile when the expert has an
odd number of m-tiles; and it must reach every expert with tokens, rare ones
included."""
import numpy as np

from moe_testlib import experts_reached, stratified_tokens


def _segments(idx, E):
    return [np.nonzero((idx == e).any(axis=1))[0] for e in range(E)]


def _skewed_routing(T, E, k, seed):
    rng = np.random.default_rng(seed)
    p = 1.0 / np.arange(1, E + 1) ** 1.2
    p /= p.sum()
    rows = []
    for _ in range(T):
        rows.append(rng.choice(E, size=k, replace=False, p=p))
    return np.array(rows, dtype=np.int32)


def test_sample_holds_every_tile_case():
    E, k = 8, 2
    idx = _skewed_routing(5000, E, k, seed=1)
    toks = set(stratified_tokens(idx, E, seed=1).tolist())
    for e, rows in enumerate(_segments(idx, E)):
        n = len(rows)
        assert rows[0] in toks and rows[-1] in toks
        if n > 128:
            last_b = ((n - 1) // 128) * 128
            for r in (127, 128, last_b - 1, last_b):
                assert rows[r] in toks, (e, r)
        mt = (n + 127) // 128
        if mt % 2 == 1:
            tail = rows[(mt - 1) * 128:]
            assert len(set(tail.tolist()) & toks) >= min(2, len(tail)), e
    assert experts_reached(idx, sorted(toks)) == set(range(E))


def test_sample_reaches_rare_experts_and_skips_empty_ones():
    E, k, T = 6, 2, 3000
    idx = np.zeros((T, k), dtype=np.int32)
    idx[:, 1] = 1
    idx[1234] = (4, 2)          # experts 2 and 4 hold one token each, 3 and 5 none
    toks = stratified_tokens(idx, E, n_random=0, seed=0)
    assert 1234 in toks
    assert experts_reached(idx, toks) == {0, 1, 2, 4}
    assert toks[0] == 0 and toks[-1] == T - 1
    assert np.all(np.diff(toks) > 0)


def test_sample_of_a_tiny_batch_is_every_token():
    idx = np.array([[0, 1], [1, 0], [2, 1]], dtype=np.int32)
    assert stratified_tokens(idx, 3, n_random=3).tolist() == [0, 1, 2]
