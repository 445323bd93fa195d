"""Host planning of sequence parallelism over a packed batch
(seqpar.plan_varlen_rank): for random batches and random cuts of the token
axis, the ranks' pieces tile every sequence exactly once and in order, every
sequence's final state is formed on exactly one rank, a sequence is carried
into a rank exactly when it began on an earlier one, and the rank it began
on is the one that holds its first token."""
import numpy as np
import pytest

from linear_attention_blocked_b200 import seqpar


def _check(lens, bounds):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    world = len(bounds) - 1
    pieces = {i: [] for i in range(len(lens))}
    ends = np.zeros(len(lens), int)
    for r in range(world):
        p = seqpar.plan_varlen_rank(cu, bounds, r)
        assert p.tok0 == bounds[r] and p.tok1 == bounds[r + 1]
        assert len(p.local_cu) == p.n_local + 1 and p.local_cu[0] == 0
        assert p.local_cu[-1] == (p.tok1 - p.tok0 if p.n_local else 0)
        lens_local = np.diff(p.local_cu)
        assert p.max_seqlen == (lens_local.max() if p.n_local else 0)
        for i in range(p.n_local):
            g = p.seq0 + i
            a, b = p.tok0 + p.local_cu[i], p.tok0 + p.local_cu[i + 1]
            pieces[g].append((a, b))
            ends[g] += int(p.ends_here[i])
        if p.n_local:
            first = p.seq0
            assert (p.carried_from < r) == (cu[first] < p.tok0)
            if p.carried_from < r:
                assert bounds[p.carried_from] <= cu[first] < bounds[p.carried_from + 1]
            assert (p.open_tail is not None) == (cu[p.seq1] > p.tok1)
    for g, ps in pieces.items():
        if lens[g] == 0:
            assert len(ps) == 1 and ps[0][0] == ps[0][1] == cu[g]
        else:
            assert ps[0][0] == cu[g] and ps[-1][1] == cu[g + 1]
            for (a, b), (c, d) in zip(ps, ps[1:]):
                assert b == c and a < b and c < d
    assert np.all(ends == 1)


def test_plans_tile_every_sequence_once():
    rng = np.random.default_rng(5)
    for _ in range(400):
        n = int(rng.integers(1, 12))
        lens = rng.integers(0, 60, n) * (rng.random(n) < 0.8)
        T = int(lens.sum())
        world = int(rng.integers(1, 7))
        if rng.random() < 0.5:
            bounds = seqpar.split_tokens(T, world)
        else:
            bounds = np.sort(np.concatenate([[0, T], rng.integers(0, T + 1, world - 1)]))
        _check(lens, bounds)


def test_plan_rejects_bad_bounds():
    cu = np.array([0, 5, 9])
    with pytest.raises(ValueError):
        seqpar.plan_varlen_rank(cu, [0, 4], 0)          # does not reach the end
    with pytest.raises(ValueError):
        seqpar.plan_varlen_rank(cu, [0, 6, 5, 9], 0)    # decreasing
    with pytest.raises(ValueError):
        seqpar.plan_varlen_rank(cu, [0, 9], 1)          # no such rank


def test_split_tokens():
    assert seqpar.split_tokens(10, 3).tolist() == [0, 3, 6, 10]
    assert seqpar.split_tokens(0, 2).tolist() == [0, 0, 0]
