"""Pin the oracle's flat layout, buckets and layers: hand-worked values
(tests/golden/layout_worked.txt) and brute-force properties on random tiny
tensor lists."""
import os

import numpy as np
import pytest

import oracle as O


def worked(path):
    for line in open(path):
        line = line.strip()
        if line and not line.startswith("#"):
            name, R, A, sizes, offs, P, L, S, T = line.split()
            yield (name, int(R), int(A), [int(x) for x in sizes.split(",")],
                   [int(x) for x in offs.split(",")], int(P), int(L), int(S), int(T))


def test_worked_values(golden_dir):
    n = 0
    for name, R, A, sizes, offs, P, L, S, T in worked(os.path.join(golden_dir, "layout_worked.txt")):
        lay = O.Layout(sizes, R, A)
        assert lay.offsets.tolist() == offs, name
        assert (lay.P, lay.L, lay.S, lay.T) == (P, L, S, T), name
        n += 1
    assert n == 4


def brute_offsets(numels, A):
    # smallest position at or after the previous tensor's end that is a multiple of A
    offs, end = [], 0
    for k in numels:
        pos = end
        while pos % A:
            pos += 1
        offs.append(pos)
        end = pos + k
    return offs, end


def random_case(rng):
    n = int(rng.integers(1, 21))
    numels = rng.integers(1, 60, n)
    if rng.random() < 0.3:
        numels[rng.integers(0, n)] = int(rng.integers(100, 400))
    R = int(rng.integers(1, 17))
    A = int(rng.choice([1, 8]))
    B = int(rng.choice([0, 1, 16, 50, 100, 1000]))
    steps = rng.integers(0, 2, n)
    steps[0] = 0
    layer_ids = np.cumsum(steps).astype(np.int32)
    return numels, R, A, B, layer_ids


@pytest.mark.parametrize("seed", range(300))
def test_properties_random_lists(seed):
    rng = np.random.default_rng(seed)
    numels, R, A, B, layer_ids = random_case(rng)
    lay = O.Layout(numels, R, A, B, layer_ids)
    n = len(numels)

    # offsets: brute-force placement
    offs, end = brute_offsets(numels.tolist(), A)
    assert lay.offsets.tolist() == offs
    assert lay.L == end and lay.P == int(numels.sum())

    # shards: equal, multiple of 8, the fewest that cover L
    assert lay.S % 8 == 0 and lay.T == R * lay.S
    assert lay.T >= lay.L >= lay.P
    assert lay.T - lay.L < 8 * R
    assert R * (lay.S - 8) < lay.L  # one multiple of 8 less would not cover L

    # buckets partition [0, T) exactly, in decreasing offset order
    bk = lay.buckets
    assert bk[0][1] == lay.T and bk[-1][0] == 0
    for (lo, hi), (lo2, hi2) in zip(bk, bk[1:]):
        assert hi2 == lo and lo < hi
    # every tensor lies inside its own bucket's range; tensors of a bucket are contiguous
    for k in range(n):
        lo, hi = bk[lay.tensor_bucket[k]]
        assert lo <= lay.offsets[k] and lay.offsets[k] + numels[k] <= hi
    assert np.all(np.diff(lay.tensor_bucket) <= 0)  # reverse order: later tensors, lower ids
    # size rule and greedy maximality
    for b in range(len(bk)):
        ks = np.flatnonzero(lay.tensor_bucket == b)
        total = int(numels[ks].sum())
        if B <= 0:
            assert len(bk) == 1
            continue
        assert total <= B or len(ks) == 1
        lower = ks.min() - 1
        if lower >= 0:
            assert total + int(numels[lower]) > B  # the next tensor did not fit

    # layers: contiguous cover of [0, L), one per distinct id, holding its tensors
    ly = lay.layers
    assert len(ly) == int(layer_ids[-1]) + 1
    assert ly[0][0] == 0 and ly[-1][1] == lay.L
    for (lo, hi), (lo2, hi2) in zip(ly, ly[1:]):
        assert hi == lo2
    for k in range(n):
        lo, hi = ly[layer_ids[k]]
        assert lo <= lay.offsets[k] and lay.offsets[k] + numels[k] <= hi


def test_no_layer_ids_means_one_layer_per_tensor():
    lay = O.Layout([5, 9, 2], 3, 8)
    assert lay.layers == [(0, 8), (8, 24), (24, 26)]


@pytest.mark.parametrize("bad", [
    dict(numels=[], R=2), dict(numels=[0, 4], R=2), dict(numels=[4], R=0),
    dict(numels=[4, 4], R=2, layer_ids=[1, 1]), dict(numels=[4, 4, 4], R=2, layer_ids=[0, 2, 2]),
    dict(numels=[4, 4], R=2, layer_ids=[0, -1]),
])
def test_rejects_invalid(bad):
    with pytest.raises(ValueError):
        O.Layout(bad["numels"], bad["R"], 8, 0, bad.get("layer_ids"))
