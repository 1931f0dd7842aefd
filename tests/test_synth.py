"""The seeded input generators (synth/): the same seed gives byte-identical arrays, and each array
has the shape and statistics of the workload it stands in for.  No GPU."""
import math

import numpy as np
import pytest

import synth


@pytest.mark.parametrize("make", [
    lambda s: synth.zipf_tokens(10_000, 32768, seed=s),
    lambda s: synth.uniform_tokens(10_000, 27, seed=s),
    lambda s: synth.byte_table(50304, 1, 12, seed=s, n_zero=3),
    lambda s: synth.normal((64, 33), s, std=0.02),
    lambda s: np.concatenate([a.reshape(-1) for a in synth.next_token_batch(4, 17, 1000, seed=s)]),
])
def test_same_seed_same_bytes_other_seed_other_bytes(make):
    a, b, c = make(5), make(5), make(6)
    assert a.dtype == b.dtype and a.tobytes() == b.tobytes()
    assert a.tobytes() != c.tobytes()


@pytest.mark.parametrize("dist", ["zipf", "uniform"])
def test_targets_are_inputs_shifted_by_one(dist):
    # "nanoGPT" wiki page, train.py: y = data[i+1 : i+1+block_size], the inputs shifted by 1
    idx, tgt = synth.next_token_batch(3, 50, 300, dist=dist, seed=9)
    assert idx.shape == tgt.shape == (3, 50) and idx.dtype == tgt.dtype == np.int32
    assert idx.flags["C_CONTIGUOUS"] and tgt.flags["C_CONTIGUOUS"]
    assert np.array_equal(idx[:, 1:], tgt[:, :-1])
    assert idx.min() >= 0 and max(idx.max(), tgt.max()) < 300


def test_zipf_frequencies_follow_the_power_law():
    V, s, n = 32768, 1.1, 2_000_000
    ids = synth.zipf_tokens(n, V, s=s, seed=1)
    assert ids.min() >= 0 and ids.max() < V
    counts = np.bincount(ids, minlength=V).astype(np.float64)
    h = np.sum(np.arange(1, V + 1, dtype=np.float64) ** -s)
    # p(rank k) = k^-s / H: the head of the distribution to within sampling error (5 sigma)
    for k in (1, 2, 3, 10, 100):
        p = k ** -s / h
        assert abs(counts[k - 1] / n - p) <= 5 * math.sqrt(p * (1 - p) / n), k
    # frequencies fall with rank: rank 1 vs rank 2 in the ratio 2^s
    assert counts[0] / counts[1] == pytest.approx(2 ** s, rel=0.02)


def test_byte_table_range_and_zero_entries():
    t = synth.byte_table(32768, 1, 16, seed=2, n_zero=3)
    assert t.dtype == np.int32 and t.shape == (32768,)
    assert int((t == 0).sum()) == 3
    nz = t[t != 0]
    assert nz.min() == 1 and nz.max() == 16
    assert set(np.unique(nz)) == set(range(1, 17))
    assert synth.byte_table(27, 1, 1, seed=0).tolist() == [1] * 27


def test_normal_moments():
    x = synth.normal(1_000_000, 0, std=0.02).astype(np.float64)
    assert abs(x.mean()) < 5 * 0.02 / 1000 and x.std() == pytest.approx(0.02, rel=0.01)
