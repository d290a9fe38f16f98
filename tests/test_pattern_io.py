"""Saving and loading a frozen pattern (LoSA page, Methodology Summary: the pattern built at step t0 is reused
unchanged): a round trip keeps every array, and a file that does not describe the caller's layer, or whose arrays are
not a valid pattern, is refused."""
import numpy as np
import pytest

from free_block_sparse_losa_b200.pattern import check_pattern, load_pattern, save_pattern

SHAPE = {"heads": 2, "n_tokens": 500, "n_padded": 512, "head_dim": 64, "block_q": 128, "block_k": 128}


def _pattern(seed=0):
    rng = np.random.default_rng(seed)
    rows, nk = 2 * 4, 4
    counts = rng.integers(1, nk + 1, rows)
    indptr = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    idx = np.concatenate([np.sort(rng.choice(nk, c, replace=False)) for c in counts]).astype(np.int32)
    order = np.argsort(-counts, kind="stable").astype(np.int32)
    return indptr, idx, order


def test_round_trip(tmp_path):
    indptr, idx, order = _pattern()
    path = str(tmp_path / "p.npz")
    save_pattern(path, SHAPE, 0.99, indptr, np.concatenate([idx, np.full(5, -7, np.int32)]), order)
    tau, i2, x2, o2 = load_pattern(path, SHAPE)
    assert tau == 0.99
    assert np.array_equal(i2, indptr) and np.array_equal(x2, idx) and np.array_equal(o2, order)


def test_refuses_another_layer(tmp_path):
    path = str(tmp_path / "p.npz")
    save_pattern(path, SHAPE, 0.99, *_pattern())
    with pytest.raises(ValueError, match="built for"):
        load_pattern(path, dict(SHAPE, heads=3))


@pytest.mark.parametrize("mistake", ["indptr_start", "empty_list", "index_range", "unsorted", "duplicate", "order"])
def test_refuses_invalid_patterns(mistake):
    indptr, idx, order = _pattern(1)
    indptr, idx, order = indptr.copy(), idx.copy(), order.copy()
    long_row = int(np.argmax(np.diff(indptr)))
    a, b = int(indptr[long_row]), int(indptr[long_row + 1])
    if mistake == "indptr_start":
        indptr = indptr + 1
    elif mistake == "empty_list":
        indptr[1] = indptr[0]
    elif mistake == "index_range":
        idx[0] = 4
    elif mistake == "unsorted":
        assert b - a >= 2
        idx[a], idx[a + 1] = idx[a + 1], idx[a]
    elif mistake == "duplicate":
        assert b - a >= 2
        idx[a + 1] = idx[a]
    else:
        order[0] = order[1]
    with pytest.raises(ValueError):
        check_pattern(SHAPE, indptr, idx, order)
