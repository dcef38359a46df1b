"""The GPU-vs-oracle comparison rules themselves (CPU): exact ids pass, a different set passes only
inside the near-tie band, and a reordering passes only between near-equal scores."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from parity import check_ids_row


def setup_row(scores):
    """One decode row whose block scores are `scores` (block size 1, one group, d_i 1)."""
    L = len(scores)
    p = oracle.Params(1, 1, 1, 1, 64, 1, 1, 2, 1, 0, L, "f32", 0.125)
    x = {"q_idx": np.ones((1, 1, 1, 1), np.float32), "k_idx": np.array(scores, np.float32).reshape(1, 1, L, 1)}
    s = oracle.token_scores(p, x["q_idx"], x["k_idx"], 0, 0, 0, L - 1)
    ids, sc, kth, kn = oracle.topk(p, oracle.block_scores(p, s, L - 1))
    return p, x, ids, sc, kth, kn


def test_exact_ids_pass():
    p, x, ids, sc, kth, kn = setup_row([1.0, 5.0, 3.0, 0.5])
    assert check_ids_row(p, x, 0, 0, 0, 3, ids, ids, kth, kn, ref_scores=sc)


def test_wrong_set_without_tie_fails():
    p, x, ids, sc, kth, kn = setup_row([1.0, 5.0, 3.0, 0.5])
    with pytest.raises(AssertionError):
        check_ids_row(p, x, 0, 0, 0, 3, [1, 0], ids, kth, kn, ref_scores=sc)


def test_swap_inside_tie_band_passes_as_tie():
    # k-th (3.0) and (k+1)-th (2.9999) are within 1e-3 relative
    p, x, ids, sc, kth, kn = setup_row([1.0, 5.0, 3.0, 2.9999])
    assert ids.tolist() == [1, 2]
    assert check_ids_row(p, x, 0, 0, 0, 3, [1, 3], ids, kth, kn, ref_scores=sc) is False


def test_reorder_between_near_equal_scores_passes_but_not_otherwise():
    p, x, ids, sc, kth, kn = setup_row([4.0, 4.0001, 1.0, 0.0])
    assert ids.tolist() == [1, 0]
    assert check_ids_row(p, x, 0, 0, 0, 3, [0, 1], ids, kth, kn, ref_scores=sc)
    p, x, ids, sc, kth, kn = setup_row([4.0, 6.0, 1.0, 0.0])
    with pytest.raises(AssertionError):
        check_ids_row(p, x, 0, 0, 0, 3, [0, 1], ids, kth, kn, ref_scores=sc)


def test_band_member_outside_band_fails():
    p, x, ids, sc, kth, kn = setup_row([1.0, 5.0, 3.0, 2.9999, 0.1])
    with pytest.raises(AssertionError):
        check_ids_row(p, x, 0, 0, 0, 4, [1, 4], ids, kth, kn, ref_scores=sc)
