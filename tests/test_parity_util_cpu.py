"""The comparison rules of the GPU parity tests, checked on the CPU with
planted errors: each rule accepts the oracle's own values and rejects a
value outside its tolerance, a NaN (an entry the kernel never wrote), a
missed clear winner, a kept clear loser, a duplicate and bad padding."""
import numpy as np
import pytest

import oracle
from parity_util import (ATTN_ATOL, attn_bound, check_attention, check_scores,
                         check_topk_band)


def _scores():
    rng = np.random.default_rng(4)
    q, w, k = rng.standard_normal((1, 6, 3, 8)), rng.standard_normal((1, 6, 3)), rng.standard_normal((1, 40, 8))
    ref = oracle.indexer_scores(q, w, k, 34)
    absum = np.einsum("bih,bihs->bis", np.abs(w), np.einsum("bihd,bsd->bihs", np.abs(q), np.abs(k)))
    return ref, absum


def test_check_scores():
    ref, absum = _scores()
    check_scores(ref.copy(), ref, absum, 34, rel=1e-4)
    ok = ref.copy()
    ok[0, 2, 37] += 0.5e-4 * absum[0, 2, 37]                  # inside the tolerance
    ok[0, 0, 39] = np.nan                                      # s > t: never compared
    check_scores(ok, ref, absum, 34, rel=1e-4)
    for s, v in ((30, None), (36, np.nan)):
        bad = ref.copy()
        bad[0, 2, s] = bad[0, 2, s] + 2e-4 * absum[0, 2, s] if v is None else v
        with pytest.raises(AssertionError, match="score mismatch"):
            check_scores(bad, ref, absum, 34, rel=1e-4)


def test_check_topk_band():
    ref, _ = _scores()
    k = 10
    idx = oracle.topk_indices(ref, 34, k)
    assert check_topk_band(idx, ref, 34, k) == 0
    t = 34 + 3
    sc = ref[0, 3, : t + 1]
    order = np.argsort(-sc)
    mutations = {
        "missed a clear winner": lambda r: np.sort(np.r_[np.setdiff1d(r, [order[0]]), order[-1]]),
        "kept a clear loser": lambda r: np.sort(np.r_[np.setdiff1d(r, [order[k - 1]]), order[-1]]),
        "ascending / duplicates": lambda r: np.r_[r[:-1], r[-2]],
        "range": lambda r: np.r_[r[:-1], t + 1],
    }
    for what, f in mutations.items():
        bad = idx.copy()
        bad[0, 3] = f(idx[0, 3])
        with pytest.raises(AssertionError, match=what.split()[0]):
            check_topk_band(bad, ref, 34, k)
    short = oracle.topk_indices(ref, 0, 8)                     # rows 0..5 keep t+1 <= 6 keys
    bad = short.copy()
    bad[0, 1, 5] = 3
    with pytest.raises(AssertionError, match="padding"):
        check_topk_band(bad, ref, 0, 8)


def test_check_attention():
    rng = np.random.default_rng(5)
    ref = rng.standard_normal((2, 3, 4, 16)) * 3
    check_attention(ref.copy(), ref)
    near = ref + 0.9 * attn_bound(ref) * rng.choice([-1, 1], ref.shape) * 0.01
    check_attention(near, ref)
    bad = ref.copy()
    bad[1, 2, 3, 4] += 2 * attn_bound(ref[1, 2, 3, 4])
    with pytest.raises(AssertionError, match="diff"):
        check_attention(bad, ref, "planted")
    # the bound is the larger of the two terms, not their sum: on an output of
    # 0.5 an error of 0.9e-2 passes and 1.1e-2 fails; on an output of 4.0,
    # 3.9e-2 passes and 4.1e-2 fails
    for v, ok_err, bad_err in ((0.5, 0.9e-2, 1.1e-2), (4.0, 3.9e-2, 4.1e-2)):
        base = np.full((40, 80), v)
        near = base.copy()
        near[2, 3] += ok_err
        check_attention(near, base, "near")
        bad = base.copy()
        bad[2, 3] += bad_err
        with pytest.raises(AssertionError, match="diff"):
            check_attention(bad, base, "planted")
    bad = ref.copy()
    bad[0, 0, 0, 0] = np.nan
    with pytest.raises(AssertionError, match="non-finite"):
        check_attention(bad, ref, "planted")
    # inside the elementwise bound everywhere, but a bias of 0.95 * atol on
    # outputs of size ~0.3 is ~3 % of their norm: the aggregate L2 rule fails
    small = ref / 10
    with pytest.raises(AssertionError, match="rel L2"):
        check_attention(small + 0.95 * ATTN_ATOL, small, "planted")
