"""Comparison rules shared by the GPU parity tests (test infrastructure).

* indexer scores: |gpu - oracle| <= rel * (sum_h |w_h| * sum_d |q_hd k_d|),
  i.e. relative to the sum of absolute terms, the scale on which float32
  accumulation errors live (d_I products then H_I head terms, each rounding
  at most 2^-24 relative: (d_I + H_I) * 2^-24 ~ 1.1e-5 for d_I=128, H_I=64;
  the tests allow 1e-4).  Bit-exact in exact mode.
* top-k on identical inputs: bit-exact.  Against the oracle's own float64
  scores (general inputs): the band rule -- with tau the k-th largest oracle
  score, every position scoring above tau + 1e-3|tau| is kept and every kept
  position scores at least tau - 1e-3|tau|; no duplicates, all in [0, t],
  ascending, -1 padded, exactly min(k, t+1) kept.
* attention: "within 1e-2 max abs and 1e-2 relative" read elementwise as
  |gpu - oracle| <= max(1e-2, 1e-2 |oracle|): 1e-2 absolute, relaxed to 1e-2
  relative only where the output is larger than 1 (a pure 1e-2 absolute
  bound cannot hold for bf16 outputs of magnitude >= 2, whose rounding step
  alone is 2^-7 or more), plus the aggregate
  ||gpu - oracle||_2 <= 1e-2 ||oracle||_2.  The bf16 rounding of the softmax
  weights (the P.V operand) and of the output stays about 4e-3 inside it
  even at sharp logits (base-2 logits of 100 and more).
"""
import numpy as np
import torch

ATTN_ATOL = 1e-2
ATTN_RTOL = 1e-2
ATTN_REL_L2 = 1e-2
TOPK_BAND = 1e-3


def host64(x: torch.Tensor) -> np.ndarray:
    """Exact float64 (or int) host copy of a device tensor."""
    if x.dtype in (torch.uint8, torch.int32, torch.int64):
        return x.cpu().numpy()
    return x.detach().to(torch.float64).cpu().numpy()


def abs_term_sum(q_I: np.ndarray, w: np.ndarray, k_I: np.ndarray, rows=None) -> np.ndarray:
    """sum_h |w_h| * sum_d |q_hd| |k_d| for every (row, key): [B, n_rows, T]."""
    q = np.abs(q_I if rows is None else q_I[:, list(rows)])
    wv = np.abs(w if rows is None else w[:, list(rows)])
    out = np.empty((q.shape[0], q.shape[1], k_I.shape[1]))
    for b in range(q.shape[0]):
        dots = np.einsum("ihd,sd->ihs", q[b], np.abs(k_I[b]))
        out[b] = np.einsum("ih,ihs->is", wv[b], dots)
    return out


def check_scores(gpu: np.ndarray, ref: np.ndarray, absum: np.ndarray, q_start: int, rel: float,
                 rows=None) -> None:
    """gpu/ref/absum: [B, n_rows, >=T]; only causal entries are compared."""
    B, n = ref.shape[0], ref.shape[1]
    row_ids = list(range(n)) if rows is None else list(rows)
    for b in range(B):
        for r, i in enumerate(row_ids):
            t = q_start + i
            g = gpu[b, r, : t + 1]
            e = ref[b, r, : t + 1]
            tol = rel * absum[b, r, : t + 1]
            bad = ~(np.abs(g - e) <= tol)        # a NaN (an unwritten entry) is bad too
            if bad.any():
                s = int(np.argmax(bad))
                raise AssertionError("score mismatch b=%d row=%d s=%d gpu=%r ref=%r tol=%r"
                                     % (b, i, s, g[s], e[s], tol[s]))


def check_topk_band(idx: np.ndarray, ref_scores: np.ndarray, q_start: int, k: int,
                    rows=None, band: float = TOPK_BAND) -> int:
    """Band rule; returns the number of rows whose set differs from the
    oracle's exact top-k (allowed near-tie swaps)."""
    B, n = idx.shape[0], idx.shape[1]
    row_ids = list(range(n)) if rows is None else list(rows)
    differ = 0
    for b in range(B):
        for r, i in enumerate(row_ids):
            t = q_start + i
            row = idx[b, r]
            m = min(k, t + 1)
            sel = row[:m]
            assert np.all(row[m:] == -1), (b, i, "padding")
            assert np.all(sel >= 0) and np.all(sel <= t), (b, i, "range")
            assert np.all(np.diff(sel) > 0), (b, i, "ascending / duplicates")
            if m == t + 1:
                assert np.array_equal(sel, np.arange(t + 1)), (b, i, "all candidates")
                continue
            sc = ref_scores[b, r, : t + 1]
            tau = np.sort(sc)[::-1][k - 1]
            eps = band * abs(tau)
            must = np.nonzero(sc > tau + eps)[0]
            assert np.all(np.isin(must, sel)), (b, i, "missed a clear winner")
            assert np.all(sc[sel] >= tau - eps), (b, i, "kept a clear loser")
            exact = np.lexsort((np.arange(t + 1), -sc))[:k]
            if not np.array_equal(np.sort(exact), sel):
                differ += 1
    return differ


def attn_bound(ref: np.ndarray) -> np.ndarray:
    """Elementwise attention bound max(1e-2, 1e-2 |ref|)."""
    return np.maximum(ATTN_ATOL, ATTN_RTOL * np.abs(ref))


def check_attention(gpu: np.ndarray, ref: np.ndarray, what: str = "") -> None:
    if not np.all(np.isfinite(gpu)):
        at = np.unravel_index(int(np.argmin(np.isfinite(gpu))), gpu.shape)
        raise AssertionError("%s non-finite output %r at %s" % (what, gpu[at], at))
    d = np.abs(gpu - ref)
    excess = d - attn_bound(ref)
    worst = float(excess.max()) if d.size else -1.0
    rel = float(np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-30))
    if worst > 0:
        at = np.unravel_index(int(np.argmax(excess)), d.shape)
        raise AssertionError("%s |diff| %g > max(%g, %g*|ref|) at %s (ref %g)"
                             % (what, d[at], ATTN_ATOL, ATTN_RTOL, at, ref[at]))
    assert rel <= ATTN_REL_L2, "%s rel L2 = %g" % (what, rel)
