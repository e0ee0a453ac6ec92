"""Float64 CPU oracle for the IndexCache hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this
module: it is used by ``tests/``, by ``__graft_entry__.smoke()`` to check a
small GPU run, and by ``bench.py`` to time a CPU baseline.  It shares no code
with the CUDA path and deliberately does no blocking, fusion or reordering
beyond what each definition below states, so a reader can check it by eye
against the pages.

Sources ("the pages" = the summaries of *IndexCache: Accelerating Sparse
Attention via Cross-Layer Index Reuse* on gist.science, in es/pt/it/de):

* Lightning indexer + top-k + sparse core attention, O(L^2) indexer vs O(Lk)
  attention: es page, section 1 "El Problema"; pt page, section 1
  "O Problema"; de page, section 1 "Problemstellung".
* F/S layer partition by a binary pattern, S layers reusing the indices of
  the nearest preceding F layer, one temporary index tensor, one conditional
  branch: es page, section 2 "Arquitectura del Método"; pt page, section 2
  "Arquitetura"; it page, section 2 "Architettura e Funzionamento"; de page,
  section 2 "Methodik: IndexCache".

The pages do not print the indexer's formula, the attention variant, the
tie-break or the FP8 format.  The readings taken (each restated where it is
used) are:

* indexer score  I[t,s] = sum_h w[t,h] * ReLU(q_I[t,h,:] . k_I[s,:]) over the
  causal candidates s <= t (a row sees its own key);
* top-k keeps the min(k, t+1) largest scores, equal scores going to the
  smaller position, and returns the positions in ascending order padded
  with -1;
* FP8 inputs are OCP E4M3 ("FN": no infinities, S.1111.111 is NaN) codes
  with one non-negative float32 scale per token: value = decode(code)*scale;
* sparse attention is multi-query attention: every query head attends over
  the same selected key/value rows with a plain softmax.

parity: every function here is pinned by ``tests/test_oracle_pins.py``
against brute force, closed forms or an independent library routine.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np

__all__ = [
    "e4m3_decode",
    "indexer_scores",
    "topk_indices",
    "sparse_attention",
    "dense_causal_attention",
    "validate_pattern",
    "layer_stack",
    "topk_overlap",
]


# ---------------------------------------------------------------------------
# FP8 E4M3 ("FN" variant of the OCP 8-bit floating point format)
# ---------------------------------------------------------------------------
def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Decode OCP E4M3FN byte codes to float64.

    Format (OCP 8-bit floating point specification, E4M3): 1 sign bit,
    4 exponent bits with bias 7, 3 mantissa bits.  Exponent field 0 encodes
    subnormals  (-1)^s * 2^-6 * m/8 ; other exponents encode normals
    (-1)^s * 2^(e-7) * (1 + m/8).  There are no infinities; the two codes with
    all exponent and mantissa bits set (0x7F, 0xFF) are NaN, so the largest
    finite magnitude is 2^8 * 1.75 = 448.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    sub = sign * (2.0 ** -6) * (m / 8.0)
    nrm = sign * np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    out = np.where(e == 0, sub, nrm)
    out = np.where((e == 0xF) & (m == 0x7), np.nan, out)
    return out.astype(np.float64)


def _dequant(x: np.ndarray, scale: Optional[np.ndarray], fp8: bool) -> np.ndarray:
    """Values of an indexer operand: FP8 codes times their per-token scale,
    or the stored floating-point values upcast exactly to float64."""
    if not fp8:
        return np.asarray(x, dtype=np.float64)
    v = e4m3_decode(x)
    s = np.asarray(scale, dtype=np.float64)
    # one scale per token: broadcast over every trailing axis of that token
    return v * s.reshape(s.shape + (1,) * (v.ndim - s.ndim))


# ---------------------------------------------------------------------------
# a1: lightning indexer (F layers only)
# ---------------------------------------------------------------------------
def indexer_scores(q_I, w, k_I, q_start: int, q_scale=None, k_scale=None,
                   fp8: bool = False, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """Indexer scores of every query row against every causal key.

    The indexer scores all preceding tokens of each query (es page, section 1;
    pt page, section 1 "O Gargalo do Indexador").  Score form (reading, not
    printed on the pages):
        I[b,i,s] = sum_h w[b,i,h] * max(0, sum_d q_I[b,i,h,d] * k_I[b,s,d])
    for s <= t = q_start + i, and -inf for s > t (not a candidate).

    Shapes: q_I [B,Lq,H,d], w [B,Lq,H], k_I [B,T,d]; with ``fp8`` the two
    operands are E4M3 codes and q_scale [B,Lq], k_scale [B,T] their per-token
    scales.  ``rows`` optionally restricts the output to those query rows i
    (the result then has len(rows) rows).  Returns float64 [B, n_rows, T].
    """
    q = _dequant(q_I, q_scale, fp8)            # [B,Lq,H,d]
    k = _dequant(k_I, k_scale, fp8)            # [B,T,d]
    wv = np.asarray(w, dtype=np.float64)       # [B,Lq,H]
    B, Lq, H, d = q.shape
    T = k.shape[1]
    row_ids = list(range(Lq)) if rows is None else list(rows)
    out = np.full((B, len(row_ids), T), -np.inf, dtype=np.float64)
    for b in range(B):
        for r, i in enumerate(row_ids):
            t = q_start + i
            dots = q[b, i] @ k[b, : t + 1].T           # [H, t+1]: q_I[t,h] . k_I[s]
            relu = np.maximum(dots, 0.0)
            out[b, r, : t + 1] = wv[b, i] @ relu        # sum over heads of w * ReLU
    return out


# ---------------------------------------------------------------------------
# a2: top-k selection
# ---------------------------------------------------------------------------
def topk_indices(scores: np.ndarray, q_start: int, k: int,
                 rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """Per query row, the positions of the k highest-scoring causal keys.

    DSA keeps the k most relevant tokens per query (es page, section 1).
    Readings: candidates of row t are s in [0, t]; the winners are the first
    min(k, t+1) candidates in the order (score descending, position
    ascending), i.e. equal scores go to the smaller position and -0.0 equals
    +0.0; the winners are returned in ascending position order, the rest of
    the k slots hold -1.

    ``scores`` is [B, n_rows, >=T]; ``rows`` gives the absolute row i of each
    of the n_rows (default 0..n_rows-1).  Returns int32 [B, n_rows, k].
    """
    s = np.asarray(scores, dtype=np.float64)
    B, n_rows = s.shape[0], s.shape[1]
    row_ids = list(range(n_rows)) if rows is None else list(rows)
    out = np.full((B, n_rows, k), -1, dtype=np.int32)
    for b in range(B):
        for r, i in enumerate(row_ids):
            t = q_start + i
            cand = s[b, r, : t + 1]
            pos = np.arange(t + 1)
            # full sort: primary key -score (descending score), secondary key
            # position (ascending); np.lexsort sorts by the LAST key first.
            order = np.lexsort((pos, -cand))
            take = min(k, t + 1)
            chosen = np.sort(pos[order[:take]])
            out[b, r, :take] = chosen
    return out


# ---------------------------------------------------------------------------
# a4: sparse multi-query attention over the selected rows (every layer)
# ---------------------------------------------------------------------------
def sparse_attention(q, K, V, idx, scale: float) -> np.ndarray:
    """Attention of every query head over only its row's selected keys.

    Core attention restricted to the k selected tokens, O(Lk) (es page,
    section 1; de page, section 1).  Multi-query form (reading): for row
    (b,i), head h and J = the entries of idx[b,i] that are >= 0,
        p_j = softmax_j( scale * q[b,i,h,:] . K[b,j,:] )
        out[b,i,h,:] = sum_j p_j * V[b,j,:]
    The softmax subtracts the row maximum before exponentiating (exact in
    real arithmetic).  An empty J gives a zero output row.

    Shapes: q [B,Lq,Hq,d_qk], K [B,T,d_qk], V [B,T,d_v], idx [B,Lq,k].
    Returns float64 [B,Lq,Hq,d_v].
    """
    qv = np.asarray(q, dtype=np.float64)
    Kv = np.asarray(K, dtype=np.float64)
    Vv = np.asarray(V, dtype=np.float64)
    ix = np.asarray(idx)
    B, Lq, Hq, _ = qv.shape
    d_v = Vv.shape[-1]
    out = np.zeros((B, Lq, Hq, d_v), dtype=np.float64)
    for b in range(B):
        for i in range(Lq):
            J = ix[b, i][ix[b, i] >= 0].astype(np.int64)
            if J.size == 0:
                continue
            logits = scale * (qv[b, i] @ Kv[b, J].T)           # [Hq, |J|]
            m = logits.max(axis=1, keepdims=True)
            e = np.exp(logits - m)
            p = e / e.sum(axis=1, keepdims=True)
            out[b, i] = p @ Vv[b, J]                           # [Hq, d_v]
    return out


def dense_causal_attention(q, K, V, q_start: int, scale: float) -> np.ndarray:
    """Ordinary dense causal attention, written independently of
    :func:`sparse_attention`: full logits matrix, -inf above the diagonal,
    softmax along keys.  With k >= t+1 for every row the selected set is all
    causal keys, so the two functions must agree (the O(Lk) attention is the
    O(L^2) attention restricted to the selected keys)."""
    qv = np.asarray(q, dtype=np.float64)
    Kv = np.asarray(K, dtype=np.float64)
    Vv = np.asarray(V, dtype=np.float64)
    B, Lq, Hq, _ = qv.shape
    T = Kv.shape[1]
    t = q_start + np.arange(Lq)[:, None]                      # [Lq,1]
    s = np.arange(T)[None, :]                                 # [1,T]
    mask = s <= t                                             # [Lq,T]
    out = np.empty((B, Lq, Hq, Vv.shape[-1]), dtype=np.float64)
    for b in range(B):
        logits = scale * np.einsum("ihd,sd->ihs", qv[b], Kv[b])
        logits = np.where(mask[:, None, :], logits, -np.inf)
        w = np.exp(logits - logits.max(axis=-1, keepdims=True))
        w /= w.sum(axis=-1, keepdims=True)
        out[b] = np.einsum("ihs,sd->ihd", w, Vv[b])
    return out


# ---------------------------------------------------------------------------
# a3: the F/S branch over a layer stack
# ---------------------------------------------------------------------------
def validate_pattern(pattern: str, n_layers: int) -> None:
    """The binary pattern partitions the N layers into F and S (es page,
    section 2 "Arquitectura del Método").  An S layer inherits from the
    nearest *preceding* F layer, so a pattern that starts with S has nothing
    to inherit (reading: an error)."""
    if len(pattern) != n_layers:
        raise ValueError("pattern length %d != number of layers %d" % (len(pattern), n_layers))
    if any(c not in "FS" for c in pattern):
        raise ValueError("pattern may only hold 'F' and 'S'")
    if n_layers > 0 and pattern[0] != "F":
        raise ValueError("the first layer must be F: an S layer needs a preceding F layer")


def layer_stack(pattern: str, layers: List[Dict], q_start: int, k: int, scale: float,
                fp8: bool = False, rows: Optional[Sequence[int]] = None):
    """Run the IndexCache stack: F layers compute fresh top-k indices and
    store them in the (single) index cache; S layers skip the indexer and use
    the cached indices unchanged; every layer runs sparse attention
    (es page, section 2 "Arquitectura del Método": one conditional branch,
    one temporary index tensor).

    Each layer dict holds 'q', 'K', 'V' and, for F layers, 'q_I', 'w', 'k_I'
    (plus 'q_scale', 'k_scale' with ``fp8``).  ``rows`` restricts the check
    to those query rows (the cache then holds only those rows).  Returns
    (idx per layer, out per layer, number of indexer evaluations).
    """
    validate_pattern(pattern, len(layers))
    idx_cache = None
    idx_all, out_all = [], []
    n_indexer = 0
    for l, kind in enumerate(pattern):
        L = layers[l]
        if kind == "F":
            sc = indexer_scores(L["q_I"], L["w"], L["k_I"], q_start,
                                L.get("q_scale"), L.get("k_scale"), fp8=fp8, rows=rows)
            idx_cache = topk_indices(sc, q_start, k, rows=rows)
            n_indexer += 1
        q = L["q"] if rows is None else np.asarray(L["q"])[:, list(rows)]
        out = sparse_attention(q, L["K"], L["V"], idx_cache, scale)
        idx_all.append(idx_cache)
        out_all.append(out)
    return idx_all, out_all, n_indexer


def topk_overlap(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Per row, |A ∩ B| / |A| of two index sets (the -1 padding ignored).
    This is the cross-layer overlap the pages report between adjacent
    layers' top-k selections (pt page, section 1 "Observação Chave")."""
    a = np.asarray(a)
    b = np.asarray(b)
    flat_a = a.reshape(-1, a.shape[-1])
    flat_b = b.reshape(-1, b.shape[-1])
    res = np.empty(flat_a.shape[0], dtype=np.float64)
    for r in range(flat_a.shape[0]):
        A = set(int(x) for x in flat_a[r] if x >= 0)
        Bs = set(int(x) for x in flat_b[r] if x >= 0)
        res[r] = len(A & Bs) / max(1, len(A))
    return res.reshape(a.shape[:-1])
