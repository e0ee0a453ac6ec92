"""Checks of one F/S layer-stack run against the oracle, on sampled outputs
the oracle computes one by one (test infrastructure).

`check_stack` takes the library's per-layer indices and outputs and the
layer inputs (tensors on any device) and verifies:
  * F layer: the indices of every row in `idx_rows` (of every sequence in
    `seqs`) obey the top-k band rule against the oracle's float64 scores;
  * S layer: its indices are the preceding F layer's, bit for bit (all rows);
  * attention, on `attn_layers` for EVERY row of `attn_rows`: the output is
    within the attention tolerance of the oracle's float64 attention over the
    index set the library used.  That set has passed the band rule above (F
    rows) or equals the F layer's bit for bit (S rows), so it is a valid
    top-k of the row; where it differs from the oracle's own exact top-k
    (an allowed near-tie swap) the oracle still computes the attention of
    the keys the library chose, so no row escapes the comparison.
The oracle reads only the selected KV rows, gathered by torch indexing, so
host memory stays bounded at full size.  The GPU workload tests call it on the library's
results; a CPU test runs it on the oracle's own results and on planted
mistakes, so the checker itself is tested without a GPU.
"""
import numpy as np
import torch

import oracle
from parity_util import check_attention, check_topk_band, host64


def sample_rows(n, count, seed, always=()):
    """Sorted union of `always` (clipped to [0, n)) and `count` seeded
    distinct rows of [0, n)."""
    rng = np.random.default_rng(seed)
    pick = rng.choice(n, min(count, n), replace=False).tolist()
    return sorted(set([r for r in always if 0 <= r < n] + pick))


def oracle_scores(wl, inp, q_start, rows, seqs, block=256):
    """float64 indexer scores [len(seqs), len(rows), T] of query rows `rows`
    (relative to the call's q_start) of sequences `seqs`, from the layer's
    device inputs; -inf beyond each row's causal range."""
    fp8 = wl.idx_dtype == "e4m3"
    T = inp["k_I"].shape[1]
    rows = list(rows)
    out = np.full((len(seqs), len(rows), T), -np.inf)
    for bi, b in enumerate(seqs):
        kI = host64(inp["k_I"][b:b + 1])
        ks = host64(inp["k_scale"][b:b + 1]) if fp8 else None
        for r0 in range(0, len(rows), block):
            sel = torch.as_tensor(rows[r0:r0 + block], dtype=torch.long,
                                  device=inp["q_I"].device)
            qI = host64(inp["q_I"][b:b + 1].index_select(1, sel))
            w = host64(inp["w"][b:b + 1].index_select(1, sel))
            qs = host64(inp["q_scale"][b:b + 1].index_select(1, sel)) if fp8 else None
            n = qI.shape[1]
            # row j of this block sits at t = q_start + rows[r0 + j]
            for j in range(n):
                i = rows[r0 + j]
                sc = oracle.indexer_scores(qI[:, j:j + 1], w[:, j:j + 1], kI, q_start + i,
                                           qs[:, j:j + 1] if fp8 else None, ks, fp8=fp8)
                out[bi, r0 + j] = sc[0, 0]
    return out


def oracle_attention_row(wl, inp, ref_idx, b, i):
    """Oracle output [Hq, d_v] of row (b, i) over the key positions ref_idx [k]
    (-1 entries skipped)."""
    J = torch.as_tensor(ref_idx[ref_idx >= 0], dtype=torch.long, device=inp["kv"].device)
    kvJ = host64(inp["kv"][b].index_select(0, J))          # only the selected rows
    q = host64(inp["q"][b, i])[None, None]
    pos = np.arange(kvJ.shape[0], dtype=np.int32)[None, None]
    return oracle.sparse_attention(q, kvJ[None], kvJ[None, :, : wl.d_v], pos, wl.scale)[0, 0]


def check_stack(wl, pattern, inputs, copies, outs, q_start, seqs, idx_rows, attn_rows,
                attn_layers, what):
    """Check one stack run (see the module docstring).  copies[l] [B, L, k]
    int32 and outs[l] [B, L, Hq, d_v] are the library's indices and outputs
    of layer l; attn_rows must be a subset of idx_rows.  Returns
    (attention rows compared, of those the rows whose index set equals the
    oracle's exact top-k); every row counted in the first is compared."""
    seqs, idx_rows, attn_rows = list(seqs), list(idx_rows), list(attn_rows)
    where = {i: r for r, i in enumerate(idx_rows)}
    assert all(i in where for i in attn_rows), "attention rows must have oracle indices"
    n_cmp = n_same = 0
    last_f, ref_idx = None, None
    for l, kind in enumerate(pattern):
        gidx = host64(copies[l])
        if kind == "F":
            last_f = l
            sc = oracle_scores(wl, inputs[l], q_start, idx_rows, seqs)
            check_topk_band(gidx[seqs][:, idx_rows], sc, q_start, wl.k, rows=idx_rows)
            ref_idx = oracle.topk_indices(sc, q_start, wl.k, rows=idx_rows)
            del sc
        else:
            assert last_f is not None and np.array_equal(gidx, host64(copies[last_f])), \
                "%s: S layer %d does not hold the F layer's indices" % (what, l)
        if l not in attn_layers:
            continue
        sel = torch.as_tensor(attn_rows, dtype=torch.long, device=outs[l].device)
        for bi, b in enumerate(seqs):
            got = host64(outs[l][b].index_select(0, sel))
            for a, i in enumerate(attn_rows):
                n_cmp += 1
                # the band rule (F) or bit-exact reuse (S) has validated gidx[b, i]
                if np.array_equal(gidx[b, i], ref_idx[bi, where[i]]):
                    n_same += 1
                ref = oracle_attention_row(wl, inputs[l], gidx[b, i], b, i)
                check_attention(got[a], ref, "%s layer %d seq %d row %d" % (what, l, b, i))
    return n_cmp, n_same
