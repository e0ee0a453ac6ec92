"""Algorithmic work counts behind the bench's roofline lines (CPU).

Each count is re-derived here from the workload's shape in closed form
(sums of arithmetic series), independently of bench.algorithmic's loops:
  causal pairs of L rows starting at q_start: sum_{t=q0}^{q0+L-1} (t+1);
  selected-row visits: sum_t min(k, t+1);
  indexer flop = 2*H_I*d_I per pair, attention flop = 2*Hq*(d_qk+d_v) per visit.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from cross_layer_top_full_b200 import synth  # noqa: E402


def _pairs(q0, L):
    a, b = q0 + 1, q0 + L            # sum of (t+1) for t = q0 .. q0+L-1
    return (a + b) * L // 2


def _visits(q0, L, k):
    lo, hi = q0, q0 + L - 1          # t range; min(k, t+1) = t+1 for t < k
    n_small = max(0, min(hi, k - 1) - lo + 1)
    small = _pairs(lo, n_small) if n_small else 0
    return small + k * (L - n_small)


@pytest.mark.parametrize("name", ["prefill_512_fp32", "prefill_8k_bf16", "decode_b32_t32k_bf16",
                                  "decode_b8_t200k_fp8"])
def test_counts_match_closed_forms(name):
    wl = synth.WORKLOADS[name]
    w = bench.algorithmic(wl)
    pairs = wl.B * _pairs(wl.q_start, wl.L)
    visits = wl.B * _visits(wl.q_start, wl.L, wl.k)
    assert w["pairs"] == pairs
    assert w["visits"] == visits
    assert w["indexer_flop"] == pytest.approx(2 * wl.H_I * wl.d_I * pairs)
    assert w["attn_flop"] == pytest.approx(2 * wl.Hq * (wl.d_qk + wl.d_v) * visits)


def test_prefill_8k_figures():
    """L = 8192 from position 0, H_I = 64, d_I = 128, k = 2048, 128 heads, 576/512."""
    w = bench.algorithmic(synth.WORKLOADS["prefill_8k_bf16"])
    assert w["pairs"] == 8192 * 8193 // 2                       # 33.56 M causal pairs
    assert w["indexer_flop"] == pytest.approx(0.5498e12, rel=1e-3)
    # rows t < 2047 see t+1 keys, the other 6145 rows see 2048
    assert w["visits"] == 2048 * 2049 // 2 + 2048 * (8192 - 2048)
    assert w["attn_flop"] == pytest.approx(4.088e12, rel=1e-3)


def test_decode_bytes():
    """Decode: the indexer reads every cached key once; attention gathers k rows."""
    c2 = bench.algorithmic(synth.WORKLOADS["decode_b32_t32k_bf16"])
    assert c2["pairs"] == 32 * 32768
    kI = 32 * 32768 * 128 * 2
    assert c2["indexer_bytes"] == pytest.approx(kI + 32 * 64 * (128 * 2 + 4) + 4 * 32 * 32768)
    kv = 32 * 2048 * 576 * 2
    assert c2["attn_bytes"] == pytest.approx(kv + 32 * 128 * (576 + 512) * 2 + 4 * 32 * 2048)
    c4 = bench.algorithmic(synth.WORKLOADS["decode_b8_t200k_fp8"])
    assert c4["indexer_bytes"] == pytest.approx(8 * 200000 * 128 + 8 * 64 * (128 + 4)
                                                + 4 * 8 * 200000)
    assert c4["attn_bytes"] == pytest.approx(8 * 2048 * 1152 + 8 * 128 * 1088 * 2 + 4 * 8 * 2048)


def test_roofline_line_uses_the_dominant_stage():
    wl = synth.WORKLOADS["prefill_8k_bf16"]
    work = bench.algorithmic(wl)
    roof, dom = bench.roofline(wl, work, {"indexer": 0.5, "topk": 0.5, "attention": 40.0},
                               {"indexer": 1, "topk": 1, "attention": 4})
    assert dom == "attention" and roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s"
    assert roof["achieved"] == pytest.approx(work["attn_flop"] / 10e-3 / 1e12)
    assert roof["frac"] == pytest.approx(roof["achieved"] / roof["peak"])
    wl = synth.WORKLOADS["decode_b32_t32k_bf16"]
    roof, dom = bench.roofline(wl, bench.algorithmic(wl), {"indexer": 0.2, "topk": 0.1,
                                                           "attention": 0.6},
                               {"indexer": 2, "topk": 2, "attention": 8})
    assert dom == "attention" and roof["bound"] == "hbm" and roof["unit"] == "GB/s"


def test_row_overlap_matches_the_oracle():
    """The chunked run's S-layer overlap equals the oracle's definition,
    |A & B| / |A| with A the reused set, on ragged (-1 padded) rows."""
    import numpy as np
    import torch
    import oracle
    rng = np.random.default_rng(7)
    T, k, rows = 300, 40, 64
    reused = np.full((rows, k), -1, dtype=np.int32)
    own = np.full((rows, k), -1, dtype=np.int32)
    for r in range(rows):
        m = int(rng.integers(1, k + 1))           # t + 1 < k gives padded rows
        pool = rng.choice(T, size=min(T, 2 * k), replace=False)
        reused[r, :m] = np.sort(rng.choice(pool, m, replace=False))
        own[r, :m] = np.sort(rng.choice(pool, m, replace=False))
    got = bench.row_overlap(torch.from_numpy(reused), torch.from_numpy(own), T).numpy()
    ref = oracle.topk_overlap(reused, own)
    assert np.array_equal(got, ref)
    assert np.all(bench.row_overlap(torch.from_numpy(reused), torch.from_numpy(reused), T).numpy() == 1.0)


@pytest.mark.parametrize("name,timed", [("prefill_8k_bf16", 4), ("decode_b32_t32k_bf16", 8),
                                        ("decode_b8_t200k_fp8", 4)])
def test_cpu_baseline_says_which_layers_the_oracle_timed(name, timed):
    wl = synth.WORKLOADS[name]
    assert len(bench.oracle_layers(wl, wl.pattern)) == timed
    cb = bench.cpu_baseline(wl, wl.pattern, 1.5, 7, 12.0, "query rows")
    assert cb["kind"] == "oracle" and cb["unit"] == "tok/s" and cb["value"] == 1.5
    assert cb["cores"] >= 1 and cb["cpu_model"]
    if timed < len(wl.pattern):
        assert "first %d of the %d layers" % (timed, len(wl.pattern)) in cb["sample"]
    else:
        assert "all %d layers" % timed in cb["sample"]


def test_oracle_stage_clock_times_each_stage_and_restores_the_oracle():
    import oracle.indexcache_oracle as om
    before = (om.indexer_scores, om.topk_indices, om.sparse_attention)
    wl = synth.WORKLOADS["prefill_512_fp32"]
    clock = bench.OracleStageClock()
    rate, done, spent = bench.oracle_sample(wl, wl.pattern, 0.3, clock)
    assert (om.indexer_scores, om.topk_indices, om.sparse_attention) == before
    assert rate > 0 and done > 0
    # FSSS: one indexer and top-k pass per row, four attention passes
    assert clock.rows["indexer"] == clock.rows["topk"] == done
    assert clock.rows["attention"] == 4 * done
    per_row = clock.per_row_ms()
    assert all(per_row[s] > 0 for s in ("indexer", "topk", "attention"))
    assert sum(clock.seconds.values()) <= spent
    cb = bench.cpu_baseline(wl, wl.pattern, rate, done, spent, "query rows", clock)
    assert cb["per_row_ms"] == per_row


def test_overlap_matrix_matches_the_oracle():
    """The all-pairs layer overlap matrix equals the oracle's topk_overlap,
    pair by pair, on ragged (-1 padded) ascending rows."""
    import numpy as np
    import torch
    import oracle
    rng = np.random.default_rng(3)
    T, k, rows, L = 60, 8, 7, 4
    sets = []
    for _ in range(L):
        a = np.full((rows, k), -1, dtype=np.int32)
        for r in range(rows):
            m = int(rng.integers(1, k + 1))
            a[r, :m] = np.sort(rng.choice(T, m, replace=False))
        sets.append(a)
    s_sum, s_min, n = bench.overlap_matrix([torch.from_numpy(a) for a in sets], T)
    assert n == rows
    for l in range(L):
        for m in range(L):
            ref = oracle.topk_overlap(sets[l], sets[m])
            assert s_sum[l, m].item() == pytest.approx(ref.sum())
            assert s_min[l, m].item() == pytest.approx(ref.min())
        assert s_sum[l, l].item() == pytest.approx(rows)
    js = bench.overlap_json(s_sum, s_min, n, "test")
    assert js["layers"] == L and len(js["mean"]) == L and js["mean"][0][0] == 1.0


def test_varlen_counts_follow_the_sequence_lengths():
    """A variable-length batch: pairs, visits and bytes from each sequence's
    own length (closed forms per sequence), and the fused selection's bytes
    carry no score traffic."""
    wl = synth.WORKLOADS["decode_b32_varlen_paged_bf16"]
    lens = [32768, 5000, 4096, 20000]
    w = bench.algorithmic(wl, lens)
    assert w["pairs"] == sum(lens)                        # one query row at t = n - 1 each
    assert w["visits"] == sum(min(wl.k, n) for n in lens)
    q_side = wl.B * 1 * wl.H_I * (wl.d_I * 2 + 4)
    assert w["indexer_bytes"] == pytest.approx(sum(lens) * wl.d_I * 2 + q_side + 4 * sum(lens))
    assert w["select_bytes"] == pytest.approx(sum(lens) * wl.d_I * 2 + q_side + 4 * wl.B * wl.k)
    assert bench.path_stages(wl) == ("select", "attention")
    assert bench.path_stages(synth.WORKLOADS["prefill_8k_bf16"]) == ("indexer", "topk", "attention")
