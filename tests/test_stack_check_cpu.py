"""The stack checker of the full-size GPU tests, run on the CPU.

The oracle's own results must pass `check_stack`, and each planted mistake
(a changed S-layer index, a dropped clear winner in an F layer, a perturbed
or misplaced attention output) must fail it, so the checker that the GPU
workload tests rely on is itself tested without a GPU.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from cross_layer_top_full_b200 import synth
from parity_util import host64
from stack_check import check_stack, sample_rows


def _tiny(idx_dtype):
    return synth.Workload(
        "tiny_latent_" + idx_dtype, B=2, L=40, T=56, q_start=16, H_I=4, d_I=32, k=12, Hq=8,
        d_qk=48, d_v=32, idx_dtype=idx_dtype, attn_dtype="bf16", latent=True, pattern="FSSFS",
        seed=11, w_std=0.5, qI_std=1 / math.sqrt(32), kI_std=1 / math.sqrt(32), q_std=1.0,
        kv_std=1.0)


def _oracle_run(wl):
    """Layer inputs (torch, CPU) and the oracle's indices and outputs in the
    library's storage types (int32 indices, bf16 outputs)."""
    inputs = [synth.layer_inputs(wl, l, "cpu") for l in range(wl.n_layers)]
    fp8 = wl.idx_dtype == "e4m3"
    layers = []
    for inp in inputs:
        kv = host64(inp["kv"])
        d = {"q": host64(inp["q"]), "K": kv, "V": kv[..., : wl.d_v],
             "q_I": host64(inp["q_I"]), "w": host64(inp["w"]), "k_I": host64(inp["k_I"])}
        if fp8:
            d["q_scale"], d["k_scale"] = host64(inp["q_scale"]), host64(inp["k_scale"])
        layers.append(d)
    q_start = wl.T - wl.L
    idx, out, _ = oracle.layer_stack(wl.pattern, layers, q_start, wl.k, wl.scale, fp8=fp8)
    copies = [torch.as_tensor(x, dtype=torch.int32) for x in idx]
    outs = [torch.as_tensor(o).to(torch.bfloat16) for o in out]
    return inputs, copies, outs, q_start


@pytest.fixture(scope="module", params=["bf16", "e4m3"])
def run(request):
    wl = _tiny(request.param)
    return (wl,) + _oracle_run(wl)


ALL_LAYERS = range(5)


def _check(wl, inputs, copies, outs, q_start, attn_rows=(0, 3, 21, 39)):
    return check_stack(wl, wl.pattern, inputs, copies, outs, q_start, range(wl.B),
                       range(wl.L), attn_rows, ALL_LAYERS, wl.name)


def test_oracle_results_pass(run):
    wl, inputs, copies, outs, q_start = run
    n_cmp, n_same = _check(wl, inputs, copies, outs, q_start)
    assert n_cmp == n_same == wl.B * 4 * len(ALL_LAYERS)


def test_changed_s_layer_index_fails(run):
    wl, inputs, copies, outs, q_start = run
    bad = list(copies)
    bad[2] = copies[2].clone()
    bad[2][1, 30, 3] = -1
    with pytest.raises(AssertionError, match="S layer 2"):
        _check(wl, inputs, bad, outs, q_start)


def test_dropped_clear_winner_fails(run):
    wl, inputs, copies, outs, q_start = run
    i = wl.L - 1                                       # t + 1 = T > k: a real selection
    t = q_start + i
    sc = oracle.indexer_scores(host64(inputs[0]["q_I"][:1, i:i + 1]),
                               host64(inputs[0]["w"][:1, i:i + 1]), host64(inputs[0]["k_I"][:1]),
                               t, host64(inputs[0]["q_scale"][:1, i:i + 1])
                               if wl.idx_dtype == "e4m3" else None,
                               host64(inputs[0]["k_scale"][:1]) if wl.idx_dtype == "e4m3" else None,
                               fp8=wl.idx_dtype == "e4m3")[0, 0, : t + 1]
    best, worst = int(np.argmax(sc)), int(np.argmin(sc))
    row = copies[0][0, i].tolist()
    assert best in row and worst not in row
    row = sorted([worst if x == best else x for x in row])
    bad = [c.clone() for c in copies]
    for l in (0, 1, 2):                                # the F layer and the S layers reusing it
        bad[l][0, i] = torch.tensor(row, dtype=torch.int32)
    with pytest.raises(AssertionError):
        _check(wl, inputs, bad, outs, q_start)


def test_perturbed_attention_output_fails(run):
    wl, inputs, copies, outs, q_start = run
    bad = list(outs)
    bad[4] = outs[4].clone()
    bad[4][1, 21, 5, 7] += 0.25
    with pytest.raises(AssertionError, match="layer 4 seq 1 row 21"):
        _check(wl, inputs, copies, bad, q_start)


def test_misplaced_attention_rows_fail(run):
    wl, inputs, copies, outs, q_start = run
    bad = list(outs)
    bad[1] = outs[1].clone()
    bad[1][0, [3, 21]] = outs[1][0, [21, 3]]
    with pytest.raises(AssertionError):
        _check(wl, inputs, copies, bad, q_start)


def test_sample_rows():
    rows = sample_rows(100, 10, seed=5, always=(0, 1, 99, 150, -1))
    assert rows == sorted(set(rows)) and rows[0] == 0 and rows[-1] == 99 and 1 in rows
    assert 11 <= len(rows) <= 13 and all(0 <= r < 100 for r in rows)
    assert sample_rows(100, 10, seed=5) == sample_rows(100, 10, seed=5)
    assert sample_rows(5, 10, seed=0) == [0, 1, 2, 3, 4]
