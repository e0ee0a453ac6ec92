"""Full-size parity of the four large workloads, in the launch configuration
the benchmark times (the whole F/S stack through ic_layer_stack_forward).

The oracle cannot redo a full workload in float64 within a test, so each
check covers sampled outputs the oracle computes one by one: sampled query
rows (prefill) or every sequence of a few layers (decode).  Per checked row:
  * F layer: the kernel's indices obey the top-k band rule against the
    oracle's float64 scores;
  * S layer: its indices are the preceding F layer's, bit for bit (all rows);
  * attention: where the kernel chose exactly the oracle's top-k set (all but
    allowed near-tie swaps), the output is within the attention tolerance of
    the oracle's, computed from the oracle's own indices.
For decode the oracle reads only its own selected KV rows, which are gathered
on the device by torch indexing with the oracle's indices (never with the
kernel's) to keep host memory bounded.
"""
import numpy as np
import pytest
import torch

import oracle
import cross_layer_top_full_b200 as ic
from cross_layer_top_full_b200 import synth
from parity_util import check_attention, check_topk_band, host64

pytestmark = pytest.mark.gpu

DT = {"f32": ic.F32, "bf16": ic.BF16, "e4m3": ic.FP8_E4M3}


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ic.lib()
    return torch.device("cuda:0")


def run_stack(wl, pattern, inputs, rows, dev):
    """ic_layer_stack_forward over `inputs`; returns (outs, per-layer idx, n indexer)."""
    B, L, q_start, T = rows
    r = ic.Rows(B, L, q_start, T)
    sh = ic.StackShape(r, wl.H_I, wl.d_I, DT[wl.idx_dtype], wl.k, wl.Hq, wl.d_qk, wl.d_v,
                       DT[wl.attn_dtype], wl.d_qk, wl.d_qk if wl.latent else wl.d_v, wl.scale)
    ws = torch.empty(ic.workspace_size(sh), dtype=torch.uint8, device=dev)
    ic.workspace_init(ws)
    idx_buf = torch.empty(B, L, wl.k, dtype=torch.int32, device=dev)
    outs = [torch.empty(B, L, wl.Hq, wl.d_v, dtype=torch.bfloat16, device=dev) for _ in pattern]
    copies = [torch.empty_like(idx_buf) for _ in pattern]
    layers = [dict(q_idx=x.get("q_I"), q_scale=x.get("q_scale"), w=x.get("w"), k_idx=x.get("k_I"),
                   k_scale=x.get("k_scale"), q=x["q"], kmat=x["kv"], vmat=x["kv"], out=o)
              for x, o in zip(inputs, outs)]
    n0 = ic.kernel_launches(1)
    ic.layer_stack_forward(pattern, layers, sh, idx_buf, ws, idx_out=copies)
    torch.cuda.synchronize()
    assert ic.read_status(ws) == 0
    return outs, copies, ic.kernel_launches(1) - n0


def oracle_scores(wl, inp, q_start, rows, seqs):
    """float64 indexer scores [len(seqs), len(rows), T] of query rows `rows`
    (relative to the call's q_start) of sequences `seqs`, each row computed
    on its own from the device inputs; -inf beyond the row's causal range."""
    fp8 = wl.idx_dtype == "e4m3"
    T = inp["k_I"].shape[1]
    out = np.full((len(seqs), len(rows), T), -np.inf)
    for bi, b in enumerate(seqs):
        kI = host64(inp["k_I"][b:b + 1])
        ks = host64(inp["k_scale"][b:b + 1]) if fp8 else None
        for ri, i in enumerate(rows):
            qs = host64(inp["q_scale"][b:b + 1, i:i + 1]) if fp8 else None
            sc = oracle.indexer_scores(host64(inp["q_I"][b:b + 1, i:i + 1]),
                                       host64(inp["w"][b:b + 1, i:i + 1]), kI, q_start + i, qs, ks,
                                       fp8=fp8)
            out[bi, ri] = sc[0, 0]
    return out


def oracle_attention_rows(wl, inp, ref_idx, b, i):
    """Oracle output of row (b, i) over the oracle's indices ref_idx [k]."""
    J = torch.as_tensor(ref_idx[ref_idx >= 0], dtype=torch.long, device=inp["kv"].device)
    kvJ = host64(inp["kv"][b].index_select(0, J))          # only the selected rows
    q = host64(inp["q"][b, i])[None, None]
    pos = np.arange(kvJ.shape[0], dtype=np.int32)[None, None]
    return oracle.sparse_attention(q, kvJ[None], kvJ[None, :, : wl.d_v], pos, wl.scale)[0, 0]


# --------------------------------------------------------------------------- prefill 8k
def test_prefill_8k_bf16_full_size(dev):
    wl = synth.WORKLOADS["prefill_8k_bf16"]
    inputs = [synth.layer_inputs(wl, l, dev) for l in range(wl.n_layers)]
    outs, copies, n_ix = run_stack(wl, wl.pattern, inputs, (wl.B, wl.L, 0, wl.T), dev)
    assert n_ix == wl.pattern.count("F")
    rng = np.random.default_rng(1)
    rows = sorted(set([0, 1, wl.k - 1, wl.k, wl.k + 1, wl.L - 1] +
                      rng.choice(wl.L, 18, replace=False).tolist()))
    n_same = 0
    last_f, ref_idx = None, None
    for l, kind in enumerate(wl.pattern):
        gidx = host64(copies[l])
        if kind == "F":
            last_f = l
            sc = oracle_scores(wl, inputs[l], 0, rows, [0])
            check_topk_band(gidx[:, rows], sc, 0, wl.k, rows=rows)
            ref_idx = oracle.topk_indices(sc, 0, wl.k, rows=rows)
        else:
            assert np.array_equal(gidx, host64(copies[last_f])), "S layer %d" % l
        got = host64(outs[l][0, rows])
        for r_i, i in enumerate(rows):
            if not np.array_equal(gidx[0, i], ref_idx[0, r_i]):
                continue                                    # allowed near-tie swap
            n_same += 1
            ref = oracle_attention_rows(wl, inputs[l], ref_idx[0, r_i], 0, i)
            check_attention(got[r_i], ref, "prefill_8k layer %d row %d" % (l, i))
    assert n_same >= 0.9 * len(rows) * wl.n_layers


# --------------------------------------------------------------------------- decode 32 x 32k
def test_decode_b32_t32k_bf16_full_size(dev):
    wl = synth.WORKLOADS["decode_b32_t32k_bf16"]
    inputs = [synth.layer_inputs(wl, l, dev) for l in range(wl.n_layers)]
    outs, copies, n_ix = run_stack(wl, wl.pattern, inputs, (wl.B, 1, wl.q_start, wl.T), dev)
    assert n_ix == wl.pattern.count("F")
    check_layers = {0, 1, 4, 7}
    n_same = 0
    last_f, ref_idx = None, None
    for l, kind in enumerate(wl.pattern):
        gidx = host64(copies[l])
        if kind == "F":
            last_f = l
            sc = oracle_scores(wl, inputs[l], wl.q_start, [0], range(wl.B))
            check_topk_band(gidx, sc, wl.q_start, wl.k)
            ref_idx = oracle.topk_indices(sc, wl.q_start, wl.k)
        else:
            assert np.array_equal(gidx, host64(copies[last_f]))
        if l not in check_layers:
            continue
        got = host64(outs[l])
        for b in range(wl.B):
            if not np.array_equal(gidx[b, 0], ref_idx[b, 0]):
                continue
            n_same += 1
            ref = oracle_attention_rows(wl, inputs[l], ref_idx[b, 0], b, 0)
            check_attention(got[b, 0], ref, "decode_b32 layer %d seq %d" % (l, b))
    assert n_same >= 0.9 * wl.B * len(check_layers)


# --------------------------------------------------------------------------- decode fp8 200k
def test_decode_b8_t200k_fp8_first_8_layers(dev):
    """Full B=8, T=200000 with the FP8 indexer; the first 8 of the 48 layers
    (FSSSFSSS) to bound device memory in a test (the benchmark runs all 48)."""
    wl = synth.WORKLOADS["decode_b8_t200k_fp8"]
    pattern = wl.pattern[:8]
    inputs = [synth.layer_inputs(wl, l, dev) for l in range(len(pattern))]
    outs, copies, n_ix = run_stack(wl, pattern, inputs, (wl.B, 1, wl.q_start, wl.T), dev)
    assert n_ix == 2
    n_same = 0
    last_f, ref_idx = None, None
    for l, kind in enumerate(pattern):
        gidx = host64(copies[l])
        if kind == "F":
            last_f = l
            sc = oracle_scores(wl, inputs[l], wl.q_start, [0], range(wl.B))
            check_topk_band(gidx, sc, wl.q_start, wl.k)
            ref_idx = oracle.topk_indices(sc, wl.q_start, wl.k)
        else:
            assert np.array_equal(gidx, host64(copies[last_f]))
        if l not in (0, 1, 4, 7):
            continue
        got = host64(outs[l])
        for b in range(wl.B):
            if not np.array_equal(gidx[b, 0], ref_idx[b, 0]):
                continue
            n_same += 1
            ref = oracle_attention_rows(wl, inputs[l], ref_idx[b, 0], b, 0)
            check_attention(got[b, 0], ref, "decode_fp8 layer %d seq %d" % (l, b))
    assert n_same >= 0.75 * wl.B * 4


# --------------------------------------------------------------------------- chunked 64k
def test_chunked_prefill_64k_bf16_sampled_chunks(dev):
    """All 12 layers, chunks 0, 7 and 15 of the 16 (keys up to 65536), each
    run as in the chunked prefill: q_start = 4096 c, T = 4096 (c + 1)."""
    wl = synth.WORKLOADS["chunked_prefill_64k_bf16"]
    C = wl.chunk
    rng = np.random.default_rng(3)
    for c in (0, 7, 15):
        inputs = [synth.layer_inputs(wl, l, dev, chunk=c) for l in range(wl.n_layers)]
        q_start, T = c * C, (c + 1) * C
        outs, copies, n_ix = run_stack(wl, wl.pattern, inputs, (1, C, q_start, T), dev)
        assert n_ix == wl.pattern.count("F")
        rows = sorted(set([0, C - 1] + rng.choice(C, 3, replace=False).tolist()))
        attn_rows = rows[:3]
        last_f, ref_idx = None, None
        for l, kind in enumerate(wl.pattern):
            gidx = host64(copies[l])
            if kind == "F":
                last_f = l
                sc = oracle_scores(wl, inputs[l], q_start, rows, [0])
                check_topk_band(gidx[:, rows], sc, q_start, wl.k, rows=rows)
                ref_idx = oracle.topk_indices(sc, q_start, wl.k, rows=rows)
            else:
                assert np.array_equal(gidx, host64(copies[last_f]))
            got = host64(outs[l][0, attn_rows])
            for r_i, i in enumerate(attn_rows):
                if not np.array_equal(gidx[0, i], ref_idx[0, r_i]):
                    continue
                ref = oracle_attention_rows(wl, inputs[l], ref_idx[0, r_i], 0, i)
                check_attention(got[r_i], ref, "chunk %d layer %d row %d" % (c, l, i))
        del inputs, outs, copies
        torch.cuda.empty_cache()
