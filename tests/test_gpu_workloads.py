"""Full-size parity of the four large workloads, in the launch configuration
the benchmark times (the whole F/S stack through ic_layer_stack_forward).

The oracle cannot redo a full workload in float64 within a test, so each
check covers outputs the oracle computes one by one (tests/stack_check.py):
  * prefill 8K: the indices of all 8192 rows; attention on 512 seeded rows
    (always rows 0, 1, k-1, k, k+1 and L-1) of all 4 layers;
  * decode 32 x 32K: every sequence, indices and attention of all 8 layers;
  * decode 8 x 200K (FP8 indexer): every sequence, all 48 layers;
  * chunked prefill 64K: all 16 chunks, 16 rows each (always the chunk's
    first and last row), indices and attention of all 12 layers.
  * prefill 8K with the FP8 indexer: indices of 512 seeded rows, attention
    on 128 of them, all 4 layers.
The decode stack is also replayed from a captured CUDA graph, as the
benchmark times it, and compared bit for bit with direct launches.
Per checked row: an F layer's indices obey the top-k band rule against the
oracle's float64 scores; an S layer's indices are the F layer's bit for bit
(all rows); attention of EVERY sampled row is within the attention
tolerance of the oracle's float64 attention over the index set the kernel
used (band-valid, so a valid top-k; where it differs from the oracle's own
exact top-k by allowed near-tie swaps, the comparison still runs).  The
number of rows whose set equals the oracle's exact top-k is printed, not
asserted: it measures near ties, not correctness.
"""
import pytest
import torch

import cross_layer_top_full_b200 as ic
from cross_layer_top_full_b200 import synth
from stack_check import check_stack, sample_rows

pytestmark = pytest.mark.gpu

DT = {"f32": ic.F32, "bf16": ic.BF16, "e4m3": ic.FP8_E4M3}


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ic.lib()
    return torch.device("cuda:0")


def report(what, n_cmp, n_same):
    """Every sampled attention row was compared; say how many of them used
    exactly the oracle's top-k set (the rest differ by allowed near ties)."""
    assert n_cmp > 0
    print("%s: %d attention rows compared, %d with the oracle's exact index set"
          % (what, n_cmp, n_same))


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


# --------------------------------------------------------------------------- prefill 8k
def test_prefill_8k_bf16_full_size(dev):
    wl = synth.WORKLOADS["prefill_8k_bf16"]
    inputs = [synth.layer_inputs(wl, l, dev) for l in range(wl.n_layers)]
    outs, copies, n_ix = run_stack(wl, wl.pattern, inputs, (wl.B, wl.L, 0, wl.T), dev)
    assert n_ix == wl.pattern.count("F")
    attn_rows = sample_rows(wl.L, 512, seed=1,
                            always=(0, 1, wl.k - 1, wl.k, wl.k + 1, wl.L - 1))
    n_cmp, n_same = check_stack(wl, wl.pattern, inputs, copies, outs, 0, [0], range(wl.L),
                                attn_rows, range(wl.n_layers), "prefill_8k")
    report("prefill_8k", n_cmp, n_same)
    del inputs, outs, copies
    torch.cuda.empty_cache()


# --------------------------------------------------------------------------- decode 32 x 32k
def test_decode_b32_t32k_bf16_full_size(dev):
    wl = synth.WORKLOADS["decode_b32_t32k_bf16"]
    inputs = [synth.layer_inputs(wl, l, dev) for l in range(wl.n_layers)]
    outs, copies, n_ix = run_stack(wl, wl.pattern, inputs, (wl.B, 1, wl.q_start, wl.T), dev)
    assert n_ix == wl.pattern.count("F")
    n_cmp, n_same = check_stack(wl, wl.pattern, inputs, copies, outs, wl.q_start, range(wl.B),
                                [0], [0], range(wl.n_layers), "decode_b32")
    report("decode_b32", n_cmp, n_same)
    del inputs, outs, copies
    torch.cuda.empty_cache()


def test_decode_graph_replay_matches_plain_launches(dev):
    """The decode stack as the benchmark runs it: captured once as a CUDA
    graph (its kernels joined by programmatic launch edges, the few-row
    calls' early launch) and replayed, against the same stack launched
    directly: the indices and every layer's output are identical bit for
    bit, replay after replay, and the status word stays clean."""
    wl = synth.WORKLOADS["decode_b32_t32k_bf16"]
    inputs = [synth.layer_inputs(wl, l, dev) for l in range(wl.n_layers)]
    r = ic.Rows(wl.B, 1, wl.q_start, wl.T)
    sh = ic.StackShape(r, wl.H_I, wl.d_I, DT[wl.idx_dtype], wl.k, wl.Hq, wl.d_qk, wl.d_v,
                       DT[wl.attn_dtype], wl.d_qk, wl.d_qk if wl.latent else wl.d_v, wl.scale)
    ws = torch.empty(ic.workspace_size(sh), dtype=torch.uint8, device=dev)
    ic.workspace_init(ws)
    idx_buf = torch.empty(wl.B, 1, wl.k, dtype=torch.int32, device=dev)
    outs = [torch.empty(wl.B, 1, wl.Hq, wl.d_v, dtype=torch.bfloat16, device=dev)
            for _ in wl.pattern]
    layers = [dict(q_idx=x.get("q_I"), q_scale=x.get("q_scale"), w=x.get("w"), k_idx=x.get("k_I"),
                   k_scale=x.get("k_scale"), q=x["q"], kmat=x["kv"], vmat=x["kv"], out=o)
              for x, o in zip(inputs, outs)]

    def step(stream=None):
        ic.layer_stack_forward(wl.pattern, layers, sh, idx_buf, ws, stream=stream)

    step()
    torch.cuda.synchronize()
    assert ic.read_status(ws) == 0
    ref_out = [o.clone() for o in outs]
    ref_idx = idx_buf.clone()

    g = torch.cuda.CUDAGraph()
    s_cap = torch.cuda.Stream()
    s_cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s_cap):
        step(s_cap)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s_cap):
            step(s_cap)
    torch.cuda.current_stream().wait_stream(s_cap)
    for rep in range(3):
        for o in outs:
            o.zero_()
        idx_buf.fill_(-7)
        g.replay()
        torch.cuda.synchronize()
        assert ic.read_status(ws) == 0
        assert torch.equal(idx_buf, ref_idx), "replay %d: indices differ" % rep
        for l, (o, ro) in enumerate(zip(outs, ref_out)):
            assert torch.equal(o, ro), "replay %d: layer %d output differs" % (rep, l)
    del g, inputs, outs, ref_out
    torch.cuda.empty_cache()


# --------------------------------------------------------------------------- decode fp8 200k
def test_decode_b8_t200k_fp8_full_size(dev):
    """B = 8, T = 200000, all 48 layers ((FSSS) x 12) with the FP8 indexer:
    about 98 GB of layer inputs on the device."""
    wl = synth.WORKLOADS["decode_b8_t200k_fp8"]
    inputs = [synth.layer_inputs(wl, l, dev) for l in range(wl.n_layers)]
    outs, copies, n_ix = run_stack(wl, wl.pattern, inputs, (wl.B, 1, wl.q_start, wl.T), dev)
    assert n_ix == wl.pattern.count("F") == 12
    n_cmp, n_same = check_stack(wl, wl.pattern, inputs, copies, outs, wl.q_start, range(wl.B),
                                [0], [0], range(wl.n_layers), "decode_fp8")
    report("decode_fp8", n_cmp, n_same)
    del inputs, outs, copies
    torch.cuda.empty_cache()


# --------------------------------------------------------------------------- chunked 64k
def test_chunked_prefill_64k_bf16_every_chunk(dev):
    """All 12 layers and all 16 chunks, each run as in the chunked prefill:
    q_start = 4096 c, T = 4096 (c + 1)."""
    wl = synth.WORKLOADS["chunked_prefill_64k_bf16"]
    C = wl.chunk
    n_cmp = n_same = 0
    for c in range(wl.L // C):
        inputs = [synth.layer_inputs(wl, l, dev, chunk=c) for l in range(wl.n_layers)]
        q_start, T = c * C, (c + 1) * C
        outs, copies, n_ix = run_stack(wl, wl.pattern, inputs, (1, C, q_start, T), dev)
        assert n_ix == wl.pattern.count("F")
        rows = sample_rows(C, 14, seed=3 + c, always=(0, C - 1))
        cmp_c, same_c = check_stack(wl, wl.pattern, inputs, copies, outs, q_start, [0], rows,
                                    rows, range(wl.n_layers), "chunk %d" % c)
        n_cmp += cmp_c
        n_same += same_c
        del inputs, outs, copies
        torch.cuda.empty_cache()
    report("chunked_64k", n_cmp, n_same)


# --------------------------------------------------------------------------- prefill 8k, FP8 indexer
def test_prefill_8k_fp8_indexer_full_size(dev):
    """The 8K prefill with the indexer operands in E4M3 (one scale per token):
    the prefill-shaped FP8 tensor-core indexer at full size.  Indices of 512
    seeded rows (always 0, 1, k-1, k, k+1, L-1); attention on 128 of them,
    all 4 layers."""
    wl = synth.WORKLOADS["prefill_8k_fp8"]
    inputs = [synth.layer_inputs(wl, l, dev) for l in range(wl.n_layers)]
    outs, copies, n_ix = run_stack(wl, wl.pattern, inputs, (wl.B, wl.L, 0, wl.T), dev)
    assert n_ix == wl.pattern.count("F")
    always = (0, 1, wl.k - 1, wl.k, wl.k + 1, wl.L - 1)
    idx_rows = sample_rows(wl.L, 512, seed=7, always=always)
    attn_rows = sample_rows(len(idx_rows), 122, seed=8)
    attn_rows = sorted(set([idx_rows[j] for j in attn_rows]) | set(always))
    n_cmp, n_same = check_stack(wl, wl.pattern, inputs, copies, outs, 0, [0], idx_rows,
                                attn_rows, range(wl.n_layers), "prefill_8k_fp8")
    report("prefill_8k_fp8", n_cmp, n_same)
    del inputs, outs, copies
    torch.cuda.empty_cache()

