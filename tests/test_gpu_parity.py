"""GPU parity of each call of the C ABI against the float64 oracle, at sizes
the oracle finishes in seconds that still span several tiles and ragged
tails.  Full-size workloads are in test_gpu_workloads.py."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import cross_layer_top_full_b200 as ic
from cross_layer_top_full_b200 import synth
from parity_util import (abs_term_sum, check_attention, check_scores, check_topk_band, host64)

pytestmark = pytest.mark.gpu

DT = {"f32": ic.F32, "bf16": ic.BF16, "e4m3": ic.FP8_E4M3}


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ic.lib()
    return torch.device("cuda:0")


def _ws(nbytes, dev):
    ws = torch.empty(max(nbytes, ic.STATUS_BYTES), dtype=torch.uint8, device=dev)
    ic.workspace_init(ws)
    return ws


def _gpu_scores(inp, rows, dtype, dev):
    B, Lq, q_start, T = rows
    ld = (T + 3) // 4 * 4
    scores = torch.full((B, Lq, ld), float("nan"), device=dev)
    H_I, d_I = inp["q_I"].shape[-2], inp["q_I"].shape[-1]
    ws = _ws(ic.indexer_workspace_size(rows, H_I, d_I, DT[dtype]), dev)
    tc0 = ic.kernel_launches(5)
    ic.indexer_scores(inp["q_I"], inp["w"], inp["k_I"], rows, scores, ws,
                      q_scale=inp.get("q_scale"), k_scale=inp.get("k_scale"), dtype=DT[dtype])
    torch.cuda.synchronize()
    tensor_core = dtype != "f32" and d_I == 128 and H_I in (16, 32, 64, 128)
    assert ic.kernel_launches(5) - tc0 == (1 if tensor_core else 0)
    assert ic.read_status(ws) == 0
    return scores


def _oracle_scores(inp, q_start, dtype, rows=None):
    fp8 = dtype == "e4m3"
    return oracle.indexer_scores(host64(inp["q_I"]), host64(inp["w"]), host64(inp["k_I"]), q_start,
                                 host64(inp["q_scale"]) if fp8 else None,
                                 host64(inp["k_scale"]) if fp8 else None, fp8=fp8, rows=rows)


# ------------------------------------------------------------------------- indexer
@pytest.mark.parametrize("dtype", ["f32", "bf16", "e4m3"])
@pytest.mark.parametrize("H_I,d_I", [(64, 128), (4, 32), (16, 128)])
def test_indexer_exact_mode_is_bit_exact(dev, dtype, H_I, d_I):
    rows = (2, 300, 37, 400)       # ragged: 337 causal keys max, tails in both axes
    B, Lq, q_start, T = rows
    inp = synth.exact_indexer_inputs(B, Lq, T, H_I, d_I, dtype, dev, seed=H_I + d_I)
    got = host64(_gpu_scores(inp, rows, dtype, dev))
    ref = _oracle_scores(inp, q_start, dtype)
    for b in range(B):
        for i in range(Lq):
            t = q_start + i
            assert np.array_equal(got[b, i, : t + 1], ref[b, i, : t + 1]), (dtype, b, i)


@pytest.mark.parametrize("bits", [16, 24])
@pytest.mark.parametrize("Lq", [1, 64])          # decode (one token per MMA) and prefill shapes
def test_indexer_fp8_accumulation_is_float32_wide(dev, Lq, bits):
    """Width of the tensor core's E4M3 accumulation (the float32 reading).
    All codes are positive integers, so every partial sum of a dot product is
    an integer and float32 holds it exactly below 2^24; the low bits come
    from small terms added to a large running sum, which an accumulator
    narrower than `bits` significant bits would round away:
      bits=16: q_I is 224/240/256 on 96 dims and 1/3 on 32, k_I is 1..3; each
               dot is an integer of 2^15..2^16, half of them odd, and w = +-1
               on all 64 heads keeps the head sum an integer below 2^24;
      bits=24: q_I and k_I are 384/416/448 on 64 dims, q_I is 1/3 and k_I
               1..3 on the rest; each dot is about 2^23.4, half of them odd
               (24 significant bits); one effective head
               (w = 1 on head 0, 0 elsewhere) makes the score that dot.
    The scores must equal the oracle's bit for bit; a failure reports the
    number of significant bits the accumulation kept."""
    B, T, H_I, d_I = 1, 512, 64, 128
    q_start = T - Lq
    g = torch.Generator(device="cpu").manual_seed(40 + Lq + bits)
    if bits == 16:
        nb, bigv = 96, [224.0, 240.0, 256.0]
        kbig, ksmall = [1.0, 2.0, 3.0], [1.0, 2.0, 3.0]
    else:
        nb, bigv = 64, [384.0, 416.0, 448.0]
        kbig, ksmall = [384.0, 416.0, 448.0], [1.0, 2.0, 3.0]
    big = torch.tensor(bigv)[torch.randint(0, len(bigv), (B, Lq, H_I, nb), generator=g)]
    small = torch.tensor([1.0, 3.0])[torch.randint(0, 2, (B, Lq, H_I, d_I - nb), generator=g)]
    qv = torch.cat([big, small], dim=-1)
    kv = torch.cat([torch.tensor(kbig)[torch.randint(0, len(kbig), (B, T, nb), generator=g)],
                    torch.tensor(ksmall)[torch.randint(0, len(ksmall), (B, T, d_I - nb),
                                                       generator=g)]], dim=-1)
    if bits == 16:
        w = torch.randint(0, 2, (B, Lq, H_I), generator=g).float() * 2 - 1
    else:
        w = torch.zeros(B, Lq, H_I)
        w[..., 0] = 1.0
    inp = {
        "q_I": qv.to(torch.float8_e4m3fn).view(torch.uint8).contiguous().to(dev),
        "k_I": kv.to(torch.float8_e4m3fn).view(torch.uint8).contiguous().to(dev),
        "w": w.contiguous().to(dev),
        "q_scale": torch.pow(2.0, torch.randint(-1, 2, (B, Lq), generator=g).float()).to(dev),
        "k_scale": torch.pow(2.0, torch.randint(-1, 2, (B, T), generator=g).float()).to(dev),
    }
    # the stored codes are exactly these values
    assert torch.equal(inp["q_I"].cpu().view(torch.float8_e4m3fn).float(), qv)
    assert torch.equal(inp["k_I"].cpu().view(torch.float8_e4m3fn).float(), kv)
    dots = qv.double().numpy() @ kv.double().numpy()[0].T          # [B, Lq, H, T]
    assert dots.max() < 2 ** 24 and dots.min() > 2 ** (bits - 3)
    assert 0.25 < (dots % 2 == 1).mean() < 0.75          # the lowest bit matters
    rows = (B, Lq, q_start, T)
    got = host64(_gpu_scores(inp, rows, "e4m3", dev))[..., :T]
    ref = _oracle_scores(inp, q_start, "e4m3")
    causal = np.arange(T)[None, None, :] <= (q_start + np.arange(Lq))[None, :, None]
    bad = causal & (got != ref)
    if bad.any():
        err = np.abs(got - ref)[causal].max()
        raise AssertionError("FP8 scores differ from the exact float32 sums in %d of %d entries; "
                             "max |error| %g on scores up to %g (about %.1f bits kept)"
                             % (bad.sum(), causal.sum(), err, np.abs(ref[causal]).max(),
                                np.log2(np.abs(ref[causal]).max() / err)))


@pytest.mark.parametrize("dtype,H_I", [("f32", 1), ("bf16", 1), ("bf16", 16), ("e4m3", 16)])
def test_indexer_one_effective_head_is_relu_of_the_dot_product(dev, dtype, H_I):
    """Closed form: with w = 1 on head 0 and 0 on every other head the score
    is max(0, q_I[head 0] . k_I) (times the two FP8 scales), written here
    with numpy directly.  H_I = 16 runs the tensor-core kernel, H_I = 1 the
    CUDA-core one; integer operands make the expected values exact."""
    rows = (1, 150, 70, 220)
    B, Lq, q_start, T = rows
    inp = synth.exact_indexer_inputs(B, Lq, T, H_I, 128, dtype, dev, seed=31 + H_I)
    w = torch.zeros(B, Lq, H_I, device=dev)
    w[..., 0] = 1.0
    inp["w"] = w
    got = host64(_gpu_scores(inp, rows, dtype, dev))
    if dtype == "e4m3":
        q0 = oracle.e4m3_decode(host64(inp["q_I"]))[0, :, 0]
        k = oracle.e4m3_decode(host64(inp["k_I"]))[0]
        sq, sk = host64(inp["q_scale"])[0], host64(inp["k_scale"])[0]
    else:
        q0, k = host64(inp["q_I"])[0, :, 0], host64(inp["k_I"])[0]
        sq, sk = np.ones(Lq), np.ones(T)
    expect = np.maximum(q0 @ k.T, 0.0) * sq[:, None] * sk[None, :]
    for i in range(Lq):
        t = q_start + i
        assert np.array_equal(got[0, i, : t + 1], expect[i, : t + 1]), (dtype, H_I, i)


@pytest.mark.parametrize("dtype", ["f32", "bf16", "e4m3"])
def test_indexer_general_inputs_within_tolerance(dev, dtype):
    rows = (3, 130, 5, 140)
    B, Lq, q_start, T = rows
    wl = synth.WORKLOADS["decode_b8_t200k_fp8" if dtype == "e4m3" else "prefill_8k_bf16"]
    g = torch.Generator(device=dev).manual_seed(11)
    qI = torch.randn(B, Lq, 64, 128, device=dev, generator=g) / 11.3
    kI = torch.randn(B, T, 128, device=dev, generator=g) / 11.3
    w = torch.randn(B, Lq, 64, device=dev, generator=g) / 8
    if dtype == "e4m3":
        q8, qs = synth.fp8_per_token(qI, 2)
        k8, ks = synth.fp8_per_token(kI, 2)
        inp = dict(q_I=q8, k_I=k8, q_scale=qs, k_scale=ks, w=w)
        vq = oracle.e4m3_decode(host64(q8)) * host64(qs)[..., None, None]
        vk = oracle.e4m3_decode(host64(k8)) * host64(ks)[..., None]
    else:
        dt = torch.float32 if dtype == "f32" else torch.bfloat16
        inp = dict(q_I=qI.to(dt), k_I=kI.to(dt), w=w)
        vq, vk = host64(inp["q_I"]), host64(inp["k_I"])
    got = host64(_gpu_scores(inp, rows, dtype, dev))
    ref = _oracle_scores(inp, q_start, dtype)
    absum = abs_term_sum(vq, host64(w), vk)
    check_scores(got, ref, absum, q_start, rel=1e-3 if dtype == "e4m3" else 1e-4)
    del wl


# ------------------------------------------------------------------------- top-k
@pytest.mark.parametrize("ties", [False, True])
@pytest.mark.parametrize("rows,k", [((2, 70, 0, 70), 16),        # short rows, k < and >= t+1
                                    ((1, 40, 3000, 3040), 2048),  # prefill-like long rows
                                    ((4, 1, 49999, 50000), 2048), # decode rows beyond smem cache
                                    ((3, 1, 32767, 32768), 2048), # decode rows, cached
                                    ((2, 3, 40000, 40003), 2048), # few long rows of unequal length
                                    ((1, 2, 199998, 200000), 2048),
                                    # one cluster per row: 8, 4, 2 and 1 CTAs per row
                                    ((32, 1, 32767, 32768), 2048),
                                    ((64, 1, 9999, 10000), 2048),
                                    ((100, 1, 5999, 6000), 2048),
                                    # cluster rows of which two keep every candidate (n <= k)
                                    ((2, 4, 4998, 5002), 5000),
                                    # rows too long for a cluster's shared memory: three launches
                                    ((2, 1, 399999, 400000), 2048),
                                    # row caches of 46.9 KiB and exactly 48 KiB of shared memory
                                    # (plus the static select state: past the default limit)
                                    ((1, 300, 11700, 12000), 2048),
                                    ((1, 300, 11988, 12288), 2048),
                                    ((1, 5, 10, 15), 1)])
def test_topk_is_bit_exact_on_identical_scores(dev, rows, k, ties):
    B, Lq, q_start, T = rows
    scores = synth.random_scores(B, Lq, T, dev, seed=k + T, ties=ties)
    idx = torch.full((B, Lq, k), -7, dtype=torch.int32, device=dev)
    ws = _ws(ic.topk_workspace_size(rows, k), dev)
    ic.topk(scores, rows, k, idx, ws)
    torch.cuda.synchronize()
    ref = oracle.topk_indices(host64(scores), q_start, k)
    assert np.array_equal(host64(idx), ref)


@pytest.mark.parametrize("rows", [(8, 1, 199999, 200000), (32, 1, 32767, 32768)])
def test_decode_topk_is_one_launch(dev, rows):
    """Decode rows (the two decode workloads' shapes) take the one-launch
    cluster path, bit-exact against the oracle."""
    B, Lq, q_start, T = rows
    k = 2048
    scores = synth.random_scores(B, Lq, T, dev, seed=B)
    idx = torch.full((B, Lq, k), -7, dtype=torch.int32, device=dev)
    ws = _ws(ic.topk_workspace_size(rows, k), dev)
    n0 = ic.kernel_launches(2)
    ic.topk(scores, rows, k, idx, ws)
    torch.cuda.synchronize()
    assert ic.kernel_launches(2) - n0 == 1
    assert np.array_equal(host64(idx), oracle.topk_indices(host64(scores), q_start, k))


def test_topk_long_rows_of_equal_scores(dev):
    """Every score equal (a mix of +0.0 and -0.0): the candidate bin of the
    multi-CTA path overflows and the row is resolved in one CTA; the answer is
    the k smallest positions."""
    rows = (2, 1, 99999, 100000)
    k = 2048
    g = torch.Generator(device=dev).manual_seed(4)
    scores = torch.zeros(2, 1, 100000, device=dev)
    scores[torch.rand(2, 1, 100000, generator=g, device=dev) < 0.5] = -0.0
    idx = torch.full((2, 1, k), -7, dtype=torch.int32, device=dev)
    ws = _ws(ic.topk_workspace_size(rows, k), dev)
    ic.topk(scores, rows, k, idx, ws)
    torch.cuda.synchronize()
    assert np.array_equal(host64(idx)[:, 0], np.tile(np.arange(k), (2, 1)))
    ref = oracle.topk_indices(host64(scores), 99999, k)
    assert np.array_equal(host64(idx), ref)


# ------------------------------------------------------------------------- fused selection
@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
@pytest.mark.parametrize("rows,fused", [((8, 1, 199999, 200000), None),   # the FP8 decode workload's shape
                                        ((32, 1, 32767, 32768), True),    # the bf16 decode workload's shape
                                        ((16, 1, 49999, 50000), None),    # larger clusters
                                        ((64, 1, 9999, 10000), None),     # clusters of 2 CTAs
                                        ((3, 2, 9998, 10000), None),      # two query rows per sequence
                                        ((1, 1, 5000, 5001), None)])      # one row
def test_fused_selection_equals_indexer_then_topk(dev, dtype, rows, fused):
    """ic_indexer_topk on decode rows gives exactly the indices of
    ic_indexer_scores followed by ic_topk: the same arithmetic, bit for bit.
    Where its clusters cover most of the SMs it runs ONE kernel (the
    indexer's scores kept in shared memory, selected there); with few rows
    it runs the stand-alone indexer and the one-launch top-k.  The indices
    also obey the band rule against the oracle's float64 scores (first
    sequence)."""
    B, Lq, q_start, T = rows
    k = 2048
    wl = synth.Workload("sel", B, Lq, T, q_start, 64, 128, k, 128, 576, 512, dtype, "bf16", True,
                        "F", 51, 1 / 8, 128 ** -0.5, 128 ** -0.5, 1.0, 1.0, heavy=16,
                        heavy_gain=4.0)
    inp = synth.layer_inputs(wl, 0, dev, attention=False)
    ld = (T + 3) // 4 * 4
    scores = torch.empty(B, Lq, ld, device=dev)
    ws = _ws(ic.indexer_topk_workspace_size(rows, 64, 128, DT[dtype], k), dev)
    ic.indexer_scores(inp["q_I"], inp["w"], inp["k_I"], rows, scores, ws, q_scale=inp.get("q_scale"),
                      k_scale=inp.get("k_scale"), dtype=DT[dtype])
    ref = torch.empty(B, Lq, k, dtype=torch.int32, device=dev)
    ic.topk(scores, rows, k, ref, ws)
    got = torch.full((B, Lq, k), -7, dtype=torch.int32, device=dev)
    n_sel, n_ix = ic.kernel_launches(7), ic.kernel_launches(1)
    ic.indexer_topk(inp["q_I"], inp["w"], inp["k_I"], rows, k, got, ws, q_scale=inp.get("q_scale"),
                    k_scale=inp.get("k_scale"), dtype=DT[dtype])
    torch.cuda.synchronize()
    assert ic.read_status(ws) == 0
    ran_fused = ic.kernel_launches(7) - n_sel == 1
    assert ic.kernel_launches(1) - n_ix == 1          # one indexer pass either way
    if fused is not None:
        assert ran_fused == fused
    assert torch.equal(got, ref)
    sub = {key: v[:1] for key, v in inp.items()}
    sc = _oracle_scores(sub, q_start, dtype)
    check_topk_band(host64(got[:1]), sc, q_start, k)


# ------------------------------------------------------------------------- attention
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("Hq,d_qk,d_v,latent", [(8, 64, 64, False), (128, 576, 512, True),
                                                (3, 40, 24, False),
                                                # CUDA-core path: 16 staged K/V rows of
                                                # 256 + 512 floats are exactly 48 KiB of dynamic
                                                # shared memory, past the default limit with the
                                                # kernel's static part
                                                (4, 256, 512, False)])
def test_sparse_attention_within_tolerance(dev, dtype, Hq, d_qk, d_v, latent):
    rows = (2, 37, 90, 127)        # q_start > 0, ragged
    B, Lq, q_start, T = rows
    k = 100
    torch_dt = torch.float32 if dtype == "f32" else torch.bfloat16
    g = torch.Generator(device=dev).manual_seed(Hq + d_qk)
    q = torch.randn(B, Lq, Hq, d_qk, device=dev, generator=g).to(torch_dt)
    if latent:
        kv = torch.randn(B, T, d_qk, device=dev, generator=g).to(torch_dt)
        kmat = vmat = kv
        ks = vs = d_qk
    else:
        kmat = torch.randn(B, T, d_qk, device=dev, generator=g).to(torch_dt)
        vmat = torch.randn(B, T, d_v, device=dev, generator=g).to(torch_dt)
        ks, vs = d_qk, d_v
    idx = synth.random_index_sets(B, Lq, q_start, k, dev, seed=3)
    idx[0, 0, 40:] = -1            # a row with fewer valid keys than k
    idx[1, 2, :] = -1              # a row with no valid key: zero output
    out = torch.empty(B, Lq, Hq, d_v, device=dev, dtype=torch_dt)
    scale = d_qk ** -0.5
    ws = _ws(ic.sparse_attn_workspace_size(rows, k, Hq, d_qk, d_v, DT[dtype]), dev)
    ic.sparse_attn(q, kmat, ks, vmat, vs, idx, rows, d_v, scale, out, ws)
    torch.cuda.synchronize()
    assert ic.read_status(ws) == 0
    K = host64(kmat)
    V = host64(vmat)[..., :d_v] if latent else host64(vmat)
    ref = oracle.sparse_attention(host64(q), K, V, host64(idx), scale)
    check_attention(host64(out), ref, "attention")


@pytest.mark.parametrize("rows,k", [((3, 1, 999, 1000), 512),      # decode: split-k + combine
                                    ((2, 3, 4000, 4003), 2048),    # few rows, long k
                                    ((1, 160, 0, 160), 64),        # prefill, early rows short
                                    ((2, 1, 40, 41), 2048)])       # fewer keys than k
def test_latent_attention_tensor_core_path(dev, rows, k):
    B, Lq, q_start, T = rows
    g = torch.Generator(device=dev).manual_seed(k + T)
    q = torch.randn(B, Lq, 128, 576, device=dev, generator=g).bfloat16()
    kv = (torch.randn(B, T, 576, device=dev, generator=g) / 24 ** 0.5).bfloat16()
    idx = synth.random_index_sets(B, Lq, q_start, k, dev, seed=k)
    if Lq > 1:
        idx[0, 1, 5:9] = -1                      # holes inside a row are masked
        idx[0, 2, :] = -1                        # no valid key: the row is zero
    out = torch.empty(B, Lq, 128, 512, device=dev, dtype=torch.bfloat16)
    ws = _ws(ic.sparse_attn_workspace_size(rows, k, 128, 576, 512, ic.BF16), dev)
    n0, tc0 = ic.kernel_launches(3), ic.kernel_launches(6)
    ic.sparse_attn(q, kv, 576, kv, 576, idx, rows, 512, 576 ** -0.5, out, ws)
    torch.cuda.synchronize()
    assert ic.kernel_launches(3) - n0 == 1 and ic.kernel_launches(6) - tc0 == 1
    assert ic.read_status(ws) == 0
    kvh = host64(kv)
    ref = oracle.sparse_attention(host64(q), kvh, kvh[..., :512], host64(idx), 576 ** -0.5)
    check_attention(host64(out), ref, "latent attention")


@pytest.mark.parametrize("gain", [8, 16])
@pytest.mark.parametrize("rows,k", [((1, 96, 1904, 2000), 2048),   # prefill rows: one unit each
                                    ((4, 1, 2999, 3000), 2048)])    # decode: split-k + combine
def test_latent_attention_sharp_logits(dev, gain, rows, k):
    """Sharp attention: q scaled x8 / x16 with KV ~ N(0,1) and scale 1/24, so
    the logits in base 2 reach +-100 and each CTA's partial logit (its 288 of
    the 576 columns) reaches 30-80.  The two CTAs of a pair exchange those
    partial logits; the softmax weights, and so the outputs, must still be
    within the attention tolerance of the float64 oracle, element by element,
    on prefill rows and on split-k decode rows."""
    B, Lq, q_start, T = rows
    g = torch.Generator(device=dev).manual_seed(gain * 1000 + Lq)
    q = (torch.randn(B, Lq, 128, 576, device=dev, generator=g) * gain).bfloat16()
    kv = torch.randn(B, T, 576, device=dev, generator=g).bfloat16()
    idx = synth.random_index_sets(B, Lq, q_start, k, dev, seed=gain + Lq)
    out = torch.empty(B, Lq, 128, 512, device=dev, dtype=torch.bfloat16)
    ws = _ws(ic.sparse_attn_workspace_size(rows, k, 128, 576, 512, ic.BF16), dev)
    tc0 = ic.kernel_launches(6)
    ic.sparse_attn(q, kv, 576, kv, 576, idx, rows, 512, 576 ** -0.5, out, ws)
    torch.cuda.synchronize()
    assert ic.kernel_launches(6) - tc0 == 1
    site = int(ws[4:8].view(torch.int32).item())     # the first wait that ran out, if any
    assert ic.read_status(ws) == 0, "wait site %d of CTA %d ran out" % (site & 255, site >> 8)
    qh, kvh = host64(q), host64(kv)
    # the test really is sharp: base-2 logits of the first row reach tens
    logit2 = (qh[0, 0] @ kvh[0, :T].T) * 576 ** -0.5 / np.log(2)
    assert np.abs(logit2).max() > 4 * gain
    ref = oracle.sparse_attention(qh, kvh, kvh[..., :512], host64(idx), 576 ** -0.5)
    check_attention(host64(out), ref, "sharp attention x%d" % gain)


@pytest.mark.parametrize("latent", [False, True])
def test_equal_key_rows_give_that_value_row(dev, latent):
    """Every key/value row equal: whatever the softmax weights, they sum to
    one, so every head of every row outputs that value row (fp32 CUDA-core
    path; bf16 tensor-core path, split-k decode rows included)."""
    if latent:
        rows, Hq, d_qk, d_v, dt, k = (3, 2, 1998, 2000), 128, 576, 512, torch.bfloat16, 1024
    else:
        rows, Hq, d_qk, d_v, dt, k = (2, 5, 195, 200), 8, 64, 48, torch.float32, 64
    B, Lq, q_start, T = rows
    g = torch.Generator(device=dev).manual_seed(17)
    q = torch.randn(B, Lq, Hq, d_qk, device=dev, generator=g).to(dt)
    one = torch.randn(1, 1, d_qk if latent else d_qk + d_v, device=dev, generator=g).to(dt)
    if latent:
        kmat = vmat = one.expand(B, T, d_qk).contiguous()
        ks = vs = d_qk
        v_row = host64(one)[0, 0, :d_v]
    else:
        kmat = one[..., :d_qk].expand(B, T, d_qk).contiguous()
        vmat = one[..., d_qk:].expand(B, T, d_v).contiguous()
        ks, vs = d_qk, d_v
        v_row = host64(one)[0, 0, d_qk:]
    idx = synth.random_index_sets(B, Lq, q_start, k, dev, seed=17)
    out = torch.empty(B, Lq, Hq, d_v, device=dev, dtype=dt)
    ws = _ws(ic.sparse_attn_workspace_size(rows, k, Hq, d_qk, d_v, DT["bf16" if latent else "f32"]),
             dev)
    ic.sparse_attn(q, kmat, ks, vmat, vs, idx, rows, d_v, d_qk ** -0.5, out, ws)
    torch.cuda.synchronize()
    assert ic.read_status(ws) == 0
    ref = np.broadcast_to(v_row, (B, Lq, Hq, d_v))
    check_attention(host64(out), ref, "equal key rows")


def test_attention_flags_and_skips_out_of_range_indices(dev):
    rows = (1, 4, 10, 14)
    B, Lq, q_start, T = rows
    g = torch.Generator(device=dev).manual_seed(0)
    q = torch.randn(B, Lq, 8, 64, device=dev, generator=g)
    K = torch.randn(B, T, 64, device=dev, generator=g)
    V = torch.randn(B, T, 64, device=dev, generator=g)
    idx = torch.tensor([[[0, 3, 11, -1], [1, 2, 99, -1], [4, -5, 6, 7], [0, 1, 2, 3]]],
                       dtype=torch.int32, device=dev)   # 11 > t=10, 99 >= T, -5 < -1
    out = torch.empty(B, Lq, 8, 64, device=dev)
    ws = _ws(ic.sparse_attn_workspace_size(rows, 4, 8, 64, 64, ic.F32), dev)
    ic.sparse_attn(q, K, 64, V, 64, idx, rows, 64, 0.125, out, ws)
    torch.cuda.synchronize()
    assert ic.read_status(ws) & 1
    clean = host64(idx).copy()
    clean[0, 0, 2] = clean[0, 1, 2] = clean[0, 2, 1] = -1
    ref = oracle.sparse_attention(host64(q), host64(K), host64(V), clean, 0.125)
    check_attention(host64(out), ref, "out-of-range skip")
    assert ic.read_status(ws) == 0                       # cleared by the read


# ------------------------------------------------------------------------- stack
def _stack_inputs(wl, dev, layers=None):
    n = wl.n_layers if layers is None else layers
    return [synth.layer_inputs(wl, l, dev) for l in range(n)]


def _run_stack(wl, pattern, inputs, dev, rows=None, idx_out=True):
    B, L, q_start, T = (wl.B, wl.L, wl.q_start, wl.T) if rows is None else rows
    r = ic.Rows(B, L, q_start, T)
    sh = ic.StackShape(r, wl.H_I, wl.d_I, DT[wl.idx_dtype], wl.k, wl.Hq, wl.d_qk, wl.d_v,
                       DT[wl.attn_dtype], wl.d_qk, wl.d_qk if wl.latent else wl.d_v, wl.scale)
    ws = _ws(ic.workspace_size(sh), dev)
    torch_dt = torch.float32 if wl.attn_dtype == "f32" else torch.bfloat16
    idx_buf = torch.empty(B, L, wl.k, dtype=torch.int32, device=dev)
    outs = [torch.empty(B, L, wl.Hq, wl.d_v, dtype=torch_dt, device=dev) for _ in pattern]
    idx_copies = [torch.empty_like(idx_buf) for _ in pattern] if idx_out else None
    layers = []
    for l, inp in enumerate(inputs):
        kmat = inp["kv"] if wl.latent else inp["k"]
        vmat = inp["kv"] if wl.latent else inp["v"]
        layers.append(dict(q_idx=inp.get("q_I"), q_scale=inp.get("q_scale"), w=inp.get("w"),
                           k_idx=inp.get("k_I"), k_scale=inp.get("k_scale"), q=inp["q"],
                           kmat=kmat, vmat=vmat, out=outs[l]))
    before = ic.kernel_launches(1)
    ic.layer_stack_forward(pattern, layers, sh, idx_buf, ws, idx_out=idx_copies)
    torch.cuda.synchronize()
    n_indexer = ic.kernel_launches(1) - before
    assert ic.read_status(ws) == 0
    return outs, idx_copies, n_indexer


def _oracle_layers(wl, inputs, rows=None):
    res = []
    for inp in inputs:
        d = dict(q=host64(inp["q"]))
        if wl.latent:
            kv = host64(inp["kv"])
            d["K"], d["V"] = kv, kv[..., : wl.d_v]
        else:
            d["K"], d["V"] = host64(inp["k"]), host64(inp["v"])
        for key in ("q_I", "w", "k_I", "q_scale", "k_scale"):
            if key in inp:
                d[key] = host64(inp[key])
        res.append(d)
    return res


@pytest.mark.parametrize("pattern", ["FSSS", "FFFF", "FSFS"])
def test_prefill_512_fp32_stack_every_row(dev, pattern):
    wl = synth.WORKLOADS["prefill_512_fp32"]
    inputs = _stack_inputs(wl, dev)
    outs, idx_copies, n_ix = _run_stack(wl, pattern, inputs, dev)
    assert n_ix == pattern.count("F")                           # indexer runs on F layers only
    ol = _oracle_layers(wl, inputs)
    last_f = 0
    for l, kind in enumerate(pattern):
        gidx = host64(idx_copies[l])
        if kind == "F":
            last_f = l
            sc = oracle.indexer_scores(ol[l]["q_I"], ol[l]["w"], ol[l]["k_I"], wl.q_start)
            check_topk_band(gidx, sc, wl.q_start, wl.k)
        else:                                                   # invariant: reuse, bit for bit
            assert np.array_equal(gidx, host64(idx_copies[last_f]))
        # every row: the oracle's attention over the (band-valid) keys the kernel chose
        ref = oracle.sparse_attention(ol[l]["q"], ol[l]["K"], ol[l]["V"], gidx, wl.scale)
        check_attention(host64(outs[l]), ref, "layer %d" % l)


@pytest.mark.parametrize("latent", [False, True])
def test_stack_is_dense_causal_attention_when_k_covers_the_context(dev, latent):
    """With k >= t + 1 on every row, each F layer keeps every causal key, so
    every layer's output is ordinary dense causal attention, computed by the
    oracle's separate dense routine (fp32 CUDA-core path; bf16 tensor-core
    path with the latent 576-wide KV, rows starting at q_start = 40)."""
    if latent:
        wl = synth.Workload("dense_latent", 1, 160, 200, 40, 64, 128, 256, 128, 576, 512, "bf16",
                            "bf16", True, "FS", 13, 1 / 8, 128 ** -0.5, 128 ** -0.5, 1.0, 1.0)
    else:
        wl = dataclasses.replace(synth.WORKLOADS["prefill_512_fp32"], k=512)
    inputs = _stack_inputs(wl, dev)
    outs, idx_copies, n_ix = _run_stack(wl, wl.pattern, inputs, dev)
    assert n_ix == wl.pattern.count("F")
    ol = _oracle_layers(wl, inputs)
    t = wl.q_start + np.arange(wl.L)
    for l in range(wl.n_layers):
        gidx = host64(idx_copies[l])[0]
        for i in range(wl.L):
            assert np.array_equal(gidx[i, : t[i] + 1], np.arange(t[i] + 1))
            assert np.all(gidx[i, t[i] + 1:] == -1)
        ref = oracle.dense_causal_attention(ol[l]["q"], ol[l]["K"], ol[l]["V"], wl.q_start,
                                            wl.scale)
        check_attention(host64(outs[l]), ref, "dense identity layer %d" % l)


def test_exact_mode_stack_is_bit_exact_in_indices(dev):
    """Exact-mode indexer inputs in a 2-layer bf16 stack: GPU indices equal
    the oracle's for every row, and the S layer reuses them."""
    B, L, T, H_I, d_I, k = 1, 300, 300, 64, 128, 64
    wl = synth.Workload("exact", B, L, T, 0, H_I, d_I, k, 8, 64, 64, "bf16", "bf16", False, "FS",
                        9, 1, 1, 1, 1, 1)
    inputs = []
    for l in range(2):
        inp = synth.exact_indexer_inputs(B, L, T, H_I, d_I, "bf16", dev, seed=20 + l)
        g = torch.Generator(device=dev).manual_seed(l)
        inp["q"] = torch.randn(B, L, 8, 64, device=dev, generator=g).bfloat16()
        inp["k"] = torch.randn(B, T, 64, device=dev, generator=g).bfloat16()
        inp["v"] = torch.randn(B, T, 64, device=dev, generator=g).bfloat16()
        inputs.append(inp)
    outs, idx_copies, n_ix = _run_stack(wl, "FS", inputs, dev)
    assert n_ix == 1
    ol = _oracle_layers(wl, inputs)
    idx_ref, out_ref, n_ref = oracle.layer_stack("FS", ol, 0, k, wl.scale)
    assert n_ref == 1
    for l in range(2):
        assert np.array_equal(host64(idx_copies[l]), idx_ref[l])
        check_attention(host64(outs[l]), out_ref[l], "exact layer %d" % l)


def test_degenerate_rows(dev):
    """Single candidate (t = 0) with k larger than the context: the one key
    is selected and the output is its value row.  (Empty batches are no-ops
    that return before any device work; the CPU ABI test covers them.)"""
    wl = synth.WORKLOADS["prefill_512_fp32"]
    inputs = [synth.layer_inputs(wl, 0, dev)]
    rows = (1, 1, 0, 1)
    for key in ("q_I", "w", "q"):
        inputs[0][key] = inputs[0][key][:, :1].contiguous()
    for key in ("k_I", "k", "v"):
        inputs[0][key] = inputs[0][key][:, :1].contiguous()
    outs, idx_copies, _ = _run_stack(wl, "F", inputs, dev, rows=rows)
    assert host64(idx_copies[0])[0, 0].tolist() == [0] + [-1] * (wl.k - 1)
    assert np.allclose(host64(outs[0])[0, 0], host64(inputs[0]["v"])[0, 0][None, :], atol=1e-6)


# ------------------------------------------------------------------------- failure path
def test_stalled_wait_ends_with_timeout_status_and_usable_context(dev):
    """A pipeline wait that nothing completes gives up after its bounded time:
    the status word reports the timeout bit (2), the kernel returns, and the
    context keeps working (a top-k afterwards is still bit-exact)."""
    ws = _ws(1 << 16, dev)
    ic.selftest_wait_timeout(ws)
    torch.cuda.synchronize()
    assert ic.read_status(ws) == 2
    rows, k = (1, 8, 100, 108), 16
    scores = synth.random_scores(1, 8, 108, dev, seed=5)
    idx = torch.full((1, 8, k), -7, dtype=torch.int32, device=dev)
    ic.topk(scores, rows, k, idx, _ws(ic.topk_workspace_size(rows, k), dev))
    torch.cuda.synchronize()
    assert np.array_equal(host64(idx), oracle.topk_indices(host64(scores), 100, k))
