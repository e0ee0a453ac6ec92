"""GPU parity of the variable-length, paged-cache calls (ic_*_paged,
ic_topk_varlen) against the float64 oracle.

A batch of sequences of different lengths keeps its indexer keys, their FP8
scales and its latent KV rows in pages shuffled over one physical cache (the
serving layout behind the pages' saturated-KV throughput figure).  The
oracle knows nothing of pages: each sequence's logical arrays are built
first, scattered into the pages through the block table, and the library's
results are compared, sequence by sequence, with the oracle on the logical
arrays (its own q_start = seq_len - Lq).
"""
import numpy as np
import pytest
import torch

import oracle
import cross_layer_top_full_b200 as ic
from cross_layer_top_full_b200 import synth
from parity_util import (abs_term_sum, check_attention, check_scores, check_topk_band, host64)

pytestmark = pytest.mark.gpu

DT = {"bf16": ic.BF16, "e4m3": ic.FP8_E4M3}


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


class Batch:
    """Logical per-sequence caches and their paged copies."""

    def __init__(self, lens, Lq, page_size, dev, seed, idx_dtype="bf16", T_max=None,
                 spare_pages=3, H_I=64, gain=1.0, layout_seed=None):
        g = torch.Generator(device="cpu").manual_seed(seed)
        g_layout = torch.Generator(device="cpu").manual_seed(seed if layout_seed is None
                                                             else layout_seed)
        self.lens, self.Lq, self.P = list(lens), Lq, page_size
        self.B = len(lens)
        self.T_max = T_max or max(lens)
        self.idx_dtype = idx_dtype
        pages_per = [(n + page_size - 1) // page_size for n in lens]
        self.max_pages = (self.T_max + page_size - 1) // page_size
        self.num_pages = sum(pages_per) + spare_pages
        perm = torch.randperm(self.num_pages, generator=g_layout)
        bt = torch.full((self.B, self.max_pages), -1, dtype=torch.int32)
        c = 0
        for b, np_ in enumerate(pages_per):
            bt[b, :np_] = perm[c:c + np_].to(torch.int32)
            c += np_
        self.block_table = bt
        rows = self.num_pages * page_size
        # logical arrays per sequence (host, float32 before storage rounding)
        self.kI = [torch.randn(n, 128, generator=g) / 128 ** 0.5 for n in lens]
        self.kv = [(torch.randn(n, 576, generator=g) * gain).bfloat16() for n in lens]
        self.qI = torch.randn(self.B, Lq, H_I, 128, generator=g) / 128 ** 0.5
        self.w = torch.randn(self.B, Lq, H_I, generator=g) / 8
        self.q = torch.randn(self.B, Lq, 128, 576, generator=g).bfloat16()
        # paged storage
        kv_pages = torch.zeros(rows, 576, dtype=torch.bfloat16)
        if idx_dtype == "e4m3":
            self.qI_codes, self.q_scale = synth.fp8_per_token(self.qI, 2)
            codes, scales = [], []
            for x in self.kI:
                cd, sc = synth.fp8_per_token(x[None], 2)
                codes.append(cd[0])
                scales.append(sc[0])
            self.kI_codes, self.k_scale = codes, scales
            kI_pages = torch.zeros(rows, 128, dtype=torch.uint8)
            ks_pages = torch.zeros(rows, dtype=torch.float32)
        else:
            self.kI_b = [x.bfloat16() for x in self.kI]
            kI_pages = torch.zeros(rows, 128, dtype=torch.bfloat16)
        for b, n in enumerate(lens):
            phys = self.phys_rows(b, n)
            kv_pages[phys] = self.kv[b]
            if idx_dtype == "e4m3":
                kI_pages[phys] = self.kI_codes[b]
                ks_pages[phys] = self.k_scale[b]
            else:
                kI_pages[phys] = self.kI_b[b]
        self.dev = dev
        self.d_seq = torch.tensor(lens, dtype=torch.int32, device=dev)
        self.d_bt = bt.to(dev)
        self.d_kv = kv_pages.to(dev)
        self.d_kI = kI_pages.to(dev)
        self.d_ks = ks_pages.to(dev) if idx_dtype == "e4m3" else None
        self.d_qI = (self.qI_codes if idx_dtype == "e4m3" else self.qI.bfloat16()).to(dev)
        self.d_qs = self.q_scale.to(dev) if idx_dtype == "e4m3" else None
        self.d_w = self.w.to(dev)
        self.d_q = self.q.to(dev)
        self.pr = ic.paged_rows(self.d_seq, self.d_bt, self.T_max, page_size, self.num_pages, Lq)

    def phys_rows(self, b, n):
        s = torch.arange(n)
        return self.block_table[b, s // self.P].to(torch.int64) * self.P + s % self.P

    def q_start(self, b):
        return self.lens[b] - self.Lq

    def oracle_scores(self, b):
        fp8 = self.idx_dtype == "e4m3"
        if fp8:
            return oracle.indexer_scores(host64(self.qI_codes[b:b + 1]), host64(self.w[b:b + 1]),
                                         host64(self.kI_codes[b][None]), self.q_start(b),
                                         host64(self.q_scale[b:b + 1]),
                                         host64(self.k_scale[b][None]), fp8=True)
        return oracle.indexer_scores(host64(self.qI.bfloat16()[b:b + 1]), host64(self.w[b:b + 1]),
                                     host64(self.kI_b[b][None]), self.q_start(b))

    def abs_sum(self, b):
        if self.idx_dtype == "e4m3":
            from oracle.indexcache_oracle import e4m3_decode
            q = e4m3_decode(host64(self.qI_codes[b:b + 1])) * host64(self.q_scale[b:b + 1])[..., None, None]
            k = e4m3_decode(host64(self.kI_codes[b][None])) * host64(self.k_scale[b][None])[..., None]
            return abs_term_sum(q, host64(self.w[b:b + 1]), k)
        return abs_term_sum(host64(self.qI.bfloat16()[b:b + 1]), host64(self.w[b:b + 1]),
                            host64(self.kI_b[b][None]))


LENS = [300, 5000, 4096, 131, 7777, 2049]


@pytest.mark.parametrize("idx_dtype", ["bf16", "e4m3"])
@pytest.mark.parametrize("Lq,page", [(1, 128), (3, 256)])
def test_paged_indexer_scores(dev, idx_dtype, Lq, page):
    bt = Batch(LENS, Lq, page, dev, seed=1 + Lq, idx_dtype=idx_dtype)
    ld = (bt.T_max + 3) // 4 * 4
    scores = torch.full((bt.B, Lq, ld), float("nan"), device=dev)
    ws = _ws(ic.STATUS_BYTES, dev)
    ic.indexer_scores_paged(bt.d_qI, bt.d_w, bt.d_kI, bt.pr, scores, ws, q_scale=bt.d_qs,
                            k_scale_pages=bt.d_ks, dtype=DT[idx_dtype])
    torch.cuda.synchronize()
    assert ic.read_status(ws) == 0
    got = host64(scores)
    for b in range(bt.B):
        ref = bt.oracle_scores(b)
        check_scores(got[b:b + 1, :, :bt.lens[b]], ref, bt.abs_sum(b), bt.q_start(b), 1e-4)


@pytest.mark.parametrize("ties", [False, True])
def test_topk_varlen_is_bit_exact(dev, ties):
    """Per-sequence lengths: cluster rows (few, long) and many-row rows."""
    # few long rows: one cluster per row (8 CTAs, then 1); 300 rows: one CTA per row
    for lens, Lq in (([300, 50000, 4096, 131, 77777, 2049], 1), ([9000, 3000, 6100], 40),
                     ([5000, 7000], 150)):
        T_max = max(lens) + 5
        B = len(lens)
        scores = synth.random_scores(B, Lq, T_max, dev, seed=B + Lq, ties=ties)
        seq = torch.tensor(lens, dtype=torch.int32, device=dev)
        pr = ic.paged_rows(seq, None, T_max, 128, 1, Lq)
        k = 2048
        idx = torch.full((B, Lq, k), -7, dtype=torch.int32, device=dev)
        ic.topk_varlen(scores, pr, k, idx, _ws(ic.topk_varlen_workspace_size(pr, k), dev))
        torch.cuda.synchronize()
        got, sc = host64(idx), host64(scores)
        for b, n in enumerate(lens):
            ref = oracle.topk_indices(sc[b:b + 1, :, :n], n - Lq, k)
            assert np.array_equal(got[b:b + 1], ref), (b, n)


def _oracle_attention(bt, b, idx_row_set):
    kv = host64(bt.kv[b])[None]
    return oracle.sparse_attention(host64(bt.q[b:b + 1]), kv, kv[..., :512], idx_row_set, 576 ** -0.5)


@pytest.mark.parametrize("Lq,page,k", [(1, 128, 2048), (2, 256, 512)])
def test_paged_attention(dev, Lq, page, k):
    bt = Batch(LENS, Lq, page, dev, seed=7 + k)
    idx = torch.full((bt.B, Lq, k), -1, dtype=torch.int32)
    for b, n in enumerate(bt.lens):
        sets = synth.random_index_sets(1, Lq, n - Lq, k, "cpu", seed=b + k)
        idx[b] = sets[0]
    idx[1, 0, 7:20] = -1                                   # holes
    d_idx = idx.to(dev)
    out = torch.full((bt.B, Lq, 128, 512), float("nan"), dtype=torch.bfloat16, device=dev)
    ws = _ws(ic.sparse_attn_paged_workspace_size(bt.pr, k), dev)
    ic.sparse_attn_paged(bt.d_q, bt.d_kv, d_idx, bt.pr, 576 ** -0.5, out, ws)
    torch.cuda.synchronize()
    assert ic.read_status(ws) == 0
    got = host64(out)
    for b in range(bt.B):
        ref = _oracle_attention(bt, b, host64(idx[b:b + 1]))
        check_attention(got[b:b + 1], ref, "paged attention seq %d" % b)


@pytest.mark.parametrize("idx_dtype,pattern", [("bf16", "FSSF"), ("e4m3", "FSFS")])
def test_paged_stack_matches_the_oracle_per_sequence(dev, idx_dtype, pattern):
    """The F/S stack over paged caches of a ragged decode batch: F indices obey
    the band rule against each sequence's own float64 scores, S layers reuse
    them bit for bit, and every row's attention is within tolerance of the
    oracle over the keys chosen."""
    Lq, page, k = 1, 128, 2048
    batches = [Batch(LENS, Lq, page, dev, seed=20 + l, idx_dtype=idx_dtype, layout_seed=99)
               for l in range(len(pattern))]
    bt0 = batches[0]
    sh = ic.StackShape(ic.Rows(bt0.B, Lq, 0, bt0.T_max), 64, 128, DT[idx_dtype], k, 128, 576, 512,
                       ic.BF16, 576, 576, 576 ** -0.5)
    # every layer shares the batch geometry (lengths and block table) of layer 0
    for bt in batches[1:]:
        assert torch.equal(bt.block_table, bt0.block_table)
    ws = _ws(ic.paged_workspace_size(sh, bt0.pr), dev)
    idx_buf = torch.empty(bt0.B, Lq, k, dtype=torch.int32, device=dev)
    outs = [torch.empty(bt0.B, Lq, 128, 512, dtype=torch.bfloat16, device=dev) for _ in pattern]
    copies = [torch.empty_like(idx_buf) for _ in pattern]
    layers = [dict(q_idx=bt.d_qI, q_scale=bt.d_qs, w=bt.d_w, k_idx=bt.d_kI, k_scale=bt.d_ks,
                   q=bt.d_q, kmat=bt.d_kv, vmat=bt.d_kv, out=o) for bt, o in zip(batches, outs)]
    n0 = ic.kernel_launches(1)
    ic.layer_stack_forward_paged(pattern, layers, sh, bt0.pr, idx_buf, ws, idx_out=copies)
    torch.cuda.synchronize()
    assert ic.read_status(ws) == 0
    assert ic.kernel_launches(1) - n0 == pattern.count("F")
    last_f = None
    for l, kind in enumerate(pattern):
        gidx = host64(copies[l])
        if kind == "F":
            last_f = l
            for b in range(bt0.B):
                check_topk_band(gidx[b:b + 1], batches[l].oracle_scores(b), bt0.q_start(b), k)
        else:
            assert np.array_equal(gidx, host64(copies[last_f]))
        got = host64(outs[l])
        for b in range(bt0.B):
            ref = _oracle_attention(batches[l], b, gidx[b:b + 1])
            check_attention(got[b:b + 1], ref, "paged stack layer %d seq %d" % (l, b))


def test_identity_paging_equals_the_dense_calls(dev):
    """Pages in order and every sequence T long: the paged calls give the
    dense calls' scores, indices and outputs bit for bit (same kernels, same
    arithmetic, only the row addressing differs)."""
    B, T, Lq, k = 3, 4096, 1, 1024
    wl = synth.Workload("ident", B, Lq, T, T - Lq, 64, 128, k, 128, 576, 512, "bf16", "bf16", True,
                        "F", 31, 1 / 8, 128 ** -0.5, 128 ** -0.5, 1.0, 1.0)
    inp = synth.layer_inputs(wl, 0, dev)
    P = 128
    bt = torch.arange(B * (T // P), dtype=torch.int32, device=dev).view(B, T // P)
    seq = torch.full((B,), T, dtype=torch.int32, device=dev)
    pr = ic.paged_rows(seq, bt, T, P, B * T // P, Lq)
    rows = (B, Lq, T - Lq, T)
    ws = _ws(1 << 24, dev)
    sd = torch.empty(B, Lq, T, device=dev)
    sp = torch.empty_like(sd)
    ic.indexer_scores(inp["q_I"], inp["w"], inp["k_I"], rows, sd, ws)
    ic.indexer_scores_paged(inp["q_I"], inp["w"], inp["k_I"].view(B * T, 128), pr, sp, ws)
    torch.cuda.synchronize()
    assert torch.equal(sd, sp)
    idd = torch.empty(B, Lq, k, dtype=torch.int32, device=dev)
    idp = torch.empty_like(idd)
    ic.topk(sd, rows, k, idd, ws)
    ic.topk_varlen(sd, pr, k, idp, ws)
    torch.cuda.synchronize()
    assert torch.equal(idd, idp)
    od = torch.empty(B, Lq, 128, 512, dtype=torch.bfloat16, device=dev)
    op = torch.empty_like(od)
    ic.sparse_attn(inp["q"], inp["kv"], 576, inp["kv"], 576, idd, rows, 512, wl.scale, od, ws)
    ic.sparse_attn_paged(inp["q"], inp["kv"].view(B * T, 576), idd, pr, wl.scale, op, ws)
    torch.cuda.synchronize()
    assert ic.read_status(ws) == 0
    assert torch.equal(od, op)


def test_out_of_range_lengths_give_empty_rows(dev):
    """A sequence length of 0 or above T_max: its top-k row is all -1 and its
    attention output is zero; the other sequences are unaffected."""
    lens = [600, 0, 900]
    T_max = 1000
    bt = Batch([600, 1, 900], 1, 128, dev, seed=5, T_max=T_max)
    bt.d_seq.copy_(torch.tensor(lens, dtype=torch.int32))
    k = 256
    ld = (T_max + 3) // 4 * 4
    scores = torch.zeros(bt.B, 1, ld, device=dev)
    ws = _ws(ic.sparse_attn_paged_workspace_size(bt.pr, k), dev)
    ic.indexer_scores_paged(bt.d_qI, bt.d_w, bt.d_kI, bt.pr, scores, ws)
    idx = torch.empty(bt.B, 1, k, dtype=torch.int32, device=dev)
    ic.topk_varlen(scores, bt.pr, k, idx, ws)
    out = torch.full((bt.B, 1, 128, 512), float("nan"), dtype=torch.bfloat16, device=dev)
    ic.sparse_attn_paged(bt.d_q, bt.d_kv, idx, bt.pr, 576 ** -0.5, out, ws)
    torch.cuda.synchronize()
    assert ic.read_status(ws) & 1                         # the indexer flagged the bad length
    assert np.all(host64(idx[1]) == -1)
    assert not torch.isnan(out.float()).any()
    assert host64(out[1]).max() == 0 and host64(out[1]).min() == 0
    for b in (0, 2):
        ref = oracle.topk_indices(bt.oracle_scores(b), lens[b] - 1, k)
        check_topk_band(host64(idx[b:b + 1]), bt.oracle_scores(b), lens[b] - 1, k)
        assert (host64(idx[b:b + 1]) >= 0).sum() == ref[ref >= 0].size
