"""Benchmark of the IndexCache hot path on B200.

One step = one pass of the whole layer stack (indexer -> top-k on F layers,
sparse attention on every layer) over one batch of seeded synthetic input,
through the C ABI (``ic_layer_stack_forward``).  Default workload:
prefill_8k_bf16 (1 sequence, L=8192, pattern FSSS); the all-F stack (FFFF)
is timed on the same inputs for the IndexCache comparison.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--pattern P] [--impl ours|reference]

Multi-GPU (torchrun, one process per GPU): every rank runs its own replica
of the workload (its own sequences, seed offset by rank), no data-path
collective; the time is the max over ranks and the value counts all ranks'
tokens ("scaling": "weak").  ``--impl reference`` times the float64 CPU
oracle on a bounded sample of the same workload (rank 0 only).

Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import cross_layer_top_full_b200 as ic  # noqa: E402
from cross_layer_top_full_b200 import synth  # noqa: E402

DT = {"f32": ic.F32, "bf16": ic.BF16, "e4m3": ic.FP8_E4M3}
L2_BYTES = 126 * 1024 * 1024


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p["bf16_tflops_sustained"], "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ----------------------------------------------------------------------------- workload
def replica_workload(wl, rank):
    """The workload replica of one rank: same shapes, its own sequences
    (seed offset by rank), no data shared between ranks."""
    import dataclasses
    return dataclasses.replace(wl, seed=wl.seed + 1000 * rank) if rank else wl


def max_over_ranks(ms, pg, dev):
    """Slowest rank's time (every rank gets it); ``pg`` is torch.distributed
    or None for one process."""
    if not pg:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, world, ms_per_step):
    """Units per second processed by all ranks together."""
    return units_per_rank * world / (ms_per_step / 1e3)


class Stack:
    """Device-resident inputs and buffers of one replica of a workload."""

    def __init__(self, wl, dev, rank=0):
        wl = replica_workload(wl, rank)
        self.wl = wl
        self.dev = dev
        self.inputs = [synth.layer_inputs(wl, l, dev) for l in range(wl.n_layers)]
        torch_dt = torch.float32 if wl.attn_dtype == "f32" else torch.bfloat16
        self.outs = [torch.empty(wl.B, wl.L, wl.Hq, wl.d_v, dtype=torch_dt, device=dev)
                     for _ in range(wl.n_layers)]
        self.rows = ic.Rows(wl.B, wl.L, wl.q_start, wl.T)
        self.shape = ic.StackShape(self.rows, wl.H_I, wl.d_I, DT[wl.idx_dtype], wl.k, wl.Hq,
                                   wl.d_qk, wl.d_v, DT[wl.attn_dtype], wl.d_qk,
                                   wl.d_qk if wl.latent else wl.d_v, wl.scale)
        self.ws = torch.empty(ic.workspace_size(self.shape), dtype=torch.uint8, device=dev)
        ic.workspace_init(self.ws)
        self.idx = torch.empty(wl.B, wl.L, wl.k, dtype=torch.int32, device=dev)
        self.layers = self._layer_dicts(self.inputs, self.outs)
        # per-stage calls (same kernels as the stack) for the stage breakdown
        self.ld = (wl.T + 3) // 4 * 4
        self.scores = torch.empty(wl.B, wl.L, self.ld, dtype=torch.float32, device=dev)

    def _layer_dicts(self, inputs, outs):
        wl = self.wl
        res = []
        for l, inp in enumerate(inputs):
            kmat = inp["kv"] if wl.latent else inp["k"]
            vmat = inp["kv"] if wl.latent else inp["v"]
            res.append(dict(q_idx=inp.get("q_I"), q_scale=inp.get("q_scale"), w=inp.get("w"),
                            k_idx=inp.get("k_I"), k_scale=inp.get("k_scale"), q=inp["q"],
                            kmat=kmat, vmat=vmat, out=outs[l]))
        return res

    def step(self, pattern, stream=None):
        ic.layer_stack_forward(pattern, self.layers, self.shape, self.idx, self.ws, stream=stream)

    def stage_step(self, pattern, ev):
        """The same step as separate C-ABI calls, with CUDA events around each.
        Decode F layers run the fused key selection (ic_indexer_topk, the
        stack's path: stage "select"); the un-fused indexer and top-k are
        timed after it as references (stages "indexer" and "topk", not part
        of the step's path)."""
        wl = self.wl
        for l, kind in enumerate(pattern):
            L = self.layers[l]
            if kind == "F":
                if fused_selection(wl):
                    e = ev.new()
                    e.record()
                    ic.indexer_topk(L["q_idx"], L["w"], L["k_idx"], self.rows, wl.k, self.idx,
                                    self.ws, q_scale=L["q_scale"], k_scale=L["k_scale"],
                                    dtype=DT[wl.idx_dtype])
                    e0 = ev.new()
                    e0.record()
                    ev.add("select", e, e0)
                else:
                    e0 = ev.new()
                    e0.record()
                e1, e2 = ev.new(), ev.new()
                ic.indexer_scores(L["q_idx"], L["w"], L["k_idx"], self.rows, self.scores, self.ws,
                                  q_scale=L["q_scale"], k_scale=L["k_scale"],
                                  dtype=DT[wl.idx_dtype])
                e1.record()
                ic.topk(self.scores, self.rows, wl.k, self.idx, self.ws)
                e2.record()
                ev.add("indexer", e0, e1)
                ev.add("topk", e1, e2)
            e3, e4 = ev.new(), ev.new()
            e3.record()
            ic.sparse_attn(L["q"], L["kmat"], wl.d_qk, L["vmat"], wl.d_qk if wl.latent else wl.d_v,
                           self.idx, self.rows, wl.d_v, wl.scale, L["out"], self.ws,
                           dtype=DT[wl.attn_dtype])
            e4.record()
            ev.add("attention", e3, e4)

    def own_selection(self, l):
        """Layer l's own top-k (its indexer run as if the layer were F)."""
        L = self.layers[l]
        ic.indexer_scores(L["q_idx"], L["w"], L["k_idx"], self.rows, self.scores, self.ws,
                          q_scale=L["q_scale"], k_scale=L["k_scale"], dtype=DT[self.wl.idx_dtype])
        ic.topk(self.scores, self.rows, self.wl.k, self.idx, self.ws)
        return self.idx.view(-1, self.wl.k).clone()

    def bytes_per_step(self, pattern):
        """H2D bytes of one step's inputs (F layers carry indexer inputs)."""
        n = 0
        for l, kind in enumerate(pattern):
            for key, t in self.inputs[l].items():
                if kind == "S" and key in ("q_I", "w", "k_I", "q_scale", "k_scale"):
                    continue
                n += t.numel() * t.element_size()
        return n


class PagedStack(Stack):
    """Device-resident inputs of a variable-length batch over paged caches:
    every layer's k_I / KV caches in shuffled 128-row pages, one block table
    and one set of sequence lengths for the batch."""

    def __init__(self, wl, dev, rank=0):
        wl = replica_workload(wl, rank)
        self.wl = wl
        self.dev = dev
        self.seq, self.table, self.num_pages = synth.paged_batch(wl, dev)
        self.lens = self.seq.cpu().tolist()
        self.inputs = [synth.paged_layer_inputs(wl, l, self.num_pages, dev)
                       for l in range(wl.n_layers)]
        self.outs = [torch.empty(wl.B, wl.L, wl.Hq, wl.d_v, dtype=torch.bfloat16, device=dev)
                     for _ in range(wl.n_layers)]
        self.pr = ic.paged_rows(self.seq, self.table, wl.T, wl.page, self.num_pages, wl.L)
        self.rows = ic.Rows(wl.B, wl.L, wl.T - wl.L, wl.T)
        self.shape = ic.StackShape(self.rows, wl.H_I, wl.d_I, DT[wl.idx_dtype], wl.k, wl.Hq,
                                   wl.d_qk, wl.d_v, DT[wl.attn_dtype], wl.d_qk, wl.d_qk, wl.scale)
        need = max(ic.paged_workspace_size(self.shape, self.pr),
                   ic.indexer_topk_paged_workspace_size(self.pr, wl.k),
                   ic.sparse_attn_paged_workspace_size(self.pr, wl.k))
        self.ws = torch.empty(need, dtype=torch.uint8, device=dev)
        ic.workspace_init(self.ws)
        self.idx = torch.empty(wl.B, wl.L, wl.k, dtype=torch.int32, device=dev)
        self.layers = self._layer_dicts(self.inputs, self.outs)
        self.ld = (wl.T + 3) // 4 * 4
        self.scores = torch.empty(wl.B, wl.L, self.ld, dtype=torch.float32, device=dev)
        # physical cache row of each sequence's newest key (the decode step's own row)
        last = (self.seq.to(torch.int64) - 1)
        self.new_rows = (self.table.to(torch.int64).gather(1, (last // wl.page)[:, None])[:, 0]
                         * wl.page + last % wl.page)

    def step(self, pattern, stream=None):
        ic.layer_stack_forward_paged(pattern, self.layers, self.shape, self.pr, self.idx, self.ws,
                                     stream=stream)

    def own_selection(self, l):
        L = self.layers[l]
        ic.indexer_topk_paged(L["q_idx"], L["w"], L["k_idx"], self.pr, self.wl.k, self.idx,
                              self.ws, q_scale=L["q_scale"], k_scale_pages=L["k_scale"],
                              dtype=DT[self.wl.idx_dtype])
        return self.idx.view(-1, self.wl.k).clone()

    def stage_step(self, pattern, ev):
        """As Stack.stage_step, through the paged calls."""
        wl = self.wl
        for l, kind in enumerate(pattern):
            L = self.layers[l]
            if kind == "F":
                e, e0, e1, e2 = ev.new(), ev.new(), ev.new(), ev.new()
                e.record()
                ic.indexer_topk_paged(L["q_idx"], L["w"], L["k_idx"], self.pr, wl.k, self.idx,
                                      self.ws, q_scale=L["q_scale"], k_scale_pages=L["k_scale"],
                                      dtype=DT[wl.idx_dtype])
                e0.record()
                ic.indexer_scores_paged(L["q_idx"], L["w"], L["k_idx"], self.pr, self.scores,
                                        self.ws, q_scale=L["q_scale"], k_scale_pages=L["k_scale"],
                                        dtype=DT[wl.idx_dtype])
                e1.record()
                ic.topk_varlen(self.scores, self.pr, wl.k, self.idx, self.ws)
                e2.record()
                ev.add("select", e, e0)
                ev.add("indexer", e0, e1)
                ev.add("topk", e1, e2)
            e3, e4 = ev.new(), ev.new()
            e3.record()
            ic.sparse_attn_paged(L["q"], L["kmat"], self.idx, self.pr, wl.scale, L["out"], self.ws)
            e4.record()
            ev.add("attention", e3, e4)


class Events:
    def __init__(self):
        self.pending = []

    def new(self):
        return torch.cuda.Event(enable_timing=True)

    def add(self, name, a, b):
        self.pending.append((name, a, b))

    def collect(self):
        torch.cuda.synchronize()
        out = {}
        for name, a, b in self.pending:
            out.setdefault(name, []).append(a.elapsed_time(b))
        self.pending = []
        return out


# ----------------------------------------------------------------------------- algorithmic work
def fused_selection(wl):
    """Whether the library runs an F layer's indexer and top-k as one fused
    kernel for this workload (decode rows on the tensor-core shapes): the
    library's own rule, restated."""
    T_max = wl.q_start + wl.L
    return (wl.L <= 2 and wl.idx_dtype in ("bf16", "e4m3") and wl.d_I == 128
            and wl.H_I in (16, 32, 64, 128) and 16 <= wl.B * wl.L <= 148 and T_max > wl.k
            and T_max >= 4096)


def path_stages(wl):
    """The stages one step runs, in the stack's path."""
    return ("select", "attention") if fused_selection(wl) else ("indexer", "topk", "attention")


def algorithmic(wl, lens=None):
    """Per-launch algorithmic work of each stage (pages' definitions, all rows).
    lens: per-sequence key counts of a variable-length batch (default: every
    sequence wl.T keys, queries from wl.q_start)."""
    if lens is None:
        rows = [wl.q_start + i for i in range(wl.L)] * wl.B       # t of every query row
        keys = wl.B * wl.T
    else:
        rows = [n - wl.L + i for n in lens for i in range(wl.L)]
        keys = sum(lens)
    pairs = sum(t + 1 for t in rows)                              # causal (query, key) pairs
    visits = sum(min(wl.k, t + 1) for t in rows)                  # selected KV rows visited
    ib = {"f32": 4, "bf16": 2, "e4m3": 1}[wl.idx_dtype]
    ab = {"f32": 4, "bf16": 2}[wl.attn_dtype]
    kv_w = wl.d_qk if wl.latent else wl.d_qk + wl.d_v
    q_side = wl.B * wl.L * wl.H_I * (wl.d_I * ib + 4)
    d = {
        "indexer_flop": 2.0 * wl.H_I * wl.d_I * pairs,
        "indexer_bytes": keys * wl.d_I * ib + q_side + 4.0 * pairs,
        "topk_bytes": 4.0 * pairs + 4.0 * wl.B * wl.L * wl.k,
        # fused selection: the indexer's reads and the indices written, no scores
        "select_bytes": keys * wl.d_I * ib + q_side
        + (keys * 4.0 if wl.idx_dtype == "e4m3" else 0.0) + 4.0 * wl.B * wl.L * wl.k,
        "attn_flop": 2.0 * wl.Hq * (wl.d_qk + wl.d_v) * visits,
        "attn_bytes": visits * kv_w * ab + wl.B * wl.L * wl.Hq * (wl.d_qk + wl.d_v) * ab
        + 4.0 * wl.B * wl.L * wl.k,
        "pairs": pairs, "visits": visits,
    }
    return d


def stage_bound(wl, work, stage):
    """(tensor-bound?, algorithmic work of one pass) of a stage: flops for the
    prefill indexer and the bf16 prefill attention (tensor cores), bytes
    otherwise (HBM)."""
    if stage == "attention":
        tensor = wl.attn_dtype == "bf16" and wl.L > 1
        return tensor, work["attn_flop"] if tensor else work["attn_bytes"]
    if stage == "indexer":
        tensor = wl.L > 1
        return tensor, work["indexer_flop"] if tensor else work["indexer_bytes"]
    if stage == "select":
        return False, work["select_bytes"]
    return False, work["topk_bytes"]


def _roof(num, per_pass_ms, tensor, fp8, peak):
    hbm, tf_burst, tf_sus, peak_src = _peaks()
    if tensor:
        p = tf_sus if peak == "sustained" else tf_burst
        if fp8:
            p *= 2.0                               # e4m3 dense peak: 2x the bf16 figure
        roof = {"bound": "tensor", "achieved": num / (per_pass_ms * 1e-3) / 1e12, "peak": p,
                "unit": "TFLOP/s"}
        roof["peak_source"] = "%s (%s %s)" % (peak_src, peak, "bf16 x2 for e4m3" if fp8 else "bf16")
    else:
        roof = {"bound": "hbm", "achieved": num / (per_pass_ms * 1e-3) / 1e9, "peak": hbm,
                "unit": "GB/s", "peak_source": "%s (copy bandwidth)" % peak_src}
    roof["frac"] = roof["achieved"] / roof["peak"]
    return roof


def stage_roofline(wl, work, stage, per_launch_ms, peak="burst", per_pass=1):
    """Roofline of one stage from its mean time per launch."""
    tensor, num = stage_bound(wl, work, stage)
    fp8 = stage == "indexer" and wl.idx_dtype == "e4m3"
    roof = _roof(num, per_launch_ms * per_pass, tensor, fp8, peak)
    roof["in_step_path"] = stage in path_stages(wl)
    roof["ms_per_launch"] = per_launch_ms
    return roof


def roofline(wl, work, total_ms, launches, per_pass=1, peak="sustained"):
    """Roofline line of the dominant stage.  total_ms / launches: summed
    event time and launch count per stage over the measured passes; work:
    algorithmic work of one pass of a stage over all rows (``algorithmic``;
    summed over the chunks of a chunked run), which takes ``per_pass``
    launches.  ``peak``: "burst" or "sustained" bf16 figure."""
    dom = max((k for k in total_ms if k in path_stages(wl)), key=lambda k: total_ms[k])
    passes = launches[dom] / per_pass
    per_pass_ms = total_ms[dom] / passes
    tensor, num = stage_bound(wl, work, dom)
    fp8 = dom == "indexer" and wl.idx_dtype == "e4m3"
    roof = _roof(num, per_pass_ms, tensor, fp8, peak)
    roof["kernel"] = dom
    roof["ms_per_launch"] = total_ms[dom] / launches[dom]
    return roof, dom


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index),
                 "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = max(mx, float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        load = [s for s in sm if s > 0.5 * mx] or sm
        return {"sm_mhz": float(np.median(load)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- oracle baseline
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return len(os.sched_getaffinity(0))


def oracle_layers(wl, pattern):
    """The layers the oracle sample runs: all of them, except for long decode
    caches, where the first F group (4 layers) is timed and the rate scaled
    by the share of layers it holds, so host memory stays bounded."""
    if wl.L == 1 and wl.T * len(pattern) > 2_000_000:
        return pattern[:4]
    return pattern


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baseline(wl, pattern, value, done, spent, how, clock=None):
    """The cpu_baseline object: the float64 oracle's rate on a bounded
    sample (`how` says how the query rows were drawn), and with `clock` its
    time per query row in each stage (per F layer for the indexer and
    top-k, per layer for attention) at the sampled rows' positions."""
    lay = oracle_layers(wl, pattern)
    if lay == pattern:
        layers, note = "all %d layers of %s" % (len(pattern), pattern), ""
    else:
        layers = "the first %d of the %d layers of %s" % (len(lay), len(pattern), pattern)
        note = "; rate scaled to all layers"
    res = {"value": value, "unit": "tok/s", "cores": _blas_threads(), "kind": "oracle",
           "cpu_model": cpu_model(),
           "sample": "%d %s of %s through %s (float64 NumPy, %.1f s of oracle time%s)"
                     % (done, how, wl.name, layers, spent, note)}
    if clock is not None:
        res["per_row_ms"] = clock.per_row_ms()
    return res


class OracleStageClock:
    """Adds up the time the oracle spends in each stage function while its
    layer_stack runs, and the query rows each stage handled.  The module's
    functions are wrapped for the duration of the `with` block and restored
    afterwards; the oracle's arithmetic is untouched."""
    STAGES = {"indexer": "indexer_scores", "topk": "topk_indices", "attention": "sparse_attention"}

    def __init__(self):
        import oracle.indexcache_oracle as om
        self.mod = om
        self.seconds = dict.fromkeys(self.STAGES, 0.0)
        self.rows = dict.fromkeys(self.STAGES, 0)

    def __enter__(self):
        self.saved = {st: getattr(self.mod, fn) for st, fn in self.STAGES.items()}
        for st, fn in self.STAGES.items():
            setattr(self.mod, fn, self._timed(st, self.saved[st]))
        return self

    def __exit__(self, *exc):
        for st, fn in self.STAGES.items():
            setattr(self.mod, fn, self.saved[st])
        return False

    def _timed(self, stage, fn):
        def run(*args, **kw):
            t0 = time.perf_counter()
            res = fn(*args, **kw)
            self.seconds[stage] += time.perf_counter() - t0
            self.rows[stage] += res.shape[0] * res.shape[1]      # [B, rows, ...]
            return res
        return run

    def per_row_ms(self):
        return {st: (1e3 * self.seconds[st] / self.rows[st] if self.rows[st] else None)
                for st in self.STAGES}


def oracle_sample(wl, pattern, budget_s, clock=None):
    """Time the float64 oracle (as it stands) on a bounded sample of the
    workload: prefill -> blocks of consecutive query rows at random offsets of
    one sequence; decode -> whole sequences, one at a time.  Inputs are drawn
    on the CPU with the workload's shapes and distributions (the sample's
    values differ from the GPU run's, its cost per row does not).  Grows the
    sample until about budget_s seconds of oracle time.  Returns (rows per
    second, rows done, seconds)."""
    import dataclasses
    import oracle
    if wl.page:
        # a paged batch: the oracle reads plain per-sequence arrays; sample
        # sequences of the batch's mean length
        mean = (wl.len_min + wl.T) // 2
        wl = dataclasses.replace(wl, T=mean, q_start=mean - wl.L, page=0, len_min=0)
    rng = np.random.default_rng(0)
    done, spent, n = 0, 0.0, 1
    sub_pattern = oracle_layers(wl, pattern)
    layer_share = len(sub_pattern) / len(pattern)
    dec_inputs = None
    while spent < budget_s:
        if wl.L > 1:
            n = min(n, wl.L)
            r0 = int(rng.integers(0, wl.L - n + 1))
            # rows r0..r0+n-1 of one sequence against their causal prefix
            sub = dataclasses.replace(wl, B=1, L=n, q_start=wl.q_start + r0,
                                      T=wl.q_start + r0 + n, chunk=0)
            inputs = _oracle_inputs(sub)
        else:
            # one sequence, drawn once and timed repeatedly (drawing it costs
            # more than the oracle pass; the cost per pass does not change)
            if dec_inputs is None:
                sub = dataclasses.replace(wl, B=1, seed=wl.seed + int(rng.integers(1 << 20)),
                                          pattern=sub_pattern)
                dec_inputs = _oracle_inputs(sub)
            inputs = dec_inputs
        t0 = time.perf_counter()
        if clock is None:
            oracle.layer_stack(sub.pattern, inputs, sub.q_start, sub.k, sub.scale,
                               fp8=sub.idx_dtype == "e4m3")
        else:
            with clock:
                oracle.layer_stack(sub.pattern, inputs, sub.q_start, sub.k, sub.scale,
                                   fp8=sub.idx_dtype == "e4m3")
        dt = time.perf_counter() - t0
        done += sub.B * sub.L
        spent += dt
        if wl.L > 1:
            # a row's cost grows with its causal length: plan the next block
            # (at most half the remaining budget) from the cost per row at the
            # longest prefix the next draw can have
            per_row_max = dt / n * (wl.q_start + wl.L) / max(1, sub.T)
            n = max(1, min(256, int(0.5 * (budget_s - spent) / max(per_row_max, 1e-6))))
    return done / spent * layer_share, done, spent


def _oracle_inputs(wl):
    res = []
    for l in range(wl.n_layers):
        inp = synth.layer_inputs(wl, l, "cpu")
        d = {}
        for key in ("q_I", "w", "k_I", "q_scale", "k_scale", "q"):
            if key in inp:
                t = inp[key]
                d[key] = t.numpy() if t.dtype == torch.uint8 else t.double().numpy()
        if wl.latent:
            kv = inp["kv"].double().numpy()
            d["K"], d["V"] = kv, kv[..., : wl.d_v]
        else:
            d["K"], d["V"] = inp["k"].double().numpy(), inp["v"].double().numpy()
        res.append(d)
    return res


# ----------------------------------------------------------------------------- main
DEFAULT_DECODE = (("decode_b32_t32k_bf16", 500), ("decode_b8_t200k_fp8", 150),
                  ("decode_b32_varlen_paged_bf16", 500))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="prefill_8k_bf16")
    ap.add_argument("--pattern", default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true",
                    help="time only --workload (the default run also times the decode workloads)")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--graph", action="store_true",
                    help="replay each step as a captured CUDA graph (decode: removes launch gaps)")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    wl = synth.WORKLOADS[args.workload]
    pattern = args.pattern or wl.pattern

    if args.impl == "reference":
        return run_reference(args, wl, pattern, rank, world)

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    if wl.chunk:
        return run_chunked(args, wl, pattern, dev, pg, rank, world)
    line = measure_stack(wl, pattern, dev, pg, rank, world, steps=args.steps,
                         warmup=args.warmup, graph=args.graph or wl.L == 1,
                         e2e=not args.no_e2e,
                         cpu_budget=None if args.no_cpu_baseline else args.cpu_budget)
    # the default run: the decode half of the metric (decode step us, IndexCache
    # pattern vs all-F) on the two decode workloads, CUDA-graph replay
    if args.workload == "prefill_8k_bf16" and args.pattern is None and not args.no_decode:
        line["decode"] = {}
        for name, dsteps in DEFAULT_DECODE:
            dwl = synth.WORKLOADS[name]
            entry = measure_stack(dwl, dwl.pattern, dev, pg, rank, world,
                                  steps=max(args.steps, dsteps), warmup=args.warmup, graph=True,
                                  e2e=not args.no_e2e,
                                  cpu_budget=None if args.no_cpu_baseline else args.cpu_budget / 2)
            line["decode"][name] = decode_entry(entry)
        # the FP8 prefill indexer (e4m3 operands, per-token scales) on the
        # same 8K prefill: its indexer stage against the e4m3 tensor peak
        fwl = synth.WORKLOADS["prefill_8k_fp8"]
        entry = measure_stack(fwl, fwl.pattern, dev, pg, rank, world, steps=args.steps,
                              warmup=args.warmup, graph=False, e2e=False,
                              cpu_budget=None if args.no_cpu_baseline else args.cpu_budget / 3)
        line["prefill_fp8"] = {
            "metric": "prefill tok/s (IndexCache pattern) with the FP8 indexer",
            "value": entry["value"], "unit": entry["unit"], "ms_per_step": entry["ms_per_step"],
            "all_f": entry["all_f"], "config": entry["config"], "stages_ms": entry["stages_ms"],
            "indexer_roofline": entry["roofline_by_stage"]["indexer"],
            "roofline_by_stage": entry["roofline_by_stage"],
            "cpu_baseline": entry["cpu_baseline"], "gpu_launches": entry["gpu_launches"],
            "clocks": entry["clocks"], "device_status": entry["device_status"]}
    if rank == 0:
        print(json.dumps(line), flush=True)
    _finish(pg)


def decode_entry(line):
    """The decode workload's measurement as an entry of the default line:
    step time in microseconds for the IndexCache pattern and for all-F."""
    return {
        "metric": "decode step us (IndexCache pattern) vs all-F",
        "step_us": line["ms_per_step"] * 1e3,
        "all_f_step_us": line["all_f"]["ms_per_step"] * 1e3,
        "speedup_of_pattern": line["all_f"]["speedup_of_pattern"],
        "value": line["value"], "unit": line["unit"], "steps": line["steps"],
        "config": line["config"], "stages_us": {
            k: {"per_launch": v["per_launch"] * 1e3, "launches_per_step": v["launches_per_step"]}
            for k, v in line["stages_ms"].items()},
        "roofline_by_stage": line["roofline_by_stage"],
        "indexer_share_of_step": line["indexer_share_of_step"],
        "topk_overlap_matrix": line["topk_overlap_matrix"],
        "cpu_baseline": line["cpu_baseline"], "e2e": line["e2e"],
        "gpu_launches": line["gpu_launches"], "cuda_graph": line["cuda_graph"],
        "clocks": line["clocks"], "device_status": line["device_status"],
    }


def require_clean(ws, what):
    """Read (and clear) the device status word of a workspace after a timed
    region; a kernel that flagged an index error or gave up a bounded wait
    voids the measurement."""
    bits = ic.read_status(ws)
    if bits:
        raise SystemExit("%s: device status bits %d set (1 = index out of range, "
                         "2 = wait timeout); the measurement is void" % (what, bits))
    return bits


def peak_kind(clk):
    """The bf16 peak to divide by: the sustained (power-capped) figure when
    the run itself was power-capped or ran well below its maximum clock,
    else the burst figure."""
    if clk and ("sw_power_cap" in clk["reasons"] or clk["sm_mhz"] < 0.9 * clk["sm_max_mhz"]):
        return "sustained"
    return "burst"


def measure_stack(wl, pattern, dev, pg, rank, world, *, steps, warmup, graph, e2e, cpu_budget):
    """Time one workload's layer stack (IndexCache pattern and all-F) and
    return its JSON line (as a dict)."""
    import gc
    tokens_per_step = wl.B * wl.L
    st = (PagedStack if wl.page else Stack)(wl, dev, rank)
    all_f = "F" * len(pattern)

    def timed(fn, n):
        if pg:
            pg.barrier()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(n):
            fn()
        b.record()
        torch.cuda.synchronize()
        return max_over_ranks(a.elapsed_time(b), pg, dev)

    for _ in range(max(3, warmup)):
        st.step(pattern)
        st.step(all_f)
    torch.cuda.synchronize()
    require_clean(st.ws, "%s warm-up" % wl.name)
    step_fn, step_all_f = (lambda: st.step(pattern)), (lambda: st.step(all_f))
    graphs = []
    if graph:
        for pat in (pattern, all_f):
            g = torch.cuda.CUDAGraph()
            s_cap = torch.cuda.Stream()
            s_cap.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(s_cap):
                st.step(pat)                     # warm the capture stream
                torch.cuda.synchronize()
                with torch.cuda.graph(g, stream=s_cap):
                    st.step(pat, stream=s_cap)
            torch.cuda.current_stream().wait_stream(s_cap)
            graphs.append(g)
        step_fn, step_all_f = graphs[0].replay, graphs[1].replay
        for _ in range(3):
            step_fn()
            step_all_f()
        torch.cuda.synchronize()

    # main timed region: the IndexCache pattern through the C ABI
    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    n0 = ic.kernel_launches(0)
    ms = timed(step_fn, steps)
    launches = ic.kernel_launches(0) - n0
    if graph:   # replays launch the captured kernels: count them per step
        torch.cuda.synchronize()
        n1 = ic.kernel_launches(0)
        st.step(pattern)
        launches = (ic.kernel_launches(0) - n1) * steps
        torch.cuda.synchronize()
    status = require_clean(st.ws, "%s IndexCache steps" % wl.name)
    ms_all_f = timed(step_all_f, steps)
    clk = clocks.stop()
    require_clean(st.ws, "%s all-F steps" % wl.name)
    del graphs, step_fn, step_all_f

    # stage breakdown (same kernels as separate calls, events on the launch stream);
    # one untimed pass first: the reference stages that the step's path does
    # not use (decode's stand-alone indexer and top-k) make their first calls
    # there, with the library's one-time host-side launch planning
    ev = Events()
    st.stage_step(pattern, ev)
    ev.collect()
    stage_passes = min(steps, 20)
    for _ in range(stage_passes):
        st.stage_step(pattern, ev)
    stages = ev.collect()
    require_clean(st.ws, "%s stage pass" % wl.name)

    # end to end from pinned host buffers through the public API
    e2e_line = None
    if e2e:
        e2e_line = run_e2e(st, pattern, min(steps, 50 if wl.L == 1 else steps), dev, pg)
        require_clean(st.ws, "%s e2e" % wl.name)

    # untimed: every layer's own top-k (each running its own indexer) and the
    # all-pairs layer overlap matrix a pattern search would consume
    own = [st.own_selection(l) for l in range(len(pattern))]
    s_sum, s_min, n_rows = overlap_matrix(own, wl.T)
    overlap = overlap_json(s_sum, s_min, n_rows, "%s, all %d layers, %d query rows"
                           % (wl.name, len(pattern), n_rows))
    del own
    require_clean(st.ws, "%s overlap pass" % wl.name)

    per_step_ms = ms / steps
    value = whole_job_rate(tokens_per_step, world, per_step_ms)
    lens = getattr(st, "lens", None)
    work = algorithmic(wl, lens)
    avg = {k: float(np.mean(v)) for k, v in stages.items()}
    kind = peak_kind(clk)
    totals = {k: sum(v) for k, v in stages.items()}
    counts = {k: len(v) for k, v in stages.items()}
    roof, dom = roofline(wl, work, totals, counts, peak=kind)
    roof["traffic"] = _traffic(dom, wl.name)
    by_stage = {k: stage_roofline(wl, work, k, avg[k], kind) for k in stages}
    # share of the step spent choosing keys (the selection stages of the path)
    path = path_stages(wl)
    total_stage = sum(totals[k] for k in path if k in totals)
    sel_share = sum(totals.get(k, 0.0) for k in path if k != "attention") / total_stage
    bytes_in = st.bytes_per_step(pattern)
    paged_cfg = ({"page_size": wl.page, "num_pages": st.num_pages, "seq_len_min": min(lens),
                  "seq_len_mean": sum(lens) / len(lens), "seq_len_max": max(lens)}
                 if wl.page else None)
    del st
    gc.collect()
    torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and cpu_budget:
        clock = OracleStageClock()
        rps, done, spent = oracle_sample(wl, pattern, cpu_budget, clock)
        cpu = cpu_baseline(wl, pattern, rps, done, spent,
                           "query rows" if wl.L > 1 else "single-sequence decode steps", clock)
    return {
        "metric": "prefill tok/s (IndexCache pattern) with all-F comparison; roofline of the "
                  "dominant kernel" if wl.L > 1 else "decode tok/s (IndexCache pattern)",
        "value": value, "unit": "tok/s", "n_gpus": world, "steps": steps,
        "warmup": max(3, warmup), "ms_per_step": per_step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.attn_dtype, "data": "synthetic",
        "config": {"workload": wl.name, "pattern": pattern, "B": wl.B, "L": wl.L, "T": wl.T,
                   "H_I": wl.H_I, "d_I": wl.d_I, "k": wl.k, "Hq": wl.Hq, "d_qk": wl.d_qk,
                   "d_v": wl.d_v, "indexer_dtype": wl.idx_dtype,
                   "parallelism": "replicas x%d" % world,
                   "l2": "inputs larger than L2 (%.2f GB read per step)" % (bytes_in / 1e9),
                   **({"paged": paged_cfg} if paged_cfg else {})},
        "all_f": {"pattern": all_f, "ms_per_step": ms_all_f / steps,
                  "value": tokens_per_step * world / (ms_all_f / steps / 1e3),
                  "speedup_of_pattern": ms_all_f / ms},
        "stages_ms": {k: {"per_launch": avg[k], "launches_per_step": len(v) / stage_passes}
                      for k, v in stages.items()},
        "indexer_share_of_step": sel_share,
        "roofline": roof,
        "roofline_by_stage": by_stage,
        "topk_overlap_matrix": overlap,
        "cpu_baseline": cpu,
        "e2e": e2e_line,
        "gpu_launches": launches,
        "cuda_graph": bool(graph),
        "clocks": clk,
        "device_status": status,
    }


def row_overlap(reused, own, T):
    """Per row, |own & reused| / |reused| of two [rows, k] index sets whose
    entries lie in [0, T) or are -1 padding (ignored): the top-k overlap the
    chunked run reports for S layers.  Runs on the tensors' device."""
    rows, k = reused.shape
    off = (torch.arange(rows, device=reused.device, dtype=torch.int64) * (T + 1))[:, None]
    a = reused.to(torch.int64)
    b = own.to(torch.int64)
    a = torch.where(a >= 0, a + off, torch.full_like(a, -1))
    b = torch.where(b >= 0, b + off, torch.full_like(b, -2))
    hit = torch.isin(b.flatten(), a.flatten()).view(rows, k).sum(1).to(torch.float64)
    return hit / (reused >= 0).sum(1).clamp(min=1).to(torch.float64)


def overlap_matrix(sets, T):
    """All-pairs top-k overlap of per-layer index sets: sets[l] is an [rows,
    k] tensor of layer l's own top-k (ascending positions in [0, T), -1
    padding last).  Entry (l, m) is, per row, |A_l & A_m| / |A_l| (the
    oracle's topk_overlap), returned as (sum over rows, min over rows, rows)
    so that calls over several chunks can be merged.  Runs on the sets'
    device: each row of A_m is searched for the entries of A_l."""
    L = len(sets)
    rows = sets[0].shape[0]
    big = torch.iinfo(torch.int32).max
    sorted_sets = []
    sizes = []
    for a in sets:
        a = a.to(torch.int64)
        sizes.append((a >= 0).sum(1).clamp(min=1).to(torch.float64))
        sorted_sets.append(torch.where(a >= 0, a, torch.full_like(a, big)))   # padding sorts last
    s_sum = torch.zeros(L, L, dtype=torch.float64)
    s_min = torch.ones(L, L, dtype=torch.float64)
    for l in range(L):
        a = sets[l].to(torch.int64)
        for m in range(L):
            b = sorted_sets[m]
            pos = torch.searchsorted(b, a.contiguous()).clamp(max=b.shape[1] - 1)
            hit = ((b.gather(1, pos) == a) & (a >= 0)).sum(1).to(torch.float64)
            frac = hit / sizes[l]
            s_sum[l, m] = float(frac.sum())
            s_min[l, m] = float(frac.min())
    return s_sum, s_min, rows


def overlap_json(s_sum, s_min, rows, what):
    L = s_sum.shape[0]
    return {"layers": L, "rows": rows, "of": what,
            "definition": "per row |A_l & A_m| / |A_l| of layer l's and layer m's own top-k "
                          "(each layer running its own indexer), mean and minimum over rows",
            "mean": [[round(float(s_sum[l, m]) / rows, 4) for m in range(L)] for l in range(L)],
            "min": [[round(float(s_min[l, m]), 4) for m in range(L)] for l in range(L)]}


def run_chunked(args, wl, pattern, dev, pg, rank, world):
    """Chunked prefill: the sequence's L query rows go through the layer stack
    in chunks of wl.chunk rows, chunk c against its causal prefix (q_start =
    c*chunk, T = (c+1)*chunk), the index cache living per chunk.  One step =
    every chunk through every layer.  All per-(layer, chunk) queries and all
    layers' keys stay resident on the device.  After timing, an untimed pass
    runs every S layer's own indexer and top-k and reports the overlap of its
    own selection with the reused one (per row: |own & reused| / min(k, t+1)),
    mean and minimum over all rows, per S layer."""
    import dataclasses
    C, nch, nl = wl.chunk, wl.L // wl.chunk, len(pattern)
    all_f = "F" * nl
    shared_q = bool(wl.kI_noise)              # indexer queries shared by all layers
    need = (nl * nch * C * wl.Hq * wl.d_qk * 2 + nl * wl.T * (wl.d_qk + wl.d_I) * 2
            + (1 if shared_q else nl) * nch * C * wl.H_I * (wl.d_I * 2 + 4)
            + nl * C * wl.Hq * wl.d_v * 2 + C * wl.T * 4)
    free = torch.cuda.mem_get_info(dev)[0]
    if need > 0.95 * free:
        raise SystemExit("chunked workload needs %.1f GB on the device, %.1f GB free"
                         % (need / 1e9, free / 1e9))
    outs = [torch.empty(1, C, wl.Hq, wl.d_v, dtype=torch.bfloat16, device=dev) for _ in range(nl)]
    idx_buf = torch.empty(1, C, wl.k, dtype=torch.int32, device=dev)
    shapes, rows = [], []
    for c in range(nch):
        r = ic.Rows(1, C, c * C, (c + 1) * C)
        rows.append(r)
        shapes.append(ic.StackShape(r, wl.H_I, wl.d_I, DT[wl.idx_dtype], wl.k, wl.Hq, wl.d_qk,
                                    wl.d_v, DT[wl.attn_dtype], wl.d_qk, wl.d_qk, wl.scale))
    ws = torch.empty(ic.workspace_size(shapes[-1]), dtype=torch.uint8, device=dev)
    ic.workspace_init(ws)
    ld = (wl.T + 3) // 4 * 4
    scores = torch.empty(1, C, ld, dtype=torch.float32, device=dev)
    t_start = time.time()

    def progress(msg):
        print("[chunked %6.1f s] %s" % (time.time() - t_start, msg), file=sys.stderr, flush=True)

    keys, qs, qI, wI = [], [], {}, {}
    for l in range(nl):
        inp = synth.layer_inputs(wl, l, dev, chunk=0)
        keys.append((inp["k_I"], inp["kv"]))
        ql = [inp["q"]]
        if l == 0 or not shared_q:
            qI[(l, 0)], wI[(l, 0)] = inp["q_I"], inp["w"]
        if l == 0:
            # load every kernel of the stack (and its code on the device) before
            # the bulk of the inputs fills the memory
            ic.layer_stack_forward("F", [dict(q_idx=inp["q_I"], w=inp["w"], k_idx=inp["k_I"],
                                              q=inp["q"], kmat=inp["kv"], vmat=inp["kv"],
                                              out=outs[0])], shapes[0], idx_buf, ws)
            torch.cuda.synchronize()
        del inp
        for c in range(1, nch):
            d = synth.chunk_queries(wl, l, c, dev, indexer=(l == 0 or not shared_q))
            ql.append(d["q"])
            if "q_I" in d:
                qI[(l, c)], wI[(l, c)] = d["q_I"], d["w"]
            del d
        qs.append(ql)
        torch.cuda.empty_cache()   # float32 temporaries of the generator
    qkey = (lambda l, c: (0, c)) if shared_q else (lambda l, c: (l, c))
    progress("inputs resident (%.1f GB)" % (need / 1e9))

    def layer_dicts(pat, c):
        res = []
        for l, kind in enumerate(pat):
            kI, kv = keys[l]
            d = dict(q=qs[l][c], kmat=kv, vmat=kv, out=outs[l])
            if kind == "F":
                d.update(q_idx=qI[qkey(l, c)], w=wI[qkey(l, c)], k_idx=kI)
            res.append(d)
        return res

    calls = {p: [layer_dicts(p, c) for c in range(nch)] for p in (pattern, all_f)}

    def step(pat):
        for c in range(nch):
            ic.layer_stack_forward(pat, calls[pat][c], shapes[c], idx_buf, ws)

    def timed(fn, steps):
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            fn()
        b.record()
        torch.cuda.synchronize()
        return max_over_ranks(a.elapsed_time(b), pg, dev)

    for _ in range(max(3, args.warmup)):
        step(pattern)
        step(all_f)
    progress("warm-up done")
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    clocks.start()
    n0 = ic.kernel_launches(0)
    ms = timed(lambda: step(pattern), args.steps)
    launches = ic.kernel_launches(0) - n0
    ms_all_f = timed(lambda: step(all_f), args.steps)
    clk = clocks.stop()

    # stage breakdown: the same kernels as separate calls, events around each
    ev = Events()
    for c in range(nch):
        r = rows[c]
        for l, kind in enumerate(pattern):
            kI, kv = keys[l]
            if kind == "F":
                e0, e1, e2 = ev.new(), ev.new(), ev.new()
                e0.record()
                ic.indexer_scores(qI[qkey(l, c)], wI[qkey(l, c)], kI, r, scores, ws,
                                  dtype=DT[wl.idx_dtype])
                e1.record()
                ic.topk(scores, r, wl.k, idx_buf, ws)
                e2.record()
                ev.add("indexer", e0, e1)
                ev.add("topk", e1, e2)
            e3, e4 = ev.new(), ev.new()
            e3.record()
            ic.sparse_attn(qs[l][c], kv, wl.d_qk, kv, wl.d_qk, idx_buf, r, wl.d_v, wl.scale,
                           outs[l], ws, dtype=DT[wl.attn_dtype])
            e4.record()
            ev.add("attention", e3, e4)
    stages = ev.collect()
    progress("timed steps and stage pass done")

    # algorithmic work of one layer pass over all chunks
    work = {}
    for c in range(nch):
        sub = dataclasses.replace(wl, L=C, q_start=c * C, T=(c + 1) * C, chunk=0)
        for k, v in algorithmic(sub).items():
            work[k] = work.get(k, 0.0) + v
    roof, dom = roofline(wl, work, {k: sum(v) for k, v in stages.items()},
                         {k: len(v) for k, v in stages.items()}, per_pass=nch)
    roof["traffic"] = _traffic(dom, args.workload)

    # untimed: every layer's own top-k per chunk; the top-k overlap of each S
    # layer's own selection with the reused one, and the all-pairs layer
    # overlap matrix over every row of every chunk
    own = [torch.empty(C, wl.k, dtype=torch.int32, device=dev) for _ in range(nl)]
    acc = {}
    m_sum = torch.zeros(nl, nl, dtype=torch.float64)
    m_min = torch.ones(nl, nl, dtype=torch.float64)
    for c in range(nch):
        r = rows[c]
        reused = None
        for l, kind in enumerate(pattern):
            kI = keys[l][0]
            ic.indexer_scores(qI[qkey(l, c)], wI[qkey(l, c)], kI, r, scores, ws,
                              dtype=DT[wl.idx_dtype])
            ic.topk(scores, r, wl.k, own[l].view(1, C, wl.k), ws)
            if kind == "F":
                reused = own[l]
                continue
            frac = row_overlap(reused, own[l], wl.T)
            s_, n_, mn = acc.get(l, (0.0, 0, 1.0))
            acc[l] = (s_ + float(frac.sum()), n_ + C, min(mn, float(frac.min())))
        s_sum, s_min, _ = overlap_matrix(own, wl.T)
        m_sum += s_sum
        m_min = torch.minimum(m_min, s_min)
    overlap = {"layer_%d" % l: {"mean": v[0] / v[1], "min": v[2]} for l, v in sorted(acc.items())}
    overlap_all = overlap_json(m_sum, m_min, nch * C, "%s, all %d layers, every row of the %d "
                               "chunks" % (wl.name, nl, nch))
    del own
    torch.cuda.synchronize()
    progress("overlap pass done")

    if rank != 0:
        _finish(pg)
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        clock = OracleStageClock()
        rps, done, spent = oracle_sample(wl, pattern, args.cpu_budget, clock)
        cpu = cpu_baseline(wl, pattern, rps, done, spent, "query rows at random positions",
                           clock)
    per_step_ms = ms / args.steps
    avg = {k: float(np.mean(v)) for k, v in stages.items()}
    line = {
        "metric": "chunked prefill tok/s (IndexCache pattern) with all-F comparison; roofline of "
                  "the dominant kernel; top-k overlap of S layers",
        "value": wl.B * wl.L * world / (per_step_ms / 1e3), "unit": "tok/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": per_step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": wl.attn_dtype,
        "data": "synthetic",
        "config": {"workload": wl.name, "pattern": pattern, "B": wl.B, "L": wl.L, "chunk": C,
                   "T": wl.T, "H_I": wl.H_I, "d_I": wl.d_I, "k": wl.k, "Hq": wl.Hq,
                   "d_qk": wl.d_qk, "d_v": wl.d_v, "indexer_dtype": wl.idx_dtype,
                   "k_I_per_layer": "base + %.1f x noise at the base's scale" % wl.kI_noise,
                   "parallelism": "replicas x%d" % world,
                   "l2": "inputs larger than L2 (%.1f GB resident)" % (need / 1e9)},
        "all_f": {"pattern": all_f, "ms_per_step": ms_all_f / args.steps,
                  "value": wl.B * wl.L * world / (ms_all_f / args.steps / 1e3),
                  "speedup_of_pattern": ms_all_f / ms},
        "stages_ms": {k: {"per_launch": avg[k], "launches_per_step": len(v)}
                      for k, v in stages.items()},
        "topk_overlap_s_layers": overlap,
        "topk_overlap_matrix": overlap_all,
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": None,
        "e2e_note": "not measured for this workload: one step reads %.0f GB of query inputs"
                    % (need / 1e9),
        "gpu_launches": launches,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    _finish(pg)


def _traffic(kernel, workload):
    """DRAM bytes per launch of the kernel from the committed ncu summary of
    the current kernels (profiles/traffic.json), else None."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            return json.load(f).get(workload, {}).get(kernel)
    except Exception:
        return None


CACHE_KEYS = ("kv", "k", "v", "k_I", "k_scale")


def run_e2e(st, pattern, steps, dev, pg):
    """Same metric through the public API from pinned host buffers: every step
    copies that step's inputs host->device, runs the stack through
    ic_layer_stack_forward (ic_layer_stack_forward_paged for a paged batch)
    and copies EVERY layer's output back to pinned
    host memory (each layer is an independent synthetic layer, so all of
    them are the step's result).  Prefill copies every input of the step.
    Decode keeps the KV / K_I caches resident on the device (serving state)
    and copies the new token's queries, weights and its own cache rows
    (position T-1, or each sequence's newest row in its pages).  The copies
    are torch copy_ / index_copy_ calls on the launch stream
    around the C-ABI call."""
    wl = st.wl
    decode = wl.L == 1
    paged = hasattr(st, "new_rows")
    host = []
    h2d = 0
    stage = {}
    for l, kind in enumerate(pattern):
        d = {}
        for key, t in st.inputs[l].items():
            if kind == "S" and key in ("q_I", "w", "k_I", "q_scale", "k_scale"):
                continue
            if decode and key in CACHE_KEYS:
                # the step's own cache rows: position T-1 (dense) or each
                # sequence's newest row in its pages (paged)
                src = t.index_select(0, st.new_rows) if paged else t[:, wl.T - 1]
                if paged:
                    stage[(l, key)] = torch.empty_like(src)
            else:
                src = t
            d[key] = torch.empty(src.shape, dtype=src.dtype, pin_memory=True)
            d[key].copy_(src)
            h2d += src.numel() * src.element_size()
        host.append(d)
    outs_host = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in st.outs]
    d2h = sum(o.numel() * o.element_size() for o in outs_host)

    def step():
        for l, d in enumerate(host):
            for key, t in d.items():
                if decode and key in CACHE_KEYS and paged:
                    tmp = stage[(l, key)]
                    tmp.copy_(t, non_blocking=True)
                    st.inputs[l][key].index_copy_(0, st.new_rows, tmp)
                elif decode and key in CACHE_KEYS:
                    st.inputs[l][key][:, wl.T - 1].copy_(t, non_blocking=True)
                else:
                    st.inputs[l][key].copy_(t, non_blocking=True)
        st.step(pattern)
        for o_h, o in zip(outs_host, st.outs):
            o_h.copy_(o, non_blocking=True)

    step()
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        step()
    b.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), pg, dev)
    world = pg.get_world_size() if pg else 1
    del host, outs_host
    return {"value": wl.B * wl.L * world / (ms / steps / 1e3), "unit": "tok/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "copies": "torch copy_ from/to pinned host memory on the launch stream, around "
                      "ic_layer_stack_forward; every layer's output is read back"}


def run_reference(args, wl, pattern, rank, world):
    if rank != 0:
        return
    budget = max(2.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(wl, pattern, budget / 4)
    rates, done_all, spent_all = [], 0, 0.0
    clock = OracleStageClock()
    for _ in range(args.steps):
        rps, done, spent = oracle_sample(wl, pattern, budget, clock)
        rates.append(rps)
        done_all += done
        spent_all += spent
    value = done_all / spent_all
    line = {
        "impl": "reference",
        "metric": "prefill tok/s (IndexCache pattern) with all-F comparison; roofline of the "
                  "dominant kernel" if wl.L > 1 else "decode tok/s (IndexCache pattern)",
        "value": value, "unit": "tok/s", "n_gpus": world, "steps": args.steps,
        # a reference step is one bounded sample of the workload (its rows are
        # timed, not the whole step's); ms_per_step is that sample's wall time
        "warmup": args.warmup, "ms_per_step": 1e3 * spent_all / max(1, args.steps),
        "ms_per_full_step_extrapolated": 1e3 * wl.B * wl.L / value,
        "step_definition": "one bounded oracle sample of the workload per step; the full "
                           "step's time is extrapolated from the sampled rows' rate",
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "pattern": pattern, "B": wl.B, "L": wl.L, "T": wl.T,
                   "k": wl.k},
        "cpu_baseline": cpu_baseline(wl, pattern, value, done_all, spent_all,
                                     "query rows" if wl.L > 1 else "single-sequence decode steps",
                                     clock),
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _finish(pg):
    if pg:
        pg.barrier()
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
