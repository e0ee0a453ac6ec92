"""Run one stage of the hot path on a small slice of a workload, for profilers.

    python profile_case.py --stage attention --workload prefill_8k_bf16 \
        --rows 512 --launches 3

Builds the inputs of layer 0 of the workload on cuda:0, keeps the last
``--rows`` query rows of each sequence (the heaviest rows of a prefill), runs
the stage once untimed, then ``--launches`` more times, and prints the mean
CUDA-event time per launch.  Inputs stay a few hundred MB at most, so an
``ncu --set full`` capture of one launch ends in about a minute.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import cross_layer_top_full_b200 as ic  # noqa: E402
from cross_layer_top_full_b200 import synth  # noqa: E402

DT = {"f32": ic.F32, "bf16": ic.BF16, "e4m3": ic.FP8_E4M3}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--stage", choices=["indexer", "topk", "select", "attention"], required=True)
    ap.add_argument("--workload", default="prefill_8k_bf16")
    ap.add_argument("--rows", type=int, default=512, help="query rows kept per sequence")
    ap.add_argument("--batch", type=int, default=0, help="sequences kept (0 = all)")
    ap.add_argument("--launches", type=int, default=3)
    args = ap.parse_args()

    wl = synth.WORKLOADS[args.workload]
    B = args.batch or wl.B
    wl = dataclasses.replace(wl, B=B)
    dev = torch.device("cuda:0")
    inp = synth.layer_inputs(wl, 0, dev)
    rows = min(args.rows, wl.L)
    r0 = wl.L - rows
    q_start = wl.q_start + r0
    for key in ("q_I", "w", "q", "q_scale"):
        if key in inp:
            inp[key] = inp[key][:, r0:].contiguous()
    R = ic.Rows(B, rows, q_start, wl.T)
    ld = (wl.T + 3) // 4 * 4
    scores = torch.empty(B, rows, ld, device=dev)
    idx = torch.empty(B, rows, wl.k, dtype=torch.int32, device=dev)
    kmat = inp["kv"] if wl.latent else inp["k"]
    vmat = inp["kv"] if wl.latent else inp["v"]
    ws = torch.empty(max(ic.sparse_attn_workspace_size(R, wl.k, wl.Hq, wl.d_qk, wl.d_v,
                                                       DT[wl.attn_dtype]),
                         ic.indexer_topk_workspace_size(R, wl.H_I, wl.d_I, DT[wl.idx_dtype], wl.k),
                         1 << 16),
                     dtype=torch.uint8, device=dev)
    ic.workspace_init(ws)
    out = torch.empty(B, rows, wl.Hq, wl.d_v, device=dev,
                      dtype=torch.bfloat16 if wl.attn_dtype == "bf16" else torch.float32)

    def indexer():
        ic.indexer_scores(inp["q_I"], inp["w"], inp["k_I"], R, scores, ws,
                          q_scale=inp.get("q_scale"), k_scale=inp.get("k_scale"),
                          dtype=DT[wl.idx_dtype])

    def topk():
        ic.topk(scores, R, wl.k, idx, ws)

    def select():
        ic.indexer_topk(inp["q_I"], inp["w"], inp["k_I"], R, wl.k, idx, ws,
                        q_scale=inp.get("q_scale"), k_scale=inp.get("k_scale"),
                        dtype=DT[wl.idx_dtype])

    def attention():
        ic.sparse_attn(inp["q"], kmat, wl.d_qk, vmat, wl.d_qk if wl.latent else wl.d_v, idx, R,
                       wl.d_v, wl.scale, out, ws, dtype=DT[wl.attn_dtype])

    # inputs of the later stages come from the earlier ones (untimed)
    indexer()
    topk()
    fn = {"indexer": indexer, "topk": topk, "select": select, "attention": attention}[args.stage]
    fn()  # untimed first launch (function attributes, module load)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.launches):
        fn()
    b.record()
    torch.cuda.synchronize()
    st = ic.read_status(ws)
    print(json.dumps({"stage": args.stage, "workload": wl.name, "B": B, "rows": rows,
                      "ms_per_launch": a.elapsed_time(b) / args.launches, "status": st}))


if __name__ == "__main__":
    main()
