"""Seeded synthetic inputs for the IndexCache hot path.

This module only draws random numbers and stores them in the layouts the
library reads; it holds none of the method's arithmetic, so both the CUDA
path and the CPU oracle may use it.  Everything is drawn with
``torch.Generator`` on the requested device from a seed derived from
(workload seed, layer, tensor name); CPU and CUDA generators give different
streams, so a test always moves the very tensors the GPU read to the host.

Workloads (shapes and distributions; the pages give none of them, see the
reading notes in each entry):

* ``prefill_512_fp32``     1 sequence, L=512, FSSS, indexer H_I=4, d_I=32,
  k=64; attention 8 heads sharing one K/V head, d_qk=d_v=64; float32.
* ``prefill_8k_bf16``      1 sequence, L=8192, FSSS, H_I=64, d_I=128, k=2048;
  MQA with 128 heads over one latent KV row of width 576 (V = its first 512
  columns); bf16 activations.
* ``prefill_8k_fp8``       the same with the indexer operands as E4M3 codes
  and one float32 scale per token (the FP8 prefill indexer).
* ``decode_b32_t32k_bf16`` 32 sequences x 32768 cached keys, one new query
  each, pattern FSSSFSSS; caches N(0,1)/sqrt(d) with 16 heavy-hitter
  positions per sequence scaled x4.
* ``chunked_prefill_64k_bf16`` 1 sequence, L=65536 in 4096-row chunks,
  12 layers FSSFSSSSFSSS; k_I^(l) = base + 0.3 * noise^(l).
* ``decode_b8_t200k_fp8``  8 sequences x 200000 keys, (FSSS)x12; indexer
  operands as E4M3 codes with one float32 scale per token (absmax/448).
* ``decode_b32_varlen_paged_bf16`` 32 sequences of lengths uniform in
  [4096, 32768], one new query each, FSSSFSSS, caches in 128-row pages
  shuffled over one physical cache (paged_batch / paged_layer_inputs).
"""
from __future__ import annotations

import dataclasses
import hashlib
import math
from typing import Dict, Optional

import torch

__all__ = ["Workload", "WORKLOADS", "layer_inputs", "heavy_hitters", "fp8_per_token",
           "paged_batch", "paged_layer_inputs"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    L: int                  # query rows per sequence in one pass (prefill) / 1 (decode)
    T: int                  # keys per sequence
    q_start: int
    H_I: int
    d_I: int
    k: int
    Hq: int
    d_qk: int
    d_v: int
    idx_dtype: str          # 'f32' | 'bf16' | 'e4m3'
    attn_dtype: str         # 'f32' | 'bf16'
    latent: bool            # K and V share one row of width d_qk (V = first d_v cols)
    pattern: str
    seed: int
    w_std: float
    qI_std: float
    kI_std: float
    q_std: float
    kv_std: float
    heavy: int = 0          # planted high-norm positions per sequence
    heavy_gain: float = 1.0
    chunk: int = 0          # chunked prefill: query rows per chunk (0 = one pass)
    kI_noise: float = 0.0   # chunked prefill: per-layer key noise relative to base
    len_min: int = 0        # paged batches: sequence lengths uniform in [len_min, T]
    page: int = 0           # paged batches: rows per page (0 = dense caches)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d_qk)

    @property
    def n_layers(self) -> int:
        return len(self.pattern)

    @property
    def kv_width(self) -> int:
        return self.d_qk


WORKLOADS: Dict[str, Workload] = {
    "prefill_512_fp32": Workload(
        "prefill_512_fp32", B=1, L=512, T=512, q_start=0, H_I=4, d_I=32, k=64,
        Hq=8, d_qk=64, d_v=64, idx_dtype="f32", attn_dtype="f32", latent=False,
        pattern="FSSS", seed=0, w_std=1 / math.sqrt(4), qI_std=1 / math.sqrt(32),
        kI_std=1 / math.sqrt(32), q_std=1.0, kv_std=1.0),
    "prefill_8k_bf16": Workload(
        "prefill_8k_bf16", B=1, L=8192, T=8192, q_start=0, H_I=64, d_I=128, k=2048,
        Hq=128, d_qk=576, d_v=512, idx_dtype="bf16", attn_dtype="bf16", latent=True,
        pattern="FSSS", seed=1, w_std=1 / 8, qI_std=1 / math.sqrt(128),
        kI_std=1 / math.sqrt(128), q_std=1.0, kv_std=1.0),
    # the prefill workload with the indexer operands in E4M3 (one float32
    # scale per token), the FP8 prefill indexer; same seed, so its q_I / k_I
    # are the bf16 workload's values before quantisation
    "prefill_8k_fp8": Workload(
        "prefill_8k_fp8", B=1, L=8192, T=8192, q_start=0, H_I=64, d_I=128, k=2048,
        Hq=128, d_qk=576, d_v=512, idx_dtype="e4m3", attn_dtype="bf16", latent=True,
        pattern="FSSS", seed=1, w_std=1 / 8, qI_std=1 / math.sqrt(128),
        kI_std=1 / math.sqrt(128), q_std=1.0, kv_std=1.0),
    # decode q / q_I / w follow the prefill workload (only the caches are
    # specified for decode); KV and K_I caches are N(0,1)/sqrt(d).
    "decode_b32_t32k_bf16": Workload(
        "decode_b32_t32k_bf16", B=32, L=1, T=32768, q_start=32767, H_I=64, d_I=128, k=2048,
        Hq=128, d_qk=576, d_v=512, idx_dtype="bf16", attn_dtype="bf16", latent=True,
        pattern="FSSSFSSS", seed=2, w_std=1 / 8, qI_std=1 / math.sqrt(128),
        kI_std=1 / math.sqrt(128), q_std=1.0, kv_std=1 / math.sqrt(576), heavy=16,
        heavy_gain=4.0),
    "chunked_prefill_64k_bf16": Workload(
        "chunked_prefill_64k_bf16", B=1, L=65536, T=65536, q_start=0, H_I=64, d_I=128,
        k=2048, Hq=128, d_qk=576, d_v=512, idx_dtype="bf16", attn_dtype="bf16",
        latent=True, pattern="FSSFSSSSFSSS", seed=3, w_std=1 / 8,
        qI_std=1 / math.sqrt(128), kI_std=1 / math.sqrt(128), q_std=1.0, kv_std=1.0,
        chunk=4096, kI_noise=0.3),
    # a decode batch of mixed lengths over paged caches (the serving layout):
    # the bf16 decode workload's shapes, lengths uniform in [4096, 32768],
    # 128-row pages shuffled over one cache
    "decode_b32_varlen_paged_bf16": Workload(
        "decode_b32_varlen_paged_bf16", B=32, L=1, T=32768, q_start=32767, H_I=64, d_I=128,
        k=2048, Hq=128, d_qk=576, d_v=512, idx_dtype="bf16", attn_dtype="bf16", latent=True,
        pattern="FSSSFSSS", seed=5, w_std=1 / 8, qI_std=1 / math.sqrt(128),
        kI_std=1 / math.sqrt(128), q_std=1.0, kv_std=1 / math.sqrt(576), len_min=4096, page=128),
    "decode_b8_t200k_fp8": Workload(
        "decode_b8_t200k_fp8", B=8, L=1, T=200000, q_start=199999, H_I=64, d_I=128, k=2048,
        Hq=128, d_qk=576, d_v=512, idx_dtype="e4m3", attn_dtype="bf16", latent=True,
        pattern="FSSS" * 12, seed=4, w_std=1 / 8, qI_std=1 / math.sqrt(128),
        kI_std=1 / math.sqrt(128), q_std=1.0, kv_std=1 / math.sqrt(576), heavy=16,
        heavy_gain=4.0),
}


def _gen(device, *key) -> torch.Generator:
    h = hashlib.sha256(repr(key).encode()).digest()
    g = torch.Generator(device=device)
    g.manual_seed(int.from_bytes(h[:8], "little") & ((1 << 63) - 1))
    return g


def _randn(shape, std, device, *key, dtype=torch.float32) -> torch.Tensor:
    x = torch.randn(shape, generator=_gen(device, *key), device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def _store_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def heavy_hitters(wl: Workload, device) -> Optional[torch.Tensor]:
    """[B, heavy] int64 positions per sequence, uniform without replacement;
    the same positions in every layer (they are properties of the sequence)."""
    if wl.heavy == 0:
        return None
    rows = []
    for b in range(wl.B):
        g = _gen("cpu", wl.seed, "heavy", b)
        rows.append(torch.randperm(wl.T, generator=g)[: wl.heavy])
    return torch.stack(rows).to(device)


def fp8_per_token(x: torch.Tensor, token_dims: int):
    """Store ``x`` as E4M3 codes with one float32 scale per token.

    The first ``token_dims`` axes index tokens; all remaining axes are that
    token's values.  scale = absmax/448 (1 where the token is all zero);
    codes = float8_e4m3fn(x / scale) by torch's round-to-nearest-even cast,
    after clamping to the finite range.  Returns (uint8 codes, float32 scale).
    """
    flat = x.reshape(*x.shape[:token_dims], -1)
    amax = flat.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax)).to(torch.float32)
    y = (flat / scale.unsqueeze(-1)).clamp_(-448.0, 448.0)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8).reshape(x.shape)
    return codes.contiguous(), scale.contiguous()


def _plant(x: torch.Tensor, hh: Optional[torch.Tensor], gain: float) -> torch.Tensor:
    if hh is None:
        return x
    for b in range(x.shape[0]):
        x[b, hh[b]] *= gain
    return x


def layer_inputs(wl: Workload, layer: int, device="cpu", *, indexer: bool = True,
                 attention: bool = True, chunk: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Inputs of one layer.

    Keys: 'q_I' [B,L,H_I,d_I], 'w' [B,L,H_I] f32, 'k_I' [B,T,d_I]
    (+ 'q_scale' [B,L], 'k_scale' [B,T] for e4m3), 'q' [B,L,Hq,d_qk], and
    either 'kv' [B,T,d_qk] (latent) or 'k' [B,T,d_qk], 'v' [B,T,d_v].
    For a chunked workload, ``chunk`` selects the query rows
    [chunk*wl.chunk, (chunk+1)*wl.chunk) of 'q', 'q_I' and 'w'; keys cover the
    full sequence (a call uses the causal prefix).
    """
    out: Dict[str, torch.Tensor] = {}
    B, L, T = wl.B, wl.L, wl.T
    hh = heavy_hitters(wl, device)
    if wl.chunk:
        c = 0 if chunk is None else chunk
        qrows = wl.chunk
    else:
        c, qrows = 0, L
    if indexer:
        if wl.kI_noise:
            # base shared by all layers + per-layer noise at kI_noise x base's std
            base = _randn((B, T, wl.d_I), wl.kI_std, device, wl.seed, "kI_base")
            noise = _randn((B, T, wl.d_I), wl.kI_std * wl.kI_noise, device, wl.seed, "kI_noise", layer)
            kI = base + noise
            # queries of the indexer are shared by all layers of this workload
            qkey, wkey = ("qI_shared", c), ("w_shared", c)
        else:
            kI = _randn((B, T, wl.d_I), wl.kI_std, device, wl.seed, "kI", layer)
            qkey, wkey = ("qI", layer, c), ("w", layer, c)
        kI = _plant(kI, hh, wl.heavy_gain)
        qI = _randn((B, qrows, wl.H_I, wl.d_I), wl.qI_std, device, wl.seed, *qkey)
        out["w"] = _randn((B, qrows, wl.H_I), wl.w_std, device, wl.seed, *wkey)
        if wl.idx_dtype == "e4m3":
            out["q_I"], out["q_scale"] = fp8_per_token(qI, 2)
            out["k_I"], out["k_scale"] = fp8_per_token(kI, 2)
        else:
            dt = _store_dtype(wl.idx_dtype)
            out["q_I"] = qI.to(dt).contiguous()
            out["k_I"] = kI.to(dt).contiguous()
        del qI, kI
    if attention:
        adt = _store_dtype(wl.attn_dtype)
        out["q"] = _randn((B, qrows, wl.Hq, wl.d_qk), wl.q_std, device, wl.seed, "q", layer, c,
                          dtype=adt)
        if wl.latent:
            kv = _randn((B, T, wl.d_qk), wl.kv_std, device, wl.seed, "kv", layer)
            out["kv"] = _plant(kv, hh, wl.heavy_gain).to(adt).contiguous()
        else:
            out["k"] = _randn((B, T, wl.d_qk), wl.kv_std, device, wl.seed, "k", layer, dtype=adt)
            out["v"] = _randn((B, T, wl.d_v), wl.kv_std, device, wl.seed, "v", layer, dtype=adt)
    return out


def paged_batch(wl: Workload, device="cpu"):
    """Geometry of a paged workload: (seq_lens [B] int32, block_table [B,
    max_pages] int32, num_pages).  Lengths are uniform in [len_min, T] (the
    first sequence T long, so T is reached); every sequence's pages are
    distinct physical pages in a seeded random order; unused table entries
    are -1."""
    assert wl.page, "paged workload expected"
    g = _gen("cpu", wl.seed, "paged")
    lens = torch.randint(wl.len_min, wl.T + 1, (wl.B,), generator=g)
    lens[0] = wl.T
    P = wl.page
    pages_per = (lens + P - 1) // P
    max_pages = (wl.T + P - 1) // P
    num_pages = int(pages_per.sum())
    perm = torch.randperm(num_pages, generator=g).to(torch.int32)
    table = torch.full((wl.B, max_pages), -1, dtype=torch.int32)
    c = 0
    for b in range(wl.B):
        n = int(pages_per[b])
        table[b, :n] = perm[c:c + n]
        c += n
    return lens.to(torch.int32).to(device), table.to(device), num_pages


def paged_layer_inputs(wl: Workload, layer: int, num_pages: int, device="cpu") -> Dict[str, torch.Tensor]:
    """Inputs of one layer of a paged workload: 'q_I' [B,L,H_I,d_I], 'w'
    [B,L,H_I], 'q' [B,L,Hq,d_qk] as in layer_inputs, and the paged caches
    'k_I' [num_pages*page, d_I] and 'kv' [num_pages*page, d_qk] (+ 'q_scale',
    'k_scale' for e4m3), every physical row drawn with the workload's
    distributions."""
    rows = num_pages * wl.page
    out: Dict[str, torch.Tensor] = {}
    qI = _randn((wl.B, wl.L, wl.H_I, wl.d_I), wl.qI_std, device, wl.seed, "qI", layer, 0)
    out["w"] = _randn((wl.B, wl.L, wl.H_I), wl.w_std, device, wl.seed, "w", layer, 0)
    kI = _randn((rows, wl.d_I), wl.kI_std, device, wl.seed, "kI_pages", layer)
    if wl.idx_dtype == "e4m3":
        out["q_I"], out["q_scale"] = fp8_per_token(qI, 2)
        out["k_I"], out["k_scale"] = fp8_per_token(kI, 1)
    else:
        dt = _store_dtype(wl.idx_dtype)
        out["q_I"] = qI.to(dt).contiguous()
        out["k_I"] = kI.to(dt).contiguous()
    del qI, kI
    adt = _store_dtype(wl.attn_dtype)
    out["q"] = _randn((wl.B, wl.L, wl.Hq, wl.d_qk), wl.q_std, device, wl.seed, "q", layer, 0,
                      dtype=adt)
    out["kv"] = _randn((rows, wl.d_qk), wl.kv_std, device, wl.seed, "kv_pages", layer, dtype=adt)
    return out


def chunk_queries(wl: Workload, layer: int, chunk: int, device="cpu", *,
                  indexer: bool = True) -> Dict[str, torch.Tensor]:
    """Query-side inputs of one chunk of a chunked workload, drawn exactly as
    ``layer_inputs(wl, layer, device, chunk=chunk)`` draws them: 'q'
    [B,chunk,Hq,d_qk] and, with ``indexer``, 'q_I' [B,chunk,H_I,d_I] and 'w'
    [B,chunk,H_I] (+ 'q_scale' for e4m3).  Keys are not drawn."""
    assert wl.chunk, "chunked workload expected"
    B, qrows = wl.B, wl.chunk
    out: Dict[str, torch.Tensor] = {}
    if indexer:
        if wl.kI_noise:
            qkey, wkey = ("qI_shared", chunk), ("w_shared", chunk)
        else:
            qkey, wkey = ("qI", layer, chunk), ("w", layer, chunk)
        qI = _randn((B, qrows, wl.H_I, wl.d_I), wl.qI_std, device, wl.seed, *qkey)
        out["w"] = _randn((B, qrows, wl.H_I), wl.w_std, device, wl.seed, *wkey)
        if wl.idx_dtype == "e4m3":
            out["q_I"], out["q_scale"] = fp8_per_token(qI, 2)
        else:
            out["q_I"] = qI.to(_store_dtype(wl.idx_dtype)).contiguous()
        del qI
    out["q"] = _randn((B, qrows, wl.Hq, wl.d_qk), wl.q_std, device, wl.seed, "q", layer, chunk,
                      dtype=_store_dtype(wl.attn_dtype))
    return out


def exact_indexer_inputs(B: int, Lq: int, T: int, H_I: int, d_I: int, dtype: str, device="cpu",
                         seed: int = 0) -> Dict[str, torch.Tensor]:
    """Indexer inputs whose scores are exact in float32 for any summation order.

    q_I, k_I are integers in [-3, 3]; w = +-2^-j, j in 0..3; with e4m3 the
    codes hold those integers and the per-token scales are powers of two in
    {1/2, 1, 2}.  Every product and partial sum is then a multiple of 2^-5
    below 2^22, so float32 represents it exactly and the top-k is unique up
    to exact ties (which the smaller-position rule settles).
    """
    g = _gen(device, seed, "exact")
    qI = torch.randint(-3, 4, (B, Lq, H_I, d_I), generator=g, device=device).float()
    kI = torch.randint(-3, 4, (B, T, d_I), generator=g, device=device).float()
    sign = torch.randint(0, 2, (B, Lq, H_I), generator=g, device=device).float() * 2 - 1
    j = torch.randint(0, 4, (B, Lq, H_I), generator=g, device=device).float()
    out = {"w": (sign * torch.pow(2.0, -j)).contiguous()}
    if dtype == "e4m3":
        out["q_I"] = qI.to(torch.float8_e4m3fn).view(torch.uint8).contiguous()
        out["k_I"] = kI.to(torch.float8_e4m3fn).view(torch.uint8).contiguous()
        ex_q = torch.randint(-1, 2, (B, Lq), generator=g, device=device).float()
        ex_k = torch.randint(-1, 2, (B, T), generator=g, device=device).float()
        out["q_scale"] = torch.pow(2.0, ex_q).contiguous()
        out["k_scale"] = torch.pow(2.0, ex_k).contiguous()
    else:
        dt = _store_dtype(dtype)
        out["q_I"] = qI.to(dt).contiguous()
        out["k_I"] = kI.to(dt).contiguous()
    return out


def random_scores(B: int, Lq: int, T: int, device="cpu", seed: int = 0, ties: bool = False,
                  ld: Optional[int] = None) -> torch.Tensor:
    """float32 scores [B, Lq, ld] (ld >= T, default T rounded up to 4).  With
    ``ties`` the values come from a small set including +0.0 and -0.0, so
    many scores are equal."""
    ld = ld or (T + 3) // 4 * 4
    g = _gen(device, seed, "scores", ties)
    if ties:
        pool = torch.tensor([-2.0, -1.0, -0.0, 0.0, 0.0, 0.5, 1.0, 3.0], device=device)
        pick = torch.randint(0, pool.numel(), (B, Lq, ld), generator=g, device=device)
        return pool[pick].contiguous()
    return torch.randn((B, Lq, ld), generator=g, device=device).contiguous()


def random_index_sets(B: int, Lq: int, q_start: int, k: int, device="cpu", seed: int = 0,
                      n_valid: Optional[int] = None) -> torch.Tensor:
    """int32 [B, Lq, k]: for row t, min(k, t+1, n_valid) distinct positions
    drawn uniformly from [0, t], ascending, then -1 padding."""
    g = _gen("cpu", seed, "idxsets")
    out = torch.full((B, Lq, k), -1, dtype=torch.int32)
    for b in range(B):
        for i in range(Lq):
            t = q_start + i
            m = min(k, t + 1) if n_valid is None else min(k, t + 1, n_valid)
            pos = torch.randperm(t + 1, generator=g)[:m].sort().values
            out[b, i, :m] = pos.to(torch.int32)
    return out.to(device)
