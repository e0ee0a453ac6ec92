"""Pins of the float64 CPU oracle against things other than itself.

Each test ties an oracle function to a hand-worked example (tests/golden/),
a closed form, an invariant, brute force on tiny inputs, or an independent
library routine, so that a plausible slip in the oracle (a dropped ReLU, a
wrong sign, an off-by-one causal bound, a reversed tie-break, a transposed
operand, a missing scale) fails at least one of them.
"""
import json
import math
import os
import random

import numpy as np
import pytest
import torch

import oracle
from cross_layer_top_full_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------- e4m3
def test_e4m3_decode_matches_hand_table():
    for code, val in _load("e4m3_codes.json")["pairs"]:
        got = float(oracle.e4m3_decode(np.array([int(code, 16)], dtype=np.uint8))[0])
        if val == "nan":
            assert math.isnan(got), code
        else:
            assert got == val and math.copysign(1, got) == math.copysign(1, val), code


def test_e4m3_decode_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    # sign of zero too
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))


def test_fp8_inputs_decode_close_to_the_values_they_store():
    """The generator's codes decode (oracle) to within E4M3 rounding of x."""
    g = torch.Generator().manual_seed(5)
    x = torch.randn(3, 7, 16, generator=g) * torch.tensor([1e-3, 1.0, 50.0]).view(3, 1, 1)
    x[1, 2] = 0.0
    codes, scale = synth.fp8_per_token(x, 2)
    assert codes.dtype == torch.uint8 and scale.shape == (3, 7)
    assert float(scale[1, 2]) == 1.0
    dec = oracle.e4m3_decode(codes.numpy()) * scale.numpy()[..., None].astype(np.float64)
    xs = x.double().numpy()
    amax = np.abs(xs).max(axis=-1, keepdims=True)
    # the token's absmax maps to 448 exactly up to float32 scale rounding
    err = np.abs(dec - xs)
    # normal range: half an ulp of 3 mantissa bits = 2^-4 relative; subnormal
    # step of the scaled grid is 2^-9 * scale
    bound = np.maximum(np.abs(xs) * 2.0 ** -4, (amax / 448.0) * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(err <= bound + 1e-30)


# --------------------------------------------------------------------------- indexer
def _tiny():
    d = _load("tiny_chain.json")
    ix = d["indexer"]
    qI = np.array(ix["q_I"], dtype=np.float64)[None]
    w = np.array(ix["w"], dtype=np.float64)[None]
    kI = np.array(ix["k_I"], dtype=np.float64)[None]
    return d, qI, w, kI


def test_indexer_hand_worked_example():
    d, qI, w, kI = _tiny()
    sc = oracle.indexer_scores(qI, w, kI, q_start=0)[0]
    exp = d["indexer"]["scores"]
    for t in range(3):
        for s in range(3):
            if exp[t][s] is None:
                assert sc[t, s] == -np.inf
            else:
                assert sc[t, s] == exp[t][s]


def test_indexer_single_head_unit_weight_is_relu_of_dot():
    rng = np.random.default_rng(1)
    q = rng.standard_normal((2, 5, 1, 7))
    k = rng.standard_normal((2, 9, 7))
    w = np.ones((2, 5, 1))
    sc = oracle.indexer_scores(q, w, k, q_start=4)
    for b in range(2):
        for i in range(5):
            t = 4 + i
            for s in range(9):
                want = max(0.0, float(sum(q[b, i, 0, d] * k[b, s, d] for d in range(7))))
                if s <= t:
                    assert sc[b, i, s] == pytest.approx(want, rel=1e-12, abs=1e-12)
                else:
                    assert sc[b, i, s] == -np.inf


def test_indexer_negative_weight_and_head_sum():
    """w enters linearly outside the ReLU, and heads add up."""
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 4, 3, 5))
    k = rng.standard_normal((1, 4, 5))
    w = rng.standard_normal((1, 4, 3))
    full = oracle.indexer_scores(q, w, k, 0)
    parts = sum(oracle.indexer_scores(q[:, :, h:h + 1], w[:, :, h:h + 1], k, 0)
                for h in range(3))
    fin = np.isfinite(full)
    assert np.allclose(full[fin], parts[fin], rtol=1e-12, atol=1e-12)
    neg = oracle.indexer_scores(q, -w, k, 0)
    assert np.allclose(neg[fin], -full[fin])
    # ReLU is inside: flipping q changes which dot products survive
    flip = oracle.indexer_scores(-q, w, k, 0)
    dots = np.einsum("bihd,bsd->bihs", q, k)
    want = np.einsum("bih,bihs->bis", w, np.maximum(-dots, 0))
    assert np.allclose(flip[fin], want[fin])


def test_indexer_fp8_scales_multiply_the_score():
    """Positive per-token scales factor out of the ReLU: I = sq*sk*I(codes)."""
    rng = np.random.default_rng(3)
    codes_q = rng.integers(0, 256, size=(1, 3, 2, 4)).astype(np.uint8)
    codes_k = rng.integers(0, 256, size=(1, 6, 4)).astype(np.uint8)
    codes_q[(codes_q & 0x7F) == 0x7F] = 0x38      # no NaN codes
    codes_k[(codes_k & 0x7F) == 0x7F] = 0x38
    w = rng.standard_normal((1, 3, 2))
    sq = np.array([[0.5, 2.0, 0.125]])
    sk = np.array([[1.0, 4.0, 0.25, 2.0, 8.0, 0.5]])
    got = oracle.indexer_scores(codes_q, w, codes_k, 3, sq, sk, fp8=True)
    vq = oracle.e4m3_decode(codes_q)
    vk = oracle.e4m3_decode(codes_k)
    base = oracle.indexer_scores(vq, w, vk, 3)
    fin = np.isfinite(base)
    want = base * sq[:, :, None] * sk[:, None, :]
    assert np.allclose(got[fin], want[fin], rtol=1e-12)
    assert np.array_equal(np.isfinite(got), fin)


# --------------------------------------------------------------------------- top-k
def _brute_topk_row(vals, t, k):
    cand = list(range(t + 1))
    # +0.0 and -0.0 compare equal in Python, so the tie-break sees them as equal
    cand.sort(key=lambda s: (-vals[s], s))
    chosen = sorted(cand[:k])
    return chosen + [-1] * (k - len(chosen))


def test_topk_hand_worked_example():
    d, qI, w, kI = _tiny()
    sc = oracle.indexer_scores(qI, w, kI, 0)
    assert oracle.topk_indices(sc, 0, 2)[0].tolist() == d["topk"]["k2"]
    assert oracle.topk_indices(sc, 0, 1)[0].tolist() == d["topk"]["k1"]


@pytest.mark.parametrize("seed", range(40))
def test_topk_matches_brute_force_sort(seed):
    r = random.Random(seed)
    B, Lq = r.randint(1, 2), r.randint(1, 6)
    q_start = r.choice([0, 0, 3, 10])
    T = q_start + Lq + r.randint(0, 4)
    k = r.randint(1, T + 2)
    pool = [-2.0, -1.0, -0.0, 0.0, 0.5, 1.0, 1.0, 3.0] if seed % 2 else None
    vals = np.empty((B, Lq, T))
    for idx in np.ndindex(vals.shape):
        vals[idx] = r.choice(pool) if pool else r.gauss(0, 1)
    got = oracle.topk_indices(vals, q_start, k)
    for b in range(B):
        for i in range(Lq):
            assert got[b, i].tolist() == _brute_topk_row(vals[b, i], q_start + i, k)


def test_topk_takes_every_candidate_when_k_exceeds_context():
    vals = np.random.default_rng(0).standard_normal((1, 5, 5))
    got = oracle.topk_indices(vals, 0, 8)
    for t in range(5):
        assert got[0, t].tolist() == list(range(t + 1)) + [-1] * (7 - t)


def test_topk_positive_and_negative_zero_tie_to_smaller_position():
    vals = np.array([[[0.0, -0.0, 0.0, -0.0]]])
    assert oracle.topk_indices(vals, 3, 2)[0, 0].tolist() == [0, 1]
    vals = np.array([[[-0.0, 0.0, -1.0, 0.0]]])
    assert oracle.topk_indices(vals, 3, 1)[0, 0].tolist() == [0]


# --------------------------------------------------------------------------- attention
def test_attention_hand_worked_example():
    a = _load("tiny_chain.json")["attention"]
    q = np.array(a["q"])[None]
    K = np.array(a["K"], dtype=np.float64)[None]
    V = np.array(a["V"], dtype=np.float64)[None]
    idx = np.array(a["idx"])[None]
    got = oracle.sparse_attention(q, K, V, idx, a["scale"])[0]
    assert np.allclose(got, np.array(a["out"]), rtol=0, atol=1e-12)


@pytest.mark.parametrize("q_start", [0, 5])
def test_sparse_equals_dense_when_k_covers_the_context(q_start):
    rng = np.random.default_rng(10 + q_start)
    B, Lq, Hq, d, dv = 2, 6, 3, 5, 4
    T = q_start + Lq
    q = rng.standard_normal((B, Lq, Hq, d))
    K = rng.standard_normal((B, T, d))
    V = rng.standard_normal((B, T, dv))
    sc = rng.standard_normal((B, Lq, T))
    idx = oracle.topk_indices(sc, q_start, T + 3)      # every causal key
    sp = oracle.sparse_attention(q, K, V, idx, 0.7)
    de = oracle.dense_causal_attention(q, K, V, q_start, 0.7)
    assert np.allclose(sp, de, rtol=1e-12, atol=1e-12)


def test_dense_attention_closed_forms():
    rng = np.random.default_rng(4)
    # zero query -> uniform weights -> running mean of the causal values
    V = rng.standard_normal((1, 6, 3))
    K = rng.standard_normal((1, 6, 2))
    q = np.zeros((1, 6, 2, 2))
    out = oracle.dense_causal_attention(q, K, V, 0, 1.0)
    for t in range(6):
        assert np.allclose(out[0, t, 0], V[0, : t + 1].mean(axis=0))
    # query row 0 has one causal key
    q = rng.standard_normal((1, 6, 2, 2))
    out = oracle.dense_causal_attention(q, K, V, 0, 1.0)
    assert np.allclose(out[0, 0, :], V[0, 0])


def test_attention_single_key_equal_rows_and_padding():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, 2, 4, 3))
    K = rng.standard_normal((1, 5, 3))
    V = rng.standard_normal((1, 5, 2))
    idx = np.array([[[3, -1, -1], [-1, -1, -1]]])
    out = oracle.sparse_attention(q, K, V, idx, 1.0)
    assert np.allclose(out[0, 0], V[0, 3])               # one key -> its value
    assert np.all(out[0, 1] == 0)                        # no key -> zeros
    Ve = np.repeat(V[:, :1], 5, axis=1)                  # all values equal
    idx = np.array([[[0, 2, 4], [1, 3, -1]]])
    out = oracle.sparse_attention(q, K, Ve, idx, 1.0)
    assert np.allclose(out[0], np.broadcast_to(V[0, 0], out[0].shape))


def test_attention_two_keys_is_a_sigmoid_mix():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((1, 1, 2, 4))
    K = rng.standard_normal((1, 3, 4))
    V = rng.standard_normal((1, 3, 5))
    scale = 0.3
    out = oracle.sparse_attention(q, K, V, np.array([[[2, 0]]]), scale)
    for h in range(2):
        z = scale * (q[0, 0, h] @ K[0, 2] - q[0, 0, h] @ K[0, 0])
        p2 = 1.0 / (1.0 + math.exp(-z))
        assert np.allclose(out[0, 0, h], p2 * V[0, 2] + (1 - p2) * V[0, 0])


def test_attention_ignores_index_order_and_uses_keys_not_values_for_logits():
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, 1, 2, 3))
    K = rng.standard_normal((1, 4, 3))
    V = rng.standard_normal((1, 4, 6))
    a = oracle.sparse_attention(q, K, V, np.array([[[0, 1, 3]]]), 1.0)
    b = oracle.sparse_attention(q, K, V, np.array([[[3, -1, 0, 1]]]), 1.0)
    assert np.allclose(a, b)


# --------------------------------------------------------------------------- stack
def _random_stack(pattern, seed, L=7, T=7):
    rng = np.random.default_rng(seed)
    layers = []
    for _ in pattern:
        layers.append(dict(q_I=rng.standard_normal((1, L, 2, 3)), w=rng.standard_normal((1, L, 2)),
                           k_I=rng.standard_normal((1, T, 3)), q=rng.standard_normal((1, L, 2, 4)),
                           K=rng.standard_normal((1, T, 4)), V=rng.standard_normal((1, T, 3))))
    return layers


def test_stack_shared_layers_reuse_the_preceding_full_layer():
    pattern = "FSSFS"
    layers = _random_stack(pattern, 8)
    idx, out, n_ix = oracle.layer_stack(pattern, layers, 0, 3, 0.5)
    assert n_ix == pattern.count("F")
    assert np.array_equal(idx[1], idx[0]) and np.array_equal(idx[2], idx[0])
    assert np.array_equal(idx[4], idx[3])
    fresh3 = oracle.topk_indices(oracle.indexer_scores(layers[3]["q_I"], layers[3]["w"],
                                                       layers[3]["k_I"], 0), 0, 3)
    assert np.array_equal(idx[3], fresh3)
    # an S layer's output is attention over the F layer's indices with its own q/K/V
    want = oracle.sparse_attention(layers[2]["q"], layers[2]["K"], layers[2]["V"], idx[0], 0.5)
    assert np.allclose(out[2], want)
    # the all-F stack differs on S layers in general (own indices)
    idx_f, _, n_f = oracle.layer_stack("F" * 5, layers, 0, 3, 0.5)
    assert n_f == 5 and np.array_equal(idx_f[0], idx[0])


@pytest.mark.parametrize("bad", ["SF", "FX", "F", "FSS", ""])
def test_stack_rejects_bad_patterns(bad):
    layers = _random_stack("FF", 9)
    with pytest.raises(ValueError):
        oracle.layer_stack(bad, layers, 0, 2, 1.0)


def test_topk_overlap():
    a = np.array([[0, 1, 2, -1], [5, 6, 7, 8]])
    b = np.array([[2, 1, 9, -1], [-1, -1, -1, -1]])
    assert oracle.topk_overlap(a, b).tolist() == [2 / 3, 0.0]


# --------------------------------------------------------------------------- planted mistakes
def test_pins_catch_planted_mistakes(monkeypatch):
    """Plant plausible slips in copies of oracle functions (on the CPU) and
    check that the hand-worked example and brute force detect each one."""
    d, qI, w, kI = _tiny()
    exp_scores = d["indexer"]["scores"]

    def score_ok(fn):
        sc = fn(qI, w, kI, 0)[0]
        return all((sc[t, s] == -np.inf) if exp_scores[t][s] is None else sc[t, s] == exp_scores[t][s]
                   for t in range(3) for s in range(3))

    def no_relu(q, w_, k, q_start):
        dots = np.einsum("bihd,bsd->bihs", q, k)
        out = np.einsum("bih,bihs->bis", w_, dots)
        return _mask(out, q_start)

    def relu_outside(q, w_, k, q_start):
        dots = np.einsum("bihd,bsd->bihs", q, k)
        out = np.maximum(np.einsum("bih,bihs->bis", w_, dots), 0)
        return _mask(out, q_start)

    def strict_causal(q, w_, k, q_start):
        out = oracle.indexer_scores(q, w_, k, q_start)
        for i in range(out.shape[1]):
            out[:, i, q_start + i] = -np.inf
        return out

    def _mask(out, q_start):
        T = out.shape[-1]
        for i in range(out.shape[1]):
            out[:, i, q_start + i + 1:] = -np.inf
        return out

    assert score_ok(oracle.indexer_scores)
    for bad in (no_relu, relu_outside, strict_causal):
        assert not score_ok(bad), bad.__name__

    # top-k with the tie going to the larger position fails the k=1 example
    sc = oracle.indexer_scores(qI, w, kI, 0)

    def larger_tie(scores, q_start, k):
        s = scores[0]
        out = np.full((1, s.shape[0], k), -1, np.int32)
        for i in range(s.shape[0]):
            t = q_start + i
            order = sorted(range(t + 1), key=lambda j: (-s[i, j], -j))[:k]
            out[0, i, : len(order)] = sorted(order)
        return out

    assert larger_tie(sc, 0, 1)[0].tolist() != d["topk"]["k1"]

    # attention with the scale or the K/V roles swapped fails the example
    a = d["attention"]
    q = np.array(a["q"])[None]
    K = np.array(a["K"], dtype=np.float64)[None]
    V = np.array(a["V"], dtype=np.float64)[None]
    idx = np.array(a["idx"])[None]
    assert not np.allclose(oracle.sparse_attention(q, K, V, idx, 2.0)[0], a["out"])
    Kpad = np.concatenate([V, V], axis=-1)
    assert not np.allclose(oracle.sparse_attention(q, Kpad, K[..., :1], idx, 1.0)[0], a["out"])
