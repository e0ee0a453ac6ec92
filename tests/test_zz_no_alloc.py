"""The workspace-free attention entry point, checked against ic_sparse_attn.

ic_sparse_attn_noalloc is for callers that may not allocate device memory
where they run attention (for example an engine whose memory pool owns the
whole GPU, or a plugin that is handed only its input and output buffers).  It
keeps the decode split-k partials in a fixed device array inside the library
instead of a caller workspace.  Here it is called through the C ABI twice in a
row, on different inputs; each result must be within the attention tolerance
of the float64 oracle, as must ic_sparse_attn's (the entry point with a
workspace) on the same inputs, and the two must agree with each other.  This
file sorts last so that a run stopping at the first failure has already run
every other test; it also passes when run alone.
"""
import ctypes

import pytest
import torch

import oracle
import cross_layer_top_full_b200 as ic
from cross_layer_top_full_b200 import synth
from parity_util import check_attention, host64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ic.lib()
    return torch.device("cuda:0")


def _inputs(rows, k, dev, seed):
    B, Lq, q_start, T = rows
    g = torch.Generator(device=dev).manual_seed(seed)
    q = torch.randn(B, Lq, 128, 576, device=dev, generator=g).bfloat16()
    kv = (torch.randn(B, T, 576, device=dev, generator=g) / 24 ** 0.5).bfloat16()
    idx = synth.random_index_sets(B, Lq, q_start, k, dev, seed=seed)
    return q, kv, idx


def _with_workspace(q, kv, idx, rows, scale, dev):
    B, Lq = rows[0], rows[1]
    k = idx.shape[-1]
    ws = torch.empty(ic.sparse_attn_workspace_size(rows, k, 128, 576, 512, ic.BF16),
                     dtype=torch.uint8, device=dev)
    ic.workspace_init(ws)
    out = torch.empty(B, Lq, 128, 512, dtype=torch.bfloat16, device=dev)
    ic.sparse_attn(q, kv, 576, kv, 576, idx, rows, 512, scale, out, ws)
    return out


def _noalloc(q, kv, idx, rows, scale, dev):
    B, Lq = rows[0], rows[1]
    out = torch.full((B, Lq, 128, 512), float("nan"), dtype=torch.bfloat16, device=dev)
    status = torch.full((1,), -1, dtype=torch.int32, device=dev)
    code = ic.lib().ic_sparse_attn_noalloc(q.data_ptr(), kv.data_ptr(), idx.data_ptr(),
                                           idx.shape[-1], ic.Rows(*rows), ctypes.c_float(scale),
                                           out.data_ptr(), status.data_ptr(),
                                           torch.cuda.current_stream().cuda_stream)
    assert code == 0, ic.status_string(code)
    return out, status


@pytest.mark.parametrize("rows,k", [((8, 1, 4999, 5000), 2048),     # decode, split-k partials
                                    ((6, 1, 4999, 5000), 2048),     # split count capped by the array
                                    ((12, 1, 4999, 5000), 2048),
                                    ((16, 1, 8999, 9000), 4096),    # 2+ splits per row, 64 units
                                    ((3, 2, 700, 702), 512)])
def test_noalloc_matches_workspace_entry_point_twice(dev, rows, k):
    scale = 576 ** -0.5
    # the decode cases must actually use the fixed array (split-k partials)
    need = ic.sparse_attn_workspace_size(rows, k, 128, 576, 512, ic.BF16) - ic.STATUS_BYTES
    if rows[1] == 1:
        assert need > 0
    for call, seed in enumerate((1, 2)):            # two calls in a row, different inputs
        q, kv, idx = _inputs(rows, k, dev, seed + 10 * k + rows[0])
        ref = _with_workspace(q, kv, idx, rows, scale, dev)
        got, status = _noalloc(q, kv, idx, rows, scale, dev)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, call
        kvh = host64(kv)
        want = oracle.sparse_attention(host64(q), kvh, kvh[..., :512], host64(idx), scale)
        check_attention(host64(got), want, "no-alloc call %d vs oracle" % call)
        check_attention(host64(ref), want, "workspace call %d vs oracle" % call)
        check_attention(host64(got), host64(ref), "no-alloc call %d vs workspace" % call)


def test_noalloc_rejects_problems_beyond_its_fixed_array(dev):
    """k = 4096 needs at least two splits of 2048 keys per row, so 33 decode
    rows need at least 66 partial rows, more than the array's 64, on any GPU:
    the call is refused before anything is launched and leaves the output
    untouched."""
    rows, k = (33, 1, 4999, 5000), 4096
    q, kv, idx = _inputs(rows, k, dev, 5)
    out = torch.zeros(33, 1, 128, 512, dtype=torch.bfloat16, device=dev)
    torch.cuda.synchronize()
    code = ic.lib().ic_sparse_attn_noalloc(q.data_ptr(), kv.data_ptr(), idx.data_ptr(), k,
                                           ic.Rows(*rows), ctypes.c_float(0.04), out.data_ptr(),
                                           None, torch.cuda.current_stream().cuda_stream)
    assert code == -4                              # IC_ERR_WORKSPACE, nothing launched
    torch.cuda.synchronize()
    assert not out.float().abs().sum().item()
    # one row fewer than the limit allows (32 rows x 2 splits = 64) runs
    rows, k = (32, 1, 4999, 5000), 4096
    q, kv, idx = q[:32].contiguous(), kv[:32].contiguous(), idx[:32].contiguous()
    got, status = _noalloc(q, kv, idx, rows, 0.04, dev)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kvh = host64(kv)
    want = oracle.sparse_attention(host64(q), kvh, kvh[..., :512], host64(idx), 0.04)
    check_attention(host64(got), want, "no-alloc at its limit vs oracle")
