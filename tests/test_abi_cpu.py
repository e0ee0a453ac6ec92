"""Host-side checks of the C-ABI library that need no GPU.

The library must load, export every function include/indexcache.h
declares, and reject bad arguments before it touches the device.
"""
import ctypes
import os
import re
import subprocess

import pytest

import cross_layer_top_full_b200 as ic
from cross_layer_top_full_b200 import build as icbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(ic.library_path()):
        icbuild.build()
    return ic.lib()


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(ic_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_every_declared_symbol_is_exported(lib):
    declared = _declared()
    assert len(declared) >= 12
    out = subprocess.run(["nm", "-D", "--defined-only", ic.library_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (ic_[a-z0-9_]+)\b", out))
    missing = [n for n in declared if n not in exported]
    assert not missing, missing
    for n in declared:
        assert hasattr(lib, n)


def test_status_strings(lib):
    for code, name in [(0, "IC_OK"), (-2, "IC_ERR_PATTERN"), (-6, "IC_ERR_INDEX_RANGE"),
                       (-7, "IC_ERR_TIMEOUT")]:
        assert ic.status_string(code) == name
    assert ic.version() >= 10000


def _shape(B=1, L=16, T=16, k=4):
    return ic.StackShape(ic.Rows(B, L, T - L, T), 4, 32, ic.F32, k, 8, 64, 64, ic.F32, 64, 64, 0.125)


class _FakeTensor:
    """Host memory standing in for a device buffer; the calls below must
    return before any device access."""
    def __init__(self, nbytes, align=256):
        self.buf = ctypes.create_string_buffer(nbytes + align)
        addr = ctypes.addressof(self.buf)
        self.addr = (addr + align - 1) // align * align
        self.nbytes = nbytes

    def data_ptr(self):
        return self.addr

    def numel(self):
        return self.nbytes

    def element_size(self):
        return 1


@pytest.mark.parametrize("pattern", ["SFSS", "FSXS", "FSS", "FSSSS", "fsss"])
def test_stack_rejects_bad_patterns_before_launch(lib, pattern):
    sh = _shape()
    ws = _FakeTensor(ic.workspace_size(sh))
    layers = [dict(q=1, kmat=1, vmat=1, out=1, q_idx=1, w=1, k_idx=1)] * 4
    with pytest.raises(ic.IcError) as e:
        ic.layer_stack_forward(pattern, layers, sh, 1, ws, stream=0)
    assert e.value.code == -2


def test_stack_rejects_small_or_misaligned_workspace(lib):
    sh = _shape()
    need = ic.workspace_size(sh)
    assert need >= ic.STATUS_BYTES + 16 * 16 * 4
    layers = [dict(q=1, kmat=1, vmat=1, out=1, q_idx=1, w=1, k_idx=1)] * 4
    small = _FakeTensor(need - 1)
    with pytest.raises(ic.IcError) as e:
        ic.layer_stack_forward("FSSS", layers, sh, 1, small, stream=0)
    assert e.value.code == -4
    code = lib.ic_layer_stack_forward(b"FSSS", 4, (ic.LayerIO * 4)(), ctypes.byref(sh), 1, None,
                                      _FakeTensor(need + 512).addr + 8, need + 256, None)
    assert code == -4


def test_stack_rejects_missing_layer_pointers(lib):
    sh = _shape()
    ws = _FakeTensor(ic.workspace_size(sh))
    layers = [dict(q=1, kmat=1, vmat=1, out=1, q_idx=1, w=1, k_idx=1)] + \
             [dict(q=1, kmat=1, vmat=1, out=1)] * 3
    layers_bad = [dict(q=1, kmat=1, vmat=1, out=1)] * 4      # F layer without indexer inputs
    with pytest.raises(ic.IcError) as e:
        ic.layer_stack_forward("FSSS", layers_bad, sh, 1, ws, stream=0)
    assert e.value.code == -1
    with pytest.raises(ic.IcError) as e:        # S layers may omit them; idx_buf may not be NULL
        ic.layer_stack_forward("FSSS", layers, sh, None, ws, stream=0)
    assert e.value.code == -1


def test_single_calls_validate_arguments(lib):
    r = ic.Rows(1, 8, 4, 10)       # q_start + Lq = 12 > T = 10
    ws = _FakeTensor(4096)
    assert lib.ic_topk(1, 12, r, 4, 1, ws.addr, 4096, None) == -1
    r = ic.Rows(1, 8, 2, 10)
    assert lib.ic_topk(1, 10, r, 4, 1, ws.addr, 4096, None) == -1      # ld % 4 != 0
    assert lib.ic_topk(1, 12, r, 0, 1, ws.addr, 4096, None) == -1      # k = 0
    assert lib.ic_topk(1, 12, r, 4, 1, ws.addr, 100, None) == -4       # workspace too small
    assert lib.ic_indexer_scores(1, None, 1, 1, None, 7, r, 4, 32, 1, 12, ws.addr, 4096, None) == -1
    # fp8 needs both scales
    assert lib.ic_indexer_scores(1, None, 1, 1, None, ic.FP8_E4M3, r, 4, 32, 1, 12, ws.addr, 4096,
                                 None) == -1
    # scales on a non-fp8 dtype are an error too
    assert lib.ic_indexer_scores(1, 1, 1, 1, 1, ic.BF16, r, 4, 32, 1, 12, ws.addr, 4096, None) == -1
    assert lib.ic_sparse_attn(1, 1, 63, 1, 64, 1, 4, ic.F32, r, 8, 64, 64, 0.1, 1, ws.addr, 4096,
                              None) == -1                                # row stride < d_qk
    assert lib.ic_sparse_attn(1, 1, 64, 1, 64, 1, 4, ic.FP8_E4M3, r, 8, 64, 64, 0.1, 1, ws.addr,
                              4096, None) == -1                          # fp8 attention
    # empty problems (no sequence, or no query row) are valid no-ops that
    # launch nothing, with NULL data pointers too
    before = ic.kernel_launches(0)
    for e in (ic.Rows(0, 8, 2, 10), ic.Rows(1, 0, 2, 10), ic.Rows(0, 0, 0, 0)):
        assert lib.ic_topk(None, 12, e, 4, None, ws.addr, 4096, None) == 0
        assert lib.ic_indexer_scores(None, None, None, None, None, ic.BF16, e, 64, 128, None, 12,
                                     ws.addr, 4096, None) == 0
        assert lib.ic_sparse_attn(None, None, 576, None, 576, None, 2048, ic.BF16, e, 128, 576,
                                  512, 0.04, None, ws.addr, 4096, None) == 0
        assert lib.ic_sparse_attn_noalloc(None, None, None, 2048, e, 0.04, None, None, None) == 0
        sh = ic.StackShape(e, 64, 128, ic.BF16, 2048, 128, 576, 512, ic.BF16, 576, 576, 0.04)
        big = _FakeTensor(ic.workspace_size(sh))
        assert ic.lib().ic_layer_stack_forward(b"FS", 2, None, ctypes.byref(sh), None, None,
                                               big.addr, big.nbytes, None) == -1   # no layers
        layers = (ic.LayerIO * 2)()
        assert ic.lib().ic_layer_stack_forward(b"FS", 2, layers, ctypes.byref(sh), None, None,
                                               big.addr, big.nbytes, None) == 0
    assert ic.kernel_launches(0) == before


def test_workspace_sizes_grow_with_the_problem(lib):
    a = ic.workspace_size(_shape(L=16, T=16))
    b = ic.workspace_size(_shape(L=16, T=1024))
    assert b - a >= 16 * (1024 - 16) * 4
    assert ic.topk_workspace_size((1, 4, 0, 4), 2) == ic.STATUS_BYTES
    latent = ic.sparse_attn_workspace_size((32, 1, 32767, 32768), 2048, 128, 576, 512, ic.BF16)
    assert latent >= ic.STATUS_BYTES


def test_selftest_rejects_a_bad_workspace_before_launching(lib):
    """The failure-path self-test validates its workspace on the host and
    returns before any CUDA call (this host has no GPU to launch on)."""
    ws = _FakeTensor(4096)
    assert lib.ic_selftest_wait_timeout(ws.addr + 8, 4096, None) == -1    # misaligned
    assert lib.ic_selftest_wait_timeout(ws.addr, 16, None) == -1          # < IC_STATUS_BYTES
    assert lib.ic_selftest_wait_timeout(None, 4096, None) == -1           # no workspace
    assert lib.ic_check_status(None, None) == -1                          # no workspace


def test_cuda_failure_returns_an_error_with_its_text(lib):
    """A failing launch returns IC_ERR_CUDA at once and ic_last_error names
    the CUDA error; the binding puts the text into its exception.  On this
    host (no usable GPU) every launch fails, which exercises the path."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present: the launch would run (the GPU tests cover it)")
    ws = _FakeTensor(4096)
    assert lib.ic_selftest_wait_timeout(ws.addr, 4096, None) == -5        # IC_ERR_CUDA
    text = lib.ic_last_error().decode()
    assert text.startswith("kernel launch: ") and len(text) > len("kernel launch: ")
    with pytest.raises(ic.IcError) as e:
        ic.selftest_wait_timeout(ws)
    assert e.value.code == -5 and "kernel launch" in str(e.value)
    # a failing runtime call (not a launch) goes through the same recorder
    assert lib.ic_workspace_init(ws.addr, 4096, None) == -5
    assert lib.ic_last_error().decode().startswith("api: ")


def test_binding_refuses_host_tensors_and_strided_views(lib):
    import torch
    before = ic.kernel_launches(0)
    rows = (1, 4, 0, 4)
    host = torch.zeros(1, 4, 4)
    with pytest.raises(ValueError, match="CUDA tensor"):
        ic.topk(host, rows, 2, torch.zeros(1, 4, 2, dtype=torch.int32), _FakeTensor(4096))

    class _StridedDevice:
        """A device tensor's attributes, as a transposed view would report them."""
        is_cuda = True
        shape = (1, 4, 4)
        device = "cuda:0"

        def is_contiguous(self):
            return False

        def stride(self):
            return (16, 1, 4)

        def data_ptr(self):
            return 1 << 40

    with pytest.raises(ValueError, match="contiguous"):
        ic.topk(_StridedDevice(), rows, 2, 1 << 40, _FakeTensor(4096))
    assert ic.kernel_launches(0) == before


def test_paged_calls_validate_arguments(lib):
    """The variable-length / paged calls refuse inconsistent batches before
    any launch: host memory stands in for every device array here."""
    ws = _FakeTensor(1 << 16)
    lens = _FakeTensor(64)
    table = _FakeTensor(256)

    def pr(**kw):
        d = dict(B=2, Lq=1, T_max=512, seq_lens=lens.addr, block_table=table.addr, max_pages=4,
                 page_size=128, num_pages=8)
        d.update(kw)
        return ic.PagedRows(d["B"], d["Lq"], d["T_max"], d["seq_lens"], d["block_table"],
                            d["max_pages"], d["page_size"], d["num_pages"])

    before = ic.kernel_launches(0)

    def attn(p, ws_bytes=1 << 16):
        return lib.ic_sparse_attn_paged(1, 1, 1, 64, ctypes.byref(p), 0.1, 1, ws.addr, ws_bytes,
                                        None)

    assert attn(pr(page_size=100)) == -1            # not a multiple of 128
    assert attn(pr(page_size=0)) == -1
    assert attn(pr(max_pages=3)) == -1              # 3 pages of 128 cannot hold T_max = 512
    assert attn(pr(seq_lens=None)) == -1
    assert attn(pr(block_table=None)) == -1
    assert attn(pr(T_max=0)) == -1                  # T_max < Lq
    assert attn(pr(Lq=0)) == -1
    assert attn(pr(num_pages=0)) == -1
    assert attn(pr(), ws_bytes=16) == -4            # workspace too small
    assert lib.ic_sparse_attn_paged(1, 1, 1, 0, ctypes.byref(pr()), 0.1, 1, ws.addr, 1 << 16,
                                    None) == -1     # k = 0
    # indexer: tensor-core shapes only; fp8 needs both scales
    assert lib.ic_indexer_scores_paged(1, None, 1, 1, None, ic.F32, ctypes.byref(pr()), 64, 128,
                                       1, 512, ws.addr, 1 << 16, None) == -3
    assert lib.ic_indexer_scores_paged(1, None, 1, 1, None, ic.BF16, ctypes.byref(pr()), 64, 96,
                                       1, 512, ws.addr, 1 << 16, None) == -3
    assert lib.ic_indexer_scores_paged(1, None, 1, 1, None, ic.FP8_E4M3, ctypes.byref(pr()), 64,
                                       128, 1, 512, ws.addr, 1 << 16, None) == -1
    assert lib.ic_indexer_scores_paged(1, None, 1, 1, None, ic.BF16, ctypes.byref(pr()), 64, 128,
                                       1, 510, ws.addr, 1 << 16, None) == -1   # ld < T_max
    # top-k reads only the lengths: no block table needed, but a bad ld is refused
    assert lib.ic_topk_varlen(1, 510, ctypes.byref(pr(block_table=None)), 8, 1, ws.addr, 1 << 16,
                              None) == -1
    assert lib.ic_topk_varlen(1, 512, ctypes.byref(pr(seq_lens=None)), 8, 1, ws.addr, 1 << 16,
                              None) == -1
    # the stack: tensor-core shapes only, and patterns checked first
    sh = ic.StackShape(ic.Rows(2, 1, 511, 512), 64, 128, ic.BF16, 64, 128, 576, 512, ic.BF16,
                       576, 576, 0.04)
    big = _FakeTensor(ic.paged_workspace_size(sh, pr()))
    layers = (ic.LayerIO * 2)()
    assert lib.ic_layer_stack_forward_paged(b"SF", 2, layers, ctypes.byref(sh), ctypes.byref(pr()),
                                            1, None, big.addr, big.nbytes, None) == -2
    sh_f32 = ic.StackShape(ic.Rows(2, 1, 511, 512), 4, 32, ic.F32, 64, 8, 64, 64, ic.F32, 64, 64,
                           0.1)
    assert lib.ic_layer_stack_forward_paged(b"FS", 2, layers, ctypes.byref(sh_f32),
                                            ctypes.byref(pr()), 1, None, big.addr, big.nbytes,
                                            None) == -3
    assert lib.ic_layer_stack_forward_paged(b"FS", 2, layers, ctypes.byref(sh), ctypes.byref(pr()),
                                            1, None, big.addr, big.nbytes, None) == -1  # NULL layers
    # an empty batch is a no-op
    assert attn(pr(B=0, seq_lens=None, block_table=None)) == 0
    assert ic.kernel_launches(0) == before
    assert ic.paged_workspace_size(sh, pr()) >= ic.STATUS_BYTES + 2 * 512 * 4
