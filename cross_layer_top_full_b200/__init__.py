"""IndexCache on B200: Python binding of the C-ABI library ``libindexcache.so``.

Argument marshalling only: every step of the hot path runs in the library's
CUDA kernels.  PyTorch supplies device memory and streams.  If the library is
missing this package raises on first use; there is no CPU fallback.

Entry points mirror ``include/indexcache.h``:
``indexer_scores``, ``topk``, ``sparse_attn``, ``layer_stack_forward``,
their ``*_workspace_size`` queries, ``workspace_init``, ``read_status``,
``kernel_launches`` and ``status_string``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional, Sequence

__all__ = [
    "IcError", "lib", "library_path", "Rows", "StackShape", "LayerIO", "PagedRows", "paged_rows",
    "F32", "BF16", "FP8_E4M3", "STATUS_BYTES",
    "status_string", "version", "kernel_launches", "workspace_init", "read_status",
    "indexer_workspace_size", "indexer_scores", "topk_workspace_size", "topk",
    "indexer_topk_workspace_size", "indexer_topk",
    "sparse_attn_workspace_size", "sparse_attn", "sparse_attn_noalloc", "workspace_size",
    "layer_stack_forward", "indexer_scores_paged", "topk_varlen_workspace_size", "topk_varlen",
    "indexer_topk_paged_workspace_size", "indexer_topk_paged",
    "sparse_attn_paged_workspace_size", "sparse_attn_paged", "paged_workspace_size",
    "layer_stack_forward_paged",
]

F32, BF16, FP8_E4M3 = 0, 1, 2
STATUS_BYTES = 256
CUDA_ERROR = -5
_STATUS = {0: "IC_OK", -1: "IC_ERR_INVALID_ARG", -2: "IC_ERR_PATTERN", -3: "IC_ERR_UNSUPPORTED",
           -4: "IC_ERR_WORKSPACE", -5: "IC_ERR_CUDA", -6: "IC_ERR_INDEX_RANGE",
           -7: "IC_ERR_TIMEOUT"}

_HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    return os.environ.get("INDEXCACHE_LIB", os.path.join(_HERE, "libindexcache.so"))


class IcError(RuntimeError):
    def __init__(self, code: int, where: str, detail: str = ""):
        self.code = code
        super().__init__("%s failed: %s (%d)%s" % (where, _STATUS.get(code, "?"), code,
                                                   " [%s]" % detail if detail else ""))


class Rows(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Lq", ctypes.c_int), ("q_start", ctypes.c_int),
                ("T", ctypes.c_int)]


class StackShape(ctypes.Structure):
    _fields_ = [("rows", Rows), ("H_I", ctypes.c_int), ("d_I", ctypes.c_int),
                ("idx_dtype", ctypes.c_int), ("k", ctypes.c_int), ("Hq", ctypes.c_int),
                ("d_qk", ctypes.c_int), ("d_v", ctypes.c_int), ("attn_dtype", ctypes.c_int),
                ("k_row_stride", ctypes.c_int64), ("v_row_stride", ctypes.c_int64),
                ("scale", ctypes.c_float)]


class LayerIO(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("q_idx", "q_scale", "w", "k_idx", "k_scale", "q", "kmat", "vmat", "out")]


class PagedRows(ctypes.Structure):
    """ic_paged_rows: a variable-length batch over paged caches."""
    _fields_ = [("B", ctypes.c_int), ("Lq", ctypes.c_int), ("T_max", ctypes.c_int),
                ("seq_lens", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
                ("max_pages", ctypes.c_int), ("page_size", ctypes.c_int),
                ("num_pages", ctypes.c_int)]


_P = ctypes.c_void_p
_SIG = {
    "ic_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "ic_last_error": (ctypes.c_char_p, []),
    "ic_check_status": (ctypes.c_int, [_P, _P]),
    "ic_selftest_wait_timeout": (ctypes.c_int, [_P, ctypes.c_size_t, _P]),
    "ic_version": (ctypes.c_int, []),
    "ic_kernel_launches": (ctypes.c_uint64, [ctypes.c_int]),
    "ic_workspace_init": (ctypes.c_int, [_P, ctypes.c_size_t, _P]),
    "ic_read_status": (ctypes.c_int, [_P, _P, ctypes.POINTER(ctypes.c_int32)]),
    "ic_indexer_workspace_size": (ctypes.c_size_t, [Rows, ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "ic_indexer_scores": (ctypes.c_int, [_P, _P, _P, _P, _P, ctypes.c_int, Rows, ctypes.c_int,
                                         ctypes.c_int, _P, ctypes.c_int64, _P, ctypes.c_size_t, _P]),
    "ic_indexer_topk_workspace_size": (ctypes.c_size_t, [Rows, ctypes.c_int, ctypes.c_int,
                                                         ctypes.c_int, ctypes.c_int]),
    "ic_indexer_topk": (ctypes.c_int, [_P, _P, _P, _P, _P, ctypes.c_int, Rows, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_int, _P, _P, ctypes.c_size_t, _P]),
    "ic_topk_workspace_size": (ctypes.c_size_t, [Rows, ctypes.c_int]),
    "ic_topk": (ctypes.c_int, [_P, ctypes.c_int64, Rows, ctypes.c_int, _P, _P, ctypes.c_size_t, _P]),
    "ic_sparse_attn_workspace_size": (ctypes.c_size_t, [Rows, ctypes.c_int, ctypes.c_int,
                                                        ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "ic_sparse_attn": (ctypes.c_int, [_P, _P, ctypes.c_int64, _P, ctypes.c_int64, _P, ctypes.c_int,
                                      ctypes.c_int, Rows, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_float, _P, _P, ctypes.c_size_t, _P]),
    "ic_sparse_attn_noalloc": (ctypes.c_int, [_P, _P, _P, ctypes.c_int, Rows, ctypes.c_float, _P,
                                              _P, _P]),
    "ic_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(StackShape)]),
    "ic_layer_stack_forward": (ctypes.c_int, [ctypes.c_char_p, ctypes.c_int,
                                              ctypes.POINTER(LayerIO), ctypes.POINTER(StackShape),
                                              _P, ctypes.POINTER(_P), _P, ctypes.c_size_t, _P]),
    "ic_indexer_scores_paged": (ctypes.c_int, [_P, _P, _P, _P, _P, ctypes.c_int,
                                               ctypes.POINTER(PagedRows), ctypes.c_int,
                                               ctypes.c_int, _P, ctypes.c_int64, _P,
                                               ctypes.c_size_t, _P]),
    "ic_indexer_topk_paged_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(PagedRows),
                                                               ctypes.c_int]),
    "ic_indexer_topk_paged": (ctypes.c_int, [_P, _P, _P, _P, _P, ctypes.c_int,
                                             ctypes.POINTER(PagedRows), ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, _P, _P, ctypes.c_size_t, _P]),
    "ic_topk_varlen_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(PagedRows), ctypes.c_int]),
    "ic_topk_varlen": (ctypes.c_int, [_P, ctypes.c_int64, ctypes.POINTER(PagedRows), ctypes.c_int,
                                      _P, _P, ctypes.c_size_t, _P]),
    "ic_sparse_attn_paged_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(PagedRows),
                                                              ctypes.c_int]),
    "ic_sparse_attn_paged": (ctypes.c_int, [_P, _P, _P, ctypes.c_int, ctypes.POINTER(PagedRows),
                                            ctypes.c_float, _P, _P, ctypes.c_size_t, _P]),
    "ic_paged_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(StackShape),
                                                  ctypes.POINTER(PagedRows)]),
    "ic_layer_stack_forward_paged": (ctypes.c_int, [ctypes.c_char_p, ctypes.c_int,
                                                    ctypes.POINTER(LayerIO),
                                                    ctypes.POINTER(StackShape),
                                                    ctypes.POINTER(PagedRows), _P,
                                                    ctypes.POINTER(_P), _P, ctypes.c_size_t, _P]),
}

_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """The loaded library (loaded on first use; raises if it is missing)."""
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path):
            raise ImportError("libindexcache.so not built at %s: run "
                              "`python -m cross_layer_top_full_b200.build`" % path)
        handle = ctypes.CDLL(path)
        for name, (res, args) in _SIG.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


# --------------------------------------------------------------------------- helpers
def _ptr(x) -> Optional[int]:
    """Address of a tensor, or an int address passed through, or None.

    The library reads every array argument as a dense row-major DEVICE array,
    so a torch tensor in host memory (which a kernel would dereference as a
    bad address) or a strided view (which it would misread) is refused here,
    before the call."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if getattr(x, "is_cuda", True) is False:
        raise ValueError("expected a CUDA tensor, got one on %s" % x.device)
    contiguous = getattr(x, "is_contiguous", None)
    if contiguous is not None and not contiguous():
        raise ValueError("expected a contiguous tensor, got shape %s with strides %s"
                         % (tuple(x.shape), tuple(x.stride())))
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        if torch.cuda.is_available():
            return torch.cuda.current_stream().cuda_stream
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _nbytes(x) -> int:
    return x.numel() * x.element_size()


def _check(code: int, where: str) -> None:
    if code != 0:
        detail = lib().ic_last_error().decode() if code == CUDA_ERROR else ""
        raise IcError(code, where, detail)


def _rows(rows) -> Rows:
    if isinstance(rows, Rows):
        return rows
    B, Lq, q_start, T = rows
    return Rows(int(B), int(Lq), int(q_start), int(T))


def _dtype_of(t) -> int:
    import torch
    return {torch.float32: F32, torch.bfloat16: BF16, torch.uint8: FP8_E4M3,
            torch.float8_e4m3fn: FP8_E4M3}[t.dtype]


# --------------------------------------------------------------------------- API
def status_string(code: int) -> str:
    return lib().ic_status_string(code).decode()


def version() -> int:
    return lib().ic_version()


def kernel_launches(kind: int = 0) -> int:
    return int(lib().ic_kernel_launches(kind))


def workspace_init(ws, stream=None) -> None:
    _check(lib().ic_workspace_init(_ptr(ws), _nbytes(ws), _stream(stream)), "ic_workspace_init")


def read_status(ws, stream=None) -> int:
    """Raw device status bits (0 = clean); clears them."""
    v = ctypes.c_int32(0)
    code = lib().ic_read_status(_ptr(ws), _stream(stream), ctypes.byref(v))
    if code not in (0, -6, -7):
        raise IcError(code, "ic_read_status")
    return int(v.value)


def selftest_wait_timeout(ws, stream=None) -> None:
    """Launch the failure-path self-test (a pipeline wait that never
    completes and gives up after about 1 s); read the result with read_status."""
    _check(lib().ic_selftest_wait_timeout(_ptr(ws), _nbytes(ws), _stream(stream)),
           "ic_selftest_wait_timeout")


def indexer_workspace_size(rows, H_I: int, d_I: int, dtype: int) -> int:
    return int(lib().ic_indexer_workspace_size(_rows(rows), H_I, d_I, dtype))


def indexer_scores(q_idx, w, k_idx, rows, scores, ws, *, q_scale=None, k_scale=None,
                   dtype: Optional[int] = None, ld_scores: Optional[int] = None,
                   stream=None) -> None:
    """scores[b,i,s] = sum_h w * ReLU(q_idx[b,i,h] . k_idx[b,s]) for s <= q_start+i."""
    r = _rows(rows)
    dt = _dtype_of(q_idx) if dtype is None else dtype
    H_I, d_I = q_idx.shape[-2], q_idx.shape[-1]
    ld = scores.shape[-1] if ld_scores is None else ld_scores
    _check(lib().ic_indexer_scores(_ptr(q_idx), _ptr(q_scale), _ptr(w), _ptr(k_idx), _ptr(k_scale),
                                   dt, r, H_I, d_I, _ptr(scores), ld, _ptr(ws), _nbytes(ws),
                                   _stream(stream)), "ic_indexer_scores")


def indexer_topk_workspace_size(rows, H_I: int, d_I: int, dtype: int, k: int) -> int:
    return int(lib().ic_indexer_topk_workspace_size(_rows(rows), H_I, d_I, dtype, k))


def indexer_topk(q_idx, w, k_idx, rows, k: int, idx, ws, *, q_scale=None, k_scale=None,
                 dtype: Optional[int] = None, stream=None) -> None:
    """An F layer's key selection: indexer scores and top-k in one call (one
    fused kernel for decode rows)."""
    r = _rows(rows)
    dt = _dtype_of(q_idx) if dtype is None else dtype
    H_I, d_I = q_idx.shape[-2], q_idx.shape[-1]
    _check(lib().ic_indexer_topk(_ptr(q_idx), _ptr(q_scale), _ptr(w), _ptr(k_idx), _ptr(k_scale),
                                 dt, r, H_I, d_I, k, _ptr(idx), _ptr(ws), _nbytes(ws),
                                 _stream(stream)), "ic_indexer_topk")


def topk_workspace_size(rows, k: int) -> int:
    return int(lib().ic_topk_workspace_size(_rows(rows), k))


def topk(scores, rows, k: int, idx, ws, *, ld_scores: Optional[int] = None, stream=None) -> None:
    ld = scores.shape[-1] if ld_scores is None else ld_scores
    _check(lib().ic_topk(_ptr(scores), ld, _rows(rows), k, _ptr(idx), _ptr(ws), _nbytes(ws),
                         _stream(stream)), "ic_topk")


def sparse_attn_workspace_size(rows, k: int, Hq: int, d_qk: int, d_v: int, dtype: int) -> int:
    return int(lib().ic_sparse_attn_workspace_size(_rows(rows), k, Hq, d_qk, d_v, dtype))


def sparse_attn(q, kmat, k_row_stride: int, vmat, v_row_stride: int, idx, rows, d_v: int,
                scale: float, out, ws, *, dtype: Optional[int] = None, stream=None) -> None:
    """Sparse MQA attention of q [B,Lq,Hq,d_qk] over the keys listed in idx."""
    dt = _dtype_of(q) if dtype is None else dtype
    Hq, d_qk = q.shape[-2], q.shape[-1]
    k = idx.shape[-1]
    _check(lib().ic_sparse_attn(_ptr(q), _ptr(kmat), k_row_stride, _ptr(vmat), v_row_stride,
                                _ptr(idx), k, dt, _rows(rows), Hq, d_qk, d_v, float(scale),
                                _ptr(out), _ptr(ws), _nbytes(ws), _stream(stream)),
           "ic_sparse_attn")


def sparse_attn_noalloc(q, kv, idx, rows, scale: float, out, *, device_status=None,
                        stream=None) -> None:
    """Latent sparse MQA attention (bf16, 128 heads, 576-wide KV rows) without
    a workspace: for callers that may not allocate device memory.  Its split-k
    partials live in a fixed device array inside the library, shared by all
    calls (serialise calls on one stream)."""
    k = idx.shape[-1]
    _check(lib().ic_sparse_attn_noalloc(_ptr(q), _ptr(kv), _ptr(idx), k, _rows(rows),
                                        float(scale), _ptr(out), _ptr(device_status),
                                        _stream(stream)), "ic_sparse_attn_noalloc")


def workspace_size(shape: StackShape) -> int:
    return int(lib().ic_workspace_size(ctypes.byref(shape)))


def layer_stack_forward(pattern: str, layers: Sequence[Dict], shape: StackShape, idx_buf, ws, *,
                        idx_out: Optional[List] = None, stream=None) -> None:
    """Run the F/S layer stack.  Each layer dict may hold q_idx, q_scale, w,
    k_idx, k_scale (F layers), q, kmat, vmat, out (tensors or int addresses)."""
    n = len(layers)
    arr = (LayerIO * max(1, n))()
    for l, L in enumerate(layers):
        for name, _ in LayerIO._fields_:
            setattr(arr[l], name, _ptr(L.get(name)))
    outs = None
    if idx_out is not None:
        outs = (_P * max(1, n))(*[_ptr(x) for x in idx_out])
    _check(lib().ic_layer_stack_forward(pattern.encode(), n, arr, ctypes.byref(shape),
                                        _ptr(idx_buf), outs, _ptr(ws), _nbytes(ws),
                                        _stream(stream)), "ic_layer_stack_forward")


# --------------------------------------------------------------------------- paged / varlen
def paged_rows(seq_lens, block_table, T_max: int, page_size: int, num_pages: int,
               Lq: int = 1) -> PagedRows:
    """ic_paged_rows for seq_lens [B] int32 and block_table [B, max_pages]
    int32 (device tensors, kept alive by the caller)."""
    B = int(seq_lens.shape[0])
    max_pages = int(block_table.shape[1]) if block_table is not None else 0
    return PagedRows(B, int(Lq), int(T_max), _ptr(seq_lens), _ptr(block_table), max_pages,
                     int(page_size), int(num_pages))


def indexer_scores_paged(q_idx, w, k_pages, pr: PagedRows, scores, ws, *, q_scale=None,
                         k_scale_pages=None, dtype: Optional[int] = None,
                         ld_scores: Optional[int] = None, stream=None) -> None:
    dt = _dtype_of(q_idx) if dtype is None else dtype
    H_I, d_I = q_idx.shape[-2], q_idx.shape[-1]
    ld = scores.shape[-1] if ld_scores is None else ld_scores
    _check(lib().ic_indexer_scores_paged(_ptr(q_idx), _ptr(q_scale), _ptr(w), _ptr(k_pages),
                                         _ptr(k_scale_pages), dt, ctypes.byref(pr), H_I, d_I,
                                         _ptr(scores), ld, _ptr(ws), _nbytes(ws), _stream(stream)),
           "ic_indexer_scores_paged")


def indexer_topk_paged_workspace_size(pr: PagedRows, k: int) -> int:
    return int(lib().ic_indexer_topk_paged_workspace_size(ctypes.byref(pr), k))


def indexer_topk_paged(q_idx, w, k_pages, pr: PagedRows, k: int, idx, ws, *, q_scale=None,
                       k_scale_pages=None, dtype: Optional[int] = None, stream=None) -> None:
    dt = _dtype_of(q_idx) if dtype is None else dtype
    H_I, d_I = q_idx.shape[-2], q_idx.shape[-1]
    _check(lib().ic_indexer_topk_paged(_ptr(q_idx), _ptr(q_scale), _ptr(w), _ptr(k_pages),
                                       _ptr(k_scale_pages), dt, ctypes.byref(pr), H_I, d_I, k,
                                       _ptr(idx), _ptr(ws), _nbytes(ws), _stream(stream)),
           "ic_indexer_topk_paged")


def topk_varlen_workspace_size(pr: PagedRows, k: int) -> int:
    return int(lib().ic_topk_varlen_workspace_size(ctypes.byref(pr), k))


def topk_varlen(scores, pr: PagedRows, k: int, idx, ws, *, ld_scores: Optional[int] = None,
                stream=None) -> None:
    ld = scores.shape[-1] if ld_scores is None else ld_scores
    _check(lib().ic_topk_varlen(_ptr(scores), ld, ctypes.byref(pr), k, _ptr(idx), _ptr(ws),
                                _nbytes(ws), _stream(stream)), "ic_topk_varlen")


def sparse_attn_paged_workspace_size(pr: PagedRows, k: int) -> int:
    return int(lib().ic_sparse_attn_paged_workspace_size(ctypes.byref(pr), k))


def sparse_attn_paged(q, kv_pages, idx, pr: PagedRows, scale: float, out, ws, *,
                      stream=None) -> None:
    _check(lib().ic_sparse_attn_paged(_ptr(q), _ptr(kv_pages), _ptr(idx), idx.shape[-1],
                                      ctypes.byref(pr), float(scale), _ptr(out), _ptr(ws),
                                      _nbytes(ws), _stream(stream)), "ic_sparse_attn_paged")


def paged_workspace_size(shape: StackShape, pr: PagedRows) -> int:
    return int(lib().ic_paged_workspace_size(ctypes.byref(shape), ctypes.byref(pr)))


def layer_stack_forward_paged(pattern: str, layers: Sequence[Dict], shape: StackShape,
                              pr: PagedRows, idx_buf, ws, *, idx_out: Optional[List] = None,
                              stream=None) -> None:
    """The F/S layer stack over paged caches: each layer dict holds q_idx,
    q_scale, w, k_idx (= that layer's paged k_I), k_scale (its paged scales),
    q, kmat (= its paged KV rows) and out."""
    n = len(layers)
    arr = (LayerIO * max(1, n))()
    for l, L in enumerate(layers):
        for name, _ in LayerIO._fields_:
            setattr(arr[l], name, _ptr(L.get(name)))
    outs = None
    if idx_out is not None:
        outs = (_P * max(1, n))(*[_ptr(x) for x in idx_out])
    _check(lib().ic_layer_stack_forward_paged(pattern.encode(), n, arr, ctypes.byref(shape),
                                              ctypes.byref(pr), _ptr(idx_buf), outs, _ptr(ws),
                                              _nbytes(ws), _stream(stream)),
           "ic_layer_stack_forward_paged")
