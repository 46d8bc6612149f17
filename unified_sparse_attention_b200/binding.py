"""ctypes binding of liblserve.so: the C ABI's entry points under the same names.

Argument marshalling only.  Tensors must already live on the CUDA device in the
dtype and layout ``include/lserve.h`` gives; nothing here computes any part of
the method, and a missing library or device raises instead of falling back.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))

LSERVE_HEAD_DENSE = 0
LSERVE_HEAD_STREAMING = 1
PAGE = 64

STATUS = {
    0: "LSERVE_OK",
    1: "LSERVE_ERR_INVALID_ARG",
    2: "LSERVE_ERR_UNSUPPORTED",
    3: "LSERVE_ERR_WORKSPACE",
    4: "LSERVE_ERR_CUDA",
    5: "LSERVE_ERR_DEVICE_TIMEOUT",
    6: "LSERVE_ERR_DEVICE_BOUNDS",
}

# Every symbol include/lserve.h declares.
EXPORTED_SYMBOLS = (
    "lserve_prefill_workspace_size",
    "lserve_prefill",
    "lserve_prefill_tile_lists",
    "lserve_cra_workspace_size",
    "lserve_cra",
    "lserve_vslash_workspace_size",
    "lserve_build_vslash_mask",
    "lserve_update_page_stats",
    "lserve_decode_max_selected",
    "lserve_decode_workspace_size",
    "lserve_decode",
    "lserve_decode_noalloc",
    "lserve_decode_reuse",
    "lserve_quantize_pages_int4",
    "lserve_decode_int4",
    "lserve_get_device_status",
    "lserve_last_error_string",
    "lserve_version",
)


class LServeError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("S", ctypes.c_int32), ("Hq", ctypes.c_int32),
                ("Hkv", ctypes.c_int32), ("d", ctypes.c_int32), ("scale", ctypes.c_float),
                ("lambda_tiles", ctypes.c_int32)]


class DecodeArgs(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("d", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("maxP", ctypes.c_int32),
                ("q", ctypes.c_void_p), ("k_pages", ctypes.c_void_p), ("v_pages", ctypes.c_void_p),
                ("page_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p), ("stats", ctypes.c_void_p),
                ("head_kind", ctypes.c_void_p), ("sink", ctypes.c_int32), ("local", ctypes.c_int32),
                ("token_budget", ctypes.c_int32), ("scale", ctypes.c_float)]


_lib = None


def library_path() -> str:
    return os.environ.get("LSERVE_LIBRARY", os.path.join(_HERE, "liblserve.so"))


def load_library():
    """Load liblserve.so once (raises OSError with the path when it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise OSError(f"liblserve.so not found at {path}; build it with "
                      f"`python -m unified_sparse_attention_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    sig = {
        "lserve_prefill_workspace_size": (sz, [ctypes.POINTER(Shape)]),
        "lserve_prefill": (i32, [ctypes.POINTER(Shape), vp, vp, vp, vp, i32, i32, vp, vp, vp, vp, sz, vp]),
        "lserve_cra_workspace_size": (sz, [ctypes.POINTER(Shape)]),
        "lserve_cra": (i32, [ctypes.POINTER(Shape), vp, vp, vp, vp, i32, i32, vp, vp, vp, vp, sz, vp]),
        "lserve_vslash_workspace_size": (sz, [ctypes.POINTER(Shape), i32]),
        "lserve_build_vslash_mask": (i32, [ctypes.POINTER(Shape), vp, vp, vp, i32, ctypes.c_float, vp, vp, vp, vp,
                                           vp, sz, vp]),
        "lserve_prefill_tile_lists": (i32, [ctypes.POINTER(Shape), vp, i32, i32, vp, vp, vp, ctypes.c_int64,
                                            vp, sz, vp]),
        "lserve_update_page_stats": (i32, [i32, i32, i32, i32, vp, vp, i32, vp, i32, vp, vp, vp]),
        "lserve_decode_max_selected": (i32, [ctypes.POINTER(DecodeArgs)]),
        "lserve_decode_workspace_size": (sz, [ctypes.POINTER(DecodeArgs)]),
        "lserve_decode": (i32, [ctypes.POINTER(DecodeArgs), vp, vp, vp, vp, vp, sz, vp]),
        "lserve_decode_noalloc": (i32, [ctypes.POINTER(DecodeArgs), vp, vp, vp, vp, vp]),
        "lserve_decode_reuse": (i32, [ctypes.POINTER(DecodeArgs), vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "lserve_quantize_pages_int4": (i32, [i32, i32, i32, i32, vp, vp, vp, i32, vp, i32, vp, vp, vp, vp, vp, vp,
                                             vp]),
        "lserve_decode_int4": (i32, [ctypes.POINTER(DecodeArgs), vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "lserve_get_device_status": (i32, [vp]),
        "lserve_last_error_string": (ctypes.c_char_p, []),
        "lserve_version": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def lserve_last_error_string() -> str:
    return load_library().lserve_last_error_string().decode()


def lserve_version() -> str:
    return load_library().lserve_version().decode()


def _check(status: int):
    if status != 0:
        raise LServeError(status, lserve_last_error_string())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t: torch.Tensor, name: str, dtype: torch.dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _workspace(nbytes: int, device, workspace: Optional[torch.Tensor]) -> torch.Tensor:
    if workspace is not None:
        return workspace
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


# ---------------------------------------------------------------- prefill

def _shape(q, k, scale, lambda_tiles=False):
    B, S, Hq, d = q.shape
    return Shape(B, S, Hq, k.shape[2], d, float(scale), 1 if lambda_tiles else 0)


def lserve_prefill_workspace_size(B: int, S: int, Hq: int, Hkv: int, d: int) -> int:
    return int(load_library().lserve_prefill_workspace_size(ctypes.byref(Shape(B, S, Hq, Hkv, d, 0.0, 0))))


def lserve_prefill(q, k, v, head_kind, sink: int, local: int, block_mask=None, out=None, lse=None,
                   scale: float = 0.0, workspace=None, stream=None, return_lse: bool = False,
                   lambda_tiles: bool = False):
    """Block-sparse causal prefill; see include/lserve.h.  Returns out (and lse).
    lambda_tiles: streaming heads keep whole tiles of the Lambda support."""
    lib = load_library()
    _dev(q, "q", torch.bfloat16)
    B, S, Hq, d = q.shape
    Hkv = k.shape[2]
    _dev(k, "k", torch.bfloat16, (B, S, Hkv, d))
    _dev(v, "v", torch.bfloat16, (B, S, Hkv, d))
    _dev(head_kind, "head_kind", torch.uint8, (Hkv,))
    if block_mask is not None:
        _dev(block_mask, "block_mask", torch.uint8, (B, Hkv, S // PAGE, S // PAGE))
    out = torch.empty_like(q) if out is None else _dev(out, "out", torch.bfloat16, q.shape)
    if lse is None and return_lse:
        lse = torch.empty(B, Hq, S, dtype=torch.float32, device=q.device)
    if lse is not None:
        _dev(lse, "lse", torch.float32, (B, Hq, S))
    shape = _shape(q, k, scale, lambda_tiles)
    need = int(lib.lserve_prefill_workspace_size(ctypes.byref(shape)))
    ws = _workspace(need, q.device, workspace)
    _check(lib.lserve_prefill(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(head_kind), int(sink),
                              int(local), _ptr(block_mask), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                              _stream(stream)))
    return (out, lse) if (return_lse or lse is not None) else out


def lserve_cra_workspace_size(B: int, S: int, Hq: int, Hkv: int, d: int) -> int:
    return int(load_library().lserve_cra_workspace_size(ctypes.byref(Shape(B, S, Hq, Hkv, d, 0.0, 0))))


def lserve_cra(q, k, v, head_kind, sink: int, local: int, block_mask=None, scale: float = 0.0,
               return_retained: bool = False, workspace=None, stream=None, lambda_tiles: bool = False):
    """Cumulative residual attention of a sparse prefill mask; see include/lserve.h.
    Returns cra fp32[B, Hq] (and the per-row retained mass fp32[B, Hq, S])."""
    lib = load_library()
    _dev(q, "q", torch.bfloat16)
    B, S, Hq, d = q.shape
    Hkv = k.shape[2]
    _dev(k, "k", torch.bfloat16, (B, S, Hkv, d))
    _dev(v, "v", torch.bfloat16, (B, S, Hkv, d))
    _dev(head_kind, "head_kind", torch.uint8, (Hkv,))
    if block_mask is not None:
        _dev(block_mask, "block_mask", torch.uint8, (B, Hkv, S // PAGE, S // PAGE))
    cra = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    retained = torch.empty(B, Hq, S, dtype=torch.float32, device=q.device) if return_retained else None
    shape = _shape(q, k, scale, lambda_tiles)
    need = int(lib.lserve_cra_workspace_size(ctypes.byref(shape)))
    ws = _workspace(need, q.device, workspace)
    _check(lib.lserve_cra(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(head_kind), int(sink), int(local),
                          _ptr(block_mask), _ptr(retained), _ptr(cra), _ptr(ws), ws.numel(), _stream(stream)))
    return (cra, retained) if return_retained else cra


def lserve_vslash_workspace_size(B: int, S: int, Hq: int, Hkv: int, d: int, sample_stride: int) -> int:
    return int(load_library().lserve_vslash_workspace_size(ctypes.byref(Shape(B, S, Hq, Hkv, d, 0.0, 0)),
                                                           int(sample_stride)))


def lserve_build_vslash_mask(q, k, head_kind, sample_stride: int, tau: float, scale: float = 0.0, block_mask=None,
                             workspace=None, stream=None):
    """Vertical-slash block mask of the dense heads from sampled queries; see include/lserve.h.
    Returns (block_mask uint8[B, Hkv, S/64, S/64], cra fp32[B, Hkv], n_columns, n_slashes int32[B, Hkv])."""
    lib = load_library()
    _dev(q, "q", torch.bfloat16)
    B, S, Hq, d = q.shape
    Hkv = k.shape[2]
    _dev(k, "k", torch.bfloat16, (B, S, Hkv, d))
    _dev(head_kind, "head_kind", torch.uint8, (Hkv,))
    n = S // PAGE
    dev = q.device
    block_mask = torch.empty(B, Hkv, n, n, dtype=torch.uint8, device=dev) if block_mask is None else \
        _dev(block_mask, "block_mask", torch.uint8, (B, Hkv, n, n))
    cra = torch.empty(B, Hkv, dtype=torch.float32, device=dev)
    ncol = torch.empty(B, Hkv, dtype=torch.int32, device=dev)
    nsla = torch.empty(B, Hkv, dtype=torch.int32, device=dev)
    shape = _shape(q, k, scale)
    need = int(lib.lserve_vslash_workspace_size(ctypes.byref(shape), int(sample_stride)))
    ws = _workspace(max(need, 1), dev, workspace)
    _check(lib.lserve_build_vslash_mask(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(head_kind), int(sample_stride),
                                        float(tau), _ptr(block_mask), _ptr(cra), _ptr(ncol), _ptr(nsla), _ptr(ws),
                                        ws.numel(), _stream(stream)))
    return block_mask, cra, ncol, nsla


def lserve_prefill_tile_lists(B, S, Hq, Hkv, d, head_kind, sink, local, block_mask=None, stream=None):
    """Kept-tile CSR (row_offsets int32[R+1], tile_cols uint16[nnz]) on the device."""
    lib = load_library()
    _dev(head_kind, "head_kind", torch.uint8, (Hkv,))
    n = S // PAGE
    if block_mask is not None:
        _dev(block_mask, "block_mask", torch.uint8, (B, Hkv, n, n))
    dev = head_kind.device
    R = B * Hkv * n
    max_nnz = R * (n + 1) // 2
    offsets = torch.empty(R + 1, dtype=torch.int32, device=dev)
    cols = torch.empty(max(max_nnz, 1), dtype=torch.int16, device=dev)
    shape = Shape(B, S, Hq, Hkv, d, 0.0, 0)
    ws = _workspace(lib.lserve_prefill_workspace_size(ctypes.byref(shape)), dev, None)
    _check(lib.lserve_prefill_tile_lists(ctypes.byref(shape), _ptr(head_kind), int(sink), int(local),
                                         _ptr(block_mask), _ptr(offsets), _ptr(cols), max_nnz, _ptr(ws),
                                         ws.numel(), _stream(stream)))
    return offsets, cols


# ------------------------------------------------------------ page stats

def lserve_update_page_stats(k_pages, page_table, seq_lens, head_kind, stats=None, first_logical_page: int = 0,
                             stream=None):
    """Per-logical-page key min/max; returns stats bf16[NP, Hkv, 4, 2, d]."""
    lib = load_library()
    _dev(k_pages, "k_pages", torch.bfloat16)
    NP, Hkv, P, d = k_pages.shape
    if P != PAGE:
        raise ValueError("k_pages must have 64-token pages")
    _dev(page_table, "page_table", torch.int32)
    B, maxP = page_table.shape
    _dev(seq_lens, "seq_lens", torch.int32, (B,))
    _dev(head_kind, "head_kind", torch.uint8, (Hkv,))
    if stats is None:
        stats = torch.full((NP, Hkv, 4, 2, d), float("nan"), dtype=torch.bfloat16, device=k_pages.device)
    _dev(stats, "stats", torch.bfloat16, (NP, Hkv, 4, 2, d))
    _check(lib.lserve_update_page_stats(B, Hkv, d, NP, _ptr(k_pages), _ptr(page_table), maxP, _ptr(seq_lens),
                                        int(first_logical_page), _ptr(head_kind), _ptr(stats), _stream(stream)))
    return stats


# ----------------------------------------------------------------- decode

def _decode_args(q, k_pages, v_pages, page_table, seq_lens, stats, head_kind, sink, local, token_budget, scale):
    _dev(q, "q", torch.bfloat16)
    B, Hq, d = q.shape
    _dev(k_pages, "k_pages", torch.bfloat16)
    NP, Hkv, P, d2 = k_pages.shape
    if P != PAGE or d2 != d:
        raise ValueError("k_pages must be [NP, Hkv, 64, d]")
    _dev(v_pages, "v_pages", torch.bfloat16, k_pages.shape)
    _dev(page_table, "page_table", torch.int32)
    if page_table.shape[0] != B:
        raise ValueError("page_table must be [B, maxP]")
    _dev(seq_lens, "seq_lens", torch.int32, (B,))
    if stats is not None:
        _dev(stats, "stats", torch.bfloat16, (NP, Hkv, 4, 2, d))
    _dev(head_kind, "head_kind", torch.uint8, (Hkv,))
    return DecodeArgs(B, Hq, Hkv, d, NP, page_table.shape[1], q.data_ptr(), k_pages.data_ptr(),
                      v_pages.data_ptr(), page_table.data_ptr(), seq_lens.data_ptr(),
                      None if stats is None else stats.data_ptr(),
                      head_kind.data_ptr(), int(sink), int(local), int(token_budget), float(scale))


def lserve_decode_max_selected(B, Hq, Hkv, d, num_pages, maxP, sink, local, token_budget) -> int:
    a = DecodeArgs(B, Hq, Hkv, d, num_pages, maxP, None, None, None, None, None, None, None, sink, local,
                   token_budget, 0.0)
    return int(load_library().lserve_decode_max_selected(ctypes.byref(a)))


def lserve_decode_workspace_size(q, k_pages, v_pages, page_table, seq_lens, stats, head_kind, sink, local,
                                 token_budget, scale=0.0) -> int:
    a = _decode_args(q, k_pages, v_pages, page_table, seq_lens, stats, head_kind, sink, local, token_budget, scale)
    return int(load_library().lserve_decode_workspace_size(ctypes.byref(a)))


def lserve_decode(q, k_pages, v_pages, page_table, seq_lens, stats, head_kind, sink: int, local: int,
                  token_budget: int, scale: float = 0.0, out=None, lse=None, sel_out=None, sel_n=None,
                  workspace=None, stream=None, return_selection: bool = False):
    """One sparse decode step; see include/lserve.h.  Returns out (and lse, sel, sel_n)."""
    lib = load_library()
    a = _decode_args(q, k_pages, v_pages, page_table, seq_lens, stats, head_kind, sink, local, token_budget, scale)
    B, Hq, d = q.shape
    Hkv = a.Hkv
    out = torch.empty_like(q) if out is None else _dev(out, "out", torch.bfloat16, q.shape)
    if lse is not None:
        _dev(lse, "lse", torch.float32, (B, Hq))
    kcap = int(lib.lserve_decode_max_selected(ctypes.byref(a)))
    if return_selection and sel_out is None:
        sel_out = torch.empty(B, Hkv, kcap, dtype=torch.int32, device=q.device)
        sel_n = torch.empty(B, Hkv, dtype=torch.int32, device=q.device) if sel_n is None else sel_n
    if sel_out is not None:
        _dev(sel_out, "sel_out", torch.int32, (B, Hkv, kcap))
    if sel_n is not None:
        _dev(sel_n, "sel_n", torch.int32, (B, Hkv))
    need = int(lib.lserve_decode_workspace_size(ctypes.byref(a)))
    if need == 0:   # invalid arguments: let the library report which
        _check(lib.lserve_decode(ctypes.byref(a), _ptr(out), None, None, None, None, 0, _stream(stream)))
    ws = _workspace(need, q.device, workspace)
    _check(lib.lserve_decode(ctypes.byref(a), _ptr(out), _ptr(lse), _ptr(sel_out), _ptr(sel_n), _ptr(ws),
                             ws.numel(), _stream(stream)))
    if return_selection:
        return out, lse, sel_out, sel_n
    return out


def lserve_decode_reuse(q, k_pages, v_pages, page_table, seq_lens, head_kind, sink: int, local: int,
                        token_budget: int, sel, sel_n, scale: float = 0.0, out=None, lse=None, sel_out=None,
                        sel_n_out=None, workspace=None, stream=None):
    """A decode step that keeps an earlier page selection (`sel`, `sel_n`, as
    lserve_decode returned them); see include/lserve.h.  Returns out."""
    lib = load_library()
    a = _decode_args(q, k_pages, v_pages, page_table, seq_lens, None, head_kind, sink, local, token_budget, scale)
    B, Hq, d = q.shape
    Hkv = a.Hkv
    out = torch.empty_like(q) if out is None else _dev(out, "out", torch.bfloat16, q.shape)
    if lse is not None:
        _dev(lse, "lse", torch.float32, (B, Hq))
    kcap = int(lib.lserve_decode_max_selected(ctypes.byref(a)))
    _dev(sel, "sel", torch.int32, (B, Hkv, kcap))
    _dev(sel_n, "sel_n", torch.int32, (B, Hkv))
    if sel_out is not None:
        _dev(sel_out, "sel_out", torch.int32, (B, Hkv, kcap))
    if sel_n_out is not None:
        _dev(sel_n_out, "sel_n_out", torch.int32, (B, Hkv))
    need = int(lib.lserve_decode_workspace_size(ctypes.byref(a)))
    ws = _workspace(need, q.device, workspace)
    _check(lib.lserve_decode_reuse(ctypes.byref(a), _ptr(sel), _ptr(sel_n), _ptr(out), _ptr(lse), _ptr(sel_out),
                                   _ptr(sel_n_out), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def lserve_quantize_pages_int4(k_pages, v_pages, page_table, seq_lens, head_kind, first_page: int = 0, kq=None,
                               kpar=None, vq=None, vpar=None, stats=None, stream=None):
    """INT4 codes, steps and offsets of the pages each sequence holds, and the
    page summaries of the dequantised keys; see include/lserve.h.
    Returns (kq, kpar, vq, vpar, stats); buffers passed in are updated in place."""
    lib = load_library()
    _dev(k_pages, "k_pages", torch.bfloat16)
    NP, Hkv, P, d = k_pages.shape
    if P != PAGE:
        raise ValueError("k_pages must be [NP, Hkv, 64, d]")
    _dev(v_pages, "v_pages", torch.bfloat16, k_pages.shape)
    _dev(page_table, "page_table", torch.int32)
    B, maxP = page_table.shape
    _dev(seq_lens, "seq_lens", torch.int32, (B,))
    _dev(head_kind, "head_kind", torch.uint8, (Hkv,))
    dev = k_pages.device
    mk = lambda t, name, dt, shape: (torch.zeros(shape, dtype=dt, device=dev) if t is None
                                     else _dev(t, name, dt, shape))
    kq = mk(kq, "kq", torch.uint8, (NP, Hkv, P, d // 2))
    vq = mk(vq, "vq", torch.uint8, (NP, Hkv, P * d // 2))
    kpar = mk(kpar, "kpar", torch.float32, (NP, Hkv, 2, d))
    vpar = mk(vpar, "vpar", torch.float32, (NP, Hkv, P, 2))
    stats = mk(stats, "stats", torch.bfloat16, (NP, Hkv, 4, 2, d))
    _check(lib.lserve_quantize_pages_int4(B, Hkv, d, NP, _ptr(k_pages), _ptr(v_pages), _ptr(page_table), maxP,
                                          _ptr(seq_lens), int(first_page), _ptr(head_kind), _ptr(kq), _ptr(kpar),
                                          _ptr(vq), _ptr(vpar), _ptr(stats), _stream(stream)))
    return kq, kpar, vq, vpar, stats


def lserve_decode_int4(q, kq, vq, kpar, vpar, page_table, seq_lens, stats, head_kind, sink: int, local: int,
                       token_budget: int, scale: float = 0.0, out=None, lse=None, sel_out=None, sel_n=None,
                       workspace=None, stream=None, return_selection: bool = False):
    """lserve_decode over INT4 pages (as lserve_quantize_pages_int4 wrote them);
    see include/lserve.h.  Returns out (and lse, sel, sel_n)."""
    lib = load_library()
    _dev(q, "q", torch.bfloat16)
    B, Hq, d = q.shape
    _dev(kq, "kq", torch.uint8)
    NP, Hkv, P, d2 = kq.shape
    if P != PAGE or 2 * d2 != d:
        raise ValueError("kq must be [NP, Hkv, 64, d/2]")
    _dev(vq, "vq", torch.uint8, (NP, Hkv, P * d2))
    _dev(kpar, "kpar", torch.float32, (NP, Hkv, 2, d))
    _dev(vpar, "vpar", torch.float32, (NP, Hkv, P, 2))
    _dev(page_table, "page_table", torch.int32)
    if page_table.shape[0] != B:
        raise ValueError("page_table must be [B, maxP]")
    _dev(seq_lens, "seq_lens", torch.int32, (B,))
    _dev(stats, "stats", torch.bfloat16, (NP, Hkv, 4, 2, d))
    _dev(head_kind, "head_kind", torch.uint8, (Hkv,))
    a = DecodeArgs(B, Hq, Hkv, d, NP, page_table.shape[1], q.data_ptr(), kq.data_ptr(), vq.data_ptr(),
                   page_table.data_ptr(), seq_lens.data_ptr(), stats.data_ptr(), head_kind.data_ptr(), int(sink),
                   int(local), int(token_budget), float(scale))
    out = torch.empty_like(q) if out is None else _dev(out, "out", torch.bfloat16, q.shape)
    if lse is not None:
        _dev(lse, "lse", torch.float32, (B, Hq))
    kcap = int(lib.lserve_decode_max_selected(ctypes.byref(a)))
    if return_selection and sel_out is None:
        sel_out = torch.empty(B, Hkv, kcap, dtype=torch.int32, device=q.device)
        sel_n = torch.empty(B, Hkv, dtype=torch.int32, device=q.device) if sel_n is None else sel_n
    if sel_out is not None:
        _dev(sel_out, "sel_out", torch.int32, (B, Hkv, kcap))
    if sel_n is not None:
        _dev(sel_n, "sel_n", torch.int32, (B, Hkv))
    need = int(lib.lserve_decode_workspace_size(ctypes.byref(a)))
    if need == 0:   # invalid arguments: let the library report which
        _check(lib.lserve_decode_int4(ctypes.byref(a), _ptr(kpar), _ptr(vpar), _ptr(out), None, None, None, None, 0,
                                      _stream(stream)))
    ws = _workspace(need, q.device, workspace)
    _check(lib.lserve_decode_int4(ctypes.byref(a), _ptr(kpar), _ptr(vpar), _ptr(out), _ptr(lse), _ptr(sel_out),
                                  _ptr(sel_n), _ptr(ws), ws.numel(), _stream(stream)))
    if return_selection:
        return out, lse, sel_out, sel_n
    return out


NOALLOC_SCRATCH_BYTES = 16 << 20


def lserve_decode_noalloc(q, k_pages, v_pages, page_table, seq_lens, stats, head_kind, sink: int, local: int,
                          token_budget: int, out, scale: float = 0.0, lse=None, sel_out=None, sel_n=None,
                          stream=None):
    """lserve_decode without a workspace, for callers that may not allocate device memory.

    The library takes its scratch from a fixed per-device array of
    NOALLOC_SCRATCH_BYTES.  ``out`` (and any of lse / sel_out / sel_n) must be
    provided by the caller; this wrapper allocates nothing.  Calls that overlap
    on the GPU share that array and race; keep them on one stream.
    """
    lib = load_library()
    a = _decode_args(q, k_pages, v_pages, page_table, seq_lens, stats, head_kind, sink, local, token_budget, scale)
    B, Hq, d = q.shape
    _dev(out, "out", torch.bfloat16, q.shape)
    if lse is not None:
        _dev(lse, "lse", torch.float32, (B, Hq))
    kcap = int(lib.lserve_decode_max_selected(ctypes.byref(a)))
    if sel_out is not None:
        _dev(sel_out, "sel_out", torch.int32, (B, a.Hkv, kcap))
    if sel_n is not None:
        _dev(sel_n, "sel_n", torch.int32, (B, a.Hkv))
    _check(lib.lserve_decode_noalloc(ctypes.byref(a), _ptr(out), _ptr(lse), _ptr(sel_out), _ptr(sel_n),
                                     _stream(stream)))
    return out


def lserve_get_device_status(stream=None) -> int:
    """Synchronise, read and clear the device status word (0 = OK)."""
    return int(load_library().lserve_get_device_status(_stream(stream)))
