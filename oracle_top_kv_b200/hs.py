"""Thin Python binding of the C ABI in include/hs.h (argument marshalling only).

Every function has the name of the C entry point it calls and takes the same
arguments, with torch CUDA tensors in place of raw device pointers (a plain
int is accepted as a raw device address).  All the computation happens in
libhs_b200.so; this module only loads it, converts arguments and raises
HsError on a non-OK status.  If the library is missing, loading fails loudly:
there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhs_b200.so")

HS_OK, HS_ERR_INVALID_ARG, HS_ERR_UNSUPPORTED, HS_ERR_CUDA = 0, 1, 2, 3
HS_ERR_TIMEOUT, HS_ERR_BOUNDS, HS_ERR_WORKSPACE = 4, 5, 6
HS_BF16, HS_FP32 = 0, 1
HS_SEL_BLOCK, HS_SEL_TOKEN = 0, 1
HS_DECODE_FULL_INDEX, HS_DECODE_SPARSE = 0, 1
HS_WS_FULL, HS_WS_SPARSE, HS_WS_DECODE_FULL, HS_WS_DECODE_SPARSE = 0, 1, 2, 3

EXPORTS = ("hs_full_attn_index", "hs_sparse_attn_reuse", "hs_decode_step", "hs_workspace_size",
           "hs_device_status", "hs_status_string", "hs_launch_count", "hs_decode_sparse_noalloc",
           "hs_set_wait_limit", "hs_sparse_attn_reuse_paged", "hs_decode_step_paged",
           "hs_set_select_sampling")


class HsError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {hs_status_string(code)} ({code})")
        self.code = code


class hs_params(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("hq", ctypes.c_int32), ("hkv", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("t_q", ctypes.c_int32), ("t_kv", ctypes.c_int32),
                ("q_offset", ctypes.c_int32), ("dtype", ctypes.c_int32), ("mode", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("k", ctypes.c_int32), ("window", ctypes.c_int32),
                ("scale", ctypes.c_float)]

    @property
    def ksel(self) -> int:
        return self.k // self.block_size if self.mode == HS_SEL_BLOCK else self.k


class hs_pages(ctypes.Structure):
    _fields_ = [("block_table", ctypes.c_void_p), ("page_size", ctypes.c_int32),
                ("max_pages", ctypes.c_int32), ("n_pages", ctypes.c_int32)]


def make_pages(block_table, page_size, n_pages) -> hs_pages:
    """hs_pages for a [batch][max_pages] int32 device block table."""
    return hs_pages(_ptr(block_table), int(page_size), int(block_table.shape[-1]), int(n_pages))


def make_params(batch, hq, hkv, head_dim, t_q, t_kv, q_offset=0, dtype="bf16", mode="block",
                block_size=64, k=1024, window=128, scale=0.0) -> hs_params:
    return hs_params(batch, hq, hkv, head_dim, t_q, t_kv, q_offset,
                     HS_BF16 if dtype == "bf16" else HS_FP32,
                     HS_SEL_BLOCK if mode == "block" else HS_SEL_TOKEN, block_size, k, window,
                     float(scale))


_lib = None


def load(path: str = LIB_PATH):
    """Load libhs_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m oracle_top_kv_b200.build`"
                           " (there is no fallback implementation)")
    lib = ctypes.CDLL(path)
    P, S, I32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
    PP = ctypes.POINTER(hs_params)
    lib.hs_full_attn_index.argtypes = [PP, P, P, P, P, P, P, P, P, P, S, P]
    lib.hs_sparse_attn_reuse.argtypes = [PP, P, P, P, P, P, P, P, P, P, P, P, P, S, P]
    lib.hs_decode_step.argtypes = [PP, I32, P, P, P, P, P, P, P, P, P, P, S, P]
    lib.hs_decode_sparse_noalloc.argtypes = [PP, P, P, P, P, P, P, P, P, P]
    lib.hs_sparse_gate_sink.argtypes = [PP, P, P, P, P, P, P, P, P, P, P]
    lib.hs_workspace_size.argtypes = [PP, I32]
    lib.hs_workspace_size.restype = S
    lib.hs_device_status.argtypes = [P, ctypes.POINTER(I32)]
    lib.hs_set_wait_limit.argtypes = [ctypes.c_int64]
    lib.hs_set_select_sampling.argtypes = [I32]
    PG = ctypes.POINTER(hs_pages)
    lib.hs_sparse_attn_reuse_paged.argtypes = [PP, PG, P, P, P, P, P, P, P, P]
    lib.hs_decode_step_paged.argtypes = [PP, PG, I32, P, P, P, P, P, P, P, P, P, P, S, P]
    lib.hs_status_string.argtypes = [I32]
    lib.hs_status_string.restype = ctypes.c_char_p
    lib.hs_launch_count.argtypes = []
    lib.hs_launch_count.restype = ctypes.c_uint64
    for name in ("hs_full_attn_index", "hs_sparse_attn_reuse", "hs_decode_step",
                 "hs_device_status", "hs_decode_sparse_noalloc", "hs_sparse_gate_sink"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ws(ws):
    if ws is None:
        return None, 0
    if isinstance(ws, tuple):
        return ws
    return ws.data_ptr(), ws.numel() * ws.element_size()


def _check(code, where):
    if code != HS_OK:
        raise HsError(code, where)


def hs_full_attn_index(p, q, k, v, o, lse, idx, idx_count, sel_scores=None, workspace=None,
                       stream=None):
    lib = load()
    wp, wb = _ws(workspace)
    _check(lib.hs_full_attn_index(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                  _ptr(idx), _ptr(idx_count), _ptr(sel_scores), wp, wb,
                                  _stream(stream)), "hs_full_attn_index")


def hs_sparse_attn_reuse(p, q_sparse, k_f, v_f, idx, idx_count, k_local, v_local, o_global,
                         lse_global, o_local=None, lse_local=None, workspace=None, stream=None):
    lib = load()
    wp, wb = _ws(workspace)
    _check(lib.hs_sparse_attn_reuse(ctypes.byref(p), _ptr(q_sparse), _ptr(k_f), _ptr(v_f),
                                    _ptr(idx), _ptr(idx_count), _ptr(k_local), _ptr(v_local),
                                    _ptr(o_global), _ptr(lse_global), _ptr(o_local),
                                    _ptr(lse_local), wp, wb, _stream(stream)),
           "hs_sparse_attn_reuse")


def hs_sparse_gate_sink(p, o_global, lse_global, o, o_local=None, lse_local=None,
                        sink_global=None, sink_local=None, gate_global=None, gate_local=None,
                        stream=None):
    """Per-head sinks and sigmoid-gate fusion of a sparse layer's branches
    (include/hs.h); updates lse_global / lse_local in place."""
    lib = load()
    _check(lib.hs_sparse_gate_sink(ctypes.byref(p), _ptr(o_global), _ptr(lse_global),
                                   _ptr(o_local), _ptr(lse_local), _ptr(sink_global),
                                   _ptr(sink_local), _ptr(gate_global), _ptr(gate_local), _ptr(o),
                                   _stream(stream)),
           "hs_sparse_gate_sink")


def hs_decode_step(p, kind, q, k_cache, v_cache, seq_len, idx, idx_count, o, lse=None,
                   sel_scores=None, workspace=None, stream=None):
    lib = load()
    wp, wb = _ws(workspace)
    _check(lib.hs_decode_step(ctypes.byref(p), int(kind), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                              _ptr(seq_len), _ptr(idx), _ptr(idx_count), _ptr(o), _ptr(lse),
                              _ptr(sel_scores), wp, wb, _stream(stream)), "hs_decode_step")


def hs_sparse_attn_reuse_paged(p, pages, q_sparse, k_pool, v_pool, idx, idx_count, o_global,
                               lse_global, stream=None):
    _check(load().hs_sparse_attn_reuse_paged(ctypes.byref(p), ctypes.byref(pages),
                                             _ptr(q_sparse), _ptr(k_pool), _ptr(v_pool),
                                             _ptr(idx), _ptr(idx_count), _ptr(o_global),
                                             _ptr(lse_global), _stream(stream)),
           "hs_sparse_attn_reuse_paged")


def hs_decode_step_paged(p, pages, kind, q, k_pool, v_pool, seq_len, idx, idx_count, o,
                         lse=None, sel_scores=None, workspace=None, stream=None):
    wp, wb = _ws(workspace)
    _check(load().hs_decode_step_paged(ctypes.byref(p), ctypes.byref(pages), int(kind), _ptr(q),
                                       _ptr(k_pool), _ptr(v_pool), _ptr(seq_len), _ptr(idx),
                                       _ptr(idx_count), _ptr(o), _ptr(lse), _ptr(sel_scores), wp,
                                       wb, _stream(stream)), "hs_decode_step_paged")


def hs_decode_sparse_noalloc(p, q, k_cache, v_cache, seq_len, idx, idx_count, o, lse=None,
                             stream=None):
    """hs_decode_step(HS_DECODE_SPARSE) without a workspace (library-owned scratch)."""
    _check(load().hs_decode_sparse_noalloc(ctypes.byref(p), _ptr(q), _ptr(k_cache),
                                           _ptr(v_cache), _ptr(seq_len), _ptr(idx),
                                           _ptr(idx_count), _ptr(o), _ptr(lse), _stream(stream)),
           "hs_decode_sparse_noalloc")


def hs_workspace_size(p, which) -> int:
    n = load().hs_workspace_size(ctypes.byref(p), int(which))
    if n == ctypes.c_size_t(-1).value:
        raise HsError(HS_ERR_INVALID_ARG, "hs_workspace_size")
    return int(n)


def hs_device_status(stream=None) -> int:
    out = ctypes.c_int32(0)
    _check(load().hs_device_status(_stream(stream), ctypes.byref(out)), "hs_device_status")
    return int(out.value)


def hs_set_wait_limit(cycles: int) -> None:
    """Bound, in SM cycles, of the kernels' waits (<= 0: the default)."""
    _check(load().hs_set_wait_limit(int(cycles)), "hs_set_wait_limit")


def hs_set_select_sampling(rank: int) -> None:
    """Sampled start threshold of the token selector: -1 automatic, 0 off, r > 0 that rank."""
    _check(load().hs_set_select_sampling(int(rank)), "hs_set_select_sampling")


def hs_status_string(code) -> str:
    return load().hs_status_string(int(code)).decode()


def hs_launch_count() -> int:
    return int(load().hs_launch_count())


# ------------------------------------------------------------ output helpers
def _tdtype(p):
    return torch.bfloat16 if p.dtype == HS_BF16 else torch.float32


def full_outputs(p, device="cuda", with_scores=False):
    """Allocate o, lse, idx, idx_count (and sel_scores) for hs_full_attn_index."""
    o = torch.empty(p.batch, p.hq, p.t_q, p.head_dim, dtype=_tdtype(p), device=device)
    lse = torch.empty(p.batch, p.hq, p.t_q, dtype=torch.float32, device=device)
    idx = torch.empty(p.batch, p.hkv, p.t_q, p.ksel, dtype=torch.int32, device=device)
    cnt = torch.empty(p.batch, p.hkv, p.t_q, dtype=torch.int32, device=device)
    sel = (torch.empty(p.batch, p.hkv, p.t_q, p.ksel, dtype=torch.float32, device=device)
           if with_scores else None)
    return o, lse, idx, cnt, sel


def workspace(p, which, device="cuda"):
    n = hs_workspace_size(p, which)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device) if n else None
