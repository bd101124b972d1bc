"""fp64 CPU oracle for the HySparse / HySparse2 hot path (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The product package
never imports this module, and this module never imports the product package:
the two share no code.  The arithmetic lives in ``hs_oracle.c`` (plain C,
double precision, one query row at a time); this file only marshals numpy
arrays and compiles the C file with gcc on first use.

Function map (titles of the pages the method is described on):
  full_attn_index  -- "HySparse 混合稀疏注意力（一）" sections on block-level
                      scores, GQA group max and TopKBlocks; "HySparse: A Hybrid
                      Sparse Attention Architecture ..." 3.2 / Algorithm 1;
                      "HySparse2 ..." 4.2 (token-level top-k, forced window).
  sparse_attn      -- "HySparse 混合稀疏注意力（一）" sections on cross-layer KV
                      reuse and the two memories of one query; "HySparse ..." 3.3.
  gather_pages     -- "HySparse 混合稀疏注意力（一）", 工程实现中的关键约束 item 2
                      (logical ids, block table to physical pages).
  gate_sink        -- "HySparse 混合稀疏注意力（一）" section on the two sigmoid
                      gates; "HySparse ..." 3.3 (branch fusion) and its
                      configuration note on per-head sink biases.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hs_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile hs_oracle.c into liboracle.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Params(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("hq", ctypes.c_int), ("hkv", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("t_q", ctypes.c_int), ("t_kv", ctypes.c_int),
                ("q_offset", ctypes.c_int), ("mode", ctypes.c_int),
                ("block_size", ctypes.c_int), ("k", ctypes.c_int), ("window", ctypes.c_int),
                ("scale", ctypes.c_double)]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _bind(lib):
    P = ctypes.c_void_p
    lib.orc_full_attn_index.argtypes = [ctypes.POINTER(_Params), P, P, P, P, P, ctypes.c_int,
                                        P, P, P, P, P, P, P, ctypes.c_int]
    lib.orc_full_attn_index.restype = ctypes.c_int
    lib.orc_sparse_attn.argtypes = [ctypes.POINTER(_Params), P, P, P, P, P, ctypes.c_int, P,
                                    P, P, P, P, P, P, P, P]
    lib.orc_sparse_attn.restype = ctypes.c_int
    lib.orc_num_threads.restype = ctypes.c_int
    lib.orc_gate_sink.argtypes = [ctypes.c_int, ctypes.c_int] + [P] * 11
    lib.orc_gate_sink.restype = ctypes.c_int
    return lib


@contextlib.contextmanager
def use_library(path: str):
    """Temporarily route every oracle call to another build of hs_oracle.c.

    Used only by the mutation tests, which compile deliberately broken copies
    of the oracle and check that the pins reject them.
    """
    global _lib
    with _lock:
        old = _lib
        _lib = _bind(ctypes.CDLL(path))
    try:
        yield
    finally:
        with _lock:
            _lib = old


@dataclass
class Params:
    """Shapes and the method's knobs.  mode: "block" (HySparse) or "token" (HySparse2)."""
    batch: int
    hq: int
    hkv: int
    head_dim: int
    t_q: int
    t_kv: int
    mode: str = "block"
    block_size: int = 64
    k: int = 1024
    window: int = 128
    q_offset: int = 0
    scale: float = 0.0  # 0 -> 1/sqrt(head_dim)

    @property
    def group(self) -> int:
        return self.hq // self.hkv

    @property
    def ksel(self) -> int:
        return self.k // self.block_size if self.mode == "block" else self.k

    def _c(self) -> _Params:
        s = self.scale if self.scale > 0 else 1.0 / np.sqrt(self.head_dim)
        return _Params(self.batch, self.hq, self.hkv, self.head_dim, self.t_q, self.t_kv,
                       self.q_offset, 0 if self.mode == "block" else 1, self.block_size,
                       self.k, self.window, float(s))


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _rows_array(p: Params, rows, decode: bool) -> np.ndarray:
    if rows is None:
        tq = 1 if decode else p.t_q
        b, u, j = np.meshgrid(np.arange(p.batch), np.arange(p.hkv), np.arange(tq), indexing="ij")
        rows = np.stack([b.ravel(), u.ravel(), j.ravel()], axis=1)
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 3))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_load().orc_num_threads())


def _pos(q_pos, n):
    if q_pos is None:
        return None
    a = np.ascontiguousarray(np.asarray(q_pos, dtype=np.int32).reshape(-1))
    assert len(a) == n
    return a


def full_attn_index(p: Params, q, k, v, rows=None, kv_len=None, want_scores: bool = False,
                    q_pos=None):
    """Full attention + oracle index for the listed rows (default: all rows).

    rows: int array [n, 3] of (batch, kv group, query row).  kv_len: per-batch
    cache length for decode (the query is then the newest token).  q_pos:
    optional explicit position of each listed row.
    Returns dict with o [n, g, d], lse [n, g], idx [n, ksel], cnt [n],
    sel_score [n, ksel] and, if asked, scores [n, n_cand] (-1 beyond the row's
    candidates).
    """
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    assert q.shape == (p.batch, p.hq, p.t_q, p.head_dim), q.shape
    assert k.shape == v.shape == (p.batch, p.hkv, p.t_kv, p.head_dim), k.shape
    rws = _rows_array(p, rows, kv_len is not None)
    kvl = None if kv_len is None else np.ascontiguousarray(np.asarray(kv_len, dtype=np.int32))
    n, g, d, ks = len(rws), p.group, p.head_dim, p.ksel
    o = np.zeros((n, g, d)); lse = np.zeros((n, g))
    idx = np.zeros((n, ks), dtype=np.int32); cnt = np.zeros(n, dtype=np.int32)
    sel = np.zeros((n, ks))
    stride = 0
    scores = None
    if want_scores:
        stride = (-(-p.t_kv // p.block_size)) if p.mode == "block" else p.t_kv
        scores = np.zeros((n, stride))
    c = p._c()
    qp = _pos(q_pos, n)
    rc = lib.orc_full_attn_index(ctypes.byref(c), _ptr(q), _ptr(k), _ptr(v), _ptr(kvl), _ptr(qp), n,
                                 _ptr(rws), _ptr(o), _ptr(lse), _ptr(idx), _ptr(cnt), _ptr(sel),
                                 _ptr(scores), stride)
    if rc != 0:
        raise ValueError("oracle: invalid arguments")
    out = dict(rows=rws, o=o, lse=lse, idx=idx, cnt=cnt, sel_score=sel)
    if want_scores:
        out["scores"] = scores
    return out


def sparse_attn(p: Params, q, kf, vf, idx_rows, cnt_rows, rows=None, kv_len=None,
                k_loc=None, v_loc=None, q_pos=None):
    """Sparse layer over the listed rows, reusing K^F/V^F and the given index sets.

    idx_rows [n, ksel] / cnt_rows [n] are the index sets of the listed rows.
    Returns dict with o_g [n, g, d], lse_g [n, g] and, when k_loc is given,
    o_l / lse_l of the local (own K'/V') window branch.
    """
    lib = _load()
    q, kf, vf = _f64(q), _f64(kf), _f64(vf)
    rws = _rows_array(p, rows, kv_len is not None)
    n, g, d, ks = len(rws), p.group, p.head_dim, p.ksel
    idx_rows = np.ascontiguousarray(np.asarray(idx_rows, dtype=np.int32).reshape(n, ks))
    cnt_rows = np.ascontiguousarray(np.asarray(cnt_rows, dtype=np.int32).reshape(n))
    for r in range(n):  # the oracle sums over the list as given: it must be a set
        ids = idx_rows[r, :cnt_rows[r]]
        assert len(np.unique(ids)) == len(ids), "index set has duplicates"
    kvl = None if kv_len is None else np.ascontiguousarray(np.asarray(kv_len, dtype=np.int32))
    kl = None if k_loc is None else _f64(k_loc)
    vl = None if v_loc is None else _f64(v_loc)
    o_g = np.zeros((n, g, d)); lse_g = np.zeros((n, g))
    o_l = np.zeros((n, g, d)); lse_l = np.zeros((n, g))
    c = p._c()
    qp = _pos(q_pos, n)
    rc = lib.orc_sparse_attn(ctypes.byref(c), _ptr(q), _ptr(kf), _ptr(vf), _ptr(kvl), _ptr(qp), n,
                             _ptr(rws), _ptr(idx_rows), _ptr(cnt_rows), _ptr(kl), _ptr(vl),
                             _ptr(o_g), _ptr(lse_g), _ptr(o_l), _ptr(lse_l))
    if rc != 0:
        raise ValueError("oracle: invalid arguments")
    out = dict(rows=rws, o_g=o_g, lse_g=lse_g)
    if k_loc is not None:
        out.update(o_l=o_l, lse_l=lse_l)
    return out


# ------------------------------------------------------------ sampled rows
def _units(rows):
    order = {}
    for n, (b, u, _) in enumerate(rows):
        order.setdefault((int(b), int(u)), []).append(n)
    return order


def _f64_any(t):
    """float64 numpy copy of a numpy array or a (CPU or CUDA) torch tensor."""
    if hasattr(t, "detach"):
        import torch
        return t.detach().to("cpu", torch.float64).numpy()
    return _f64(t)


def _take_rows(q, b, h0, h1, js):
    if hasattr(q, "index_select"):
        import torch
        return q[b, h0:h1].index_select(1, torch.as_tensor(js, device=q.device))[None]
    return q[b, h0:h1][:, js][None]


def full_attn_rows(q, k, v, rows, pos, mode, block_size, k_budget, window):
    """full_attn_index on the listed rows (b, u, j) at positions pos only.

    q [b, hq, tq, d], k/v [b, hkv, T, d] (numpy or torch, any device).  Per
    (batch, group) only the rows' query vectors and the group's K/V prefix
    0..max(pos) are converted to float64, so rows of very long contexts can be
    evaluated without a float64 copy of the whole cache.  Returns o, lse, idx,
    cnt and the per-row candidate scores (list of arrays) in row order.
    """
    rows = np.asarray(rows, dtype=np.int32).reshape(-1, 3)
    pos = np.asarray(pos, dtype=np.int64).reshape(-1)
    hq, d = q.shape[1], q.shape[3]
    hkv = k.shape[1]
    g = hq // hkv
    ksel = k_budget // block_size if mode == "block" else k_budget
    n = len(rows)
    out = dict(rows=rows, o=np.zeros((n, g, d)), lse=np.zeros((n, g)),
               idx=np.zeros((n, ksel), np.int32), cnt=np.zeros(n, np.int32),
               scores=[None] * n, _t=pos)
    for (b, u), ns in _units(rows).items():
        ns = np.array(ns)
        ts = pos[ns]
        tmax = int(ts.max())
        qs = _take_rows(q, b, u * g, (u + 1) * g, rows[ns, 2].astype(np.int64))
        p = Params(1, g, 1, d, len(ns), tmax + 1, mode=mode, block_size=block_size,
                   k=k_budget, window=window)
        r = full_attn_index(p, _f64_any(qs), _f64_any(k[b, u, :tmax + 1][None, None]),
                            _f64_any(v[b, u, :tmax + 1][None, None]),
                            rows=[(0, 0, x) for x in range(len(ns))], q_pos=ts, want_scores=True)
        out["o"][ns] = r["o"]
        out["lse"][ns] = r["lse"]
        out["idx"][ns] = r["idx"]
        out["cnt"][ns] = r["cnt"]
        for x, nn in enumerate(ns):
            out["scores"][nn] = r["scores"][x]
    return out


def sparse_attn_rows(q, kf, vf, idx_rows, cnt_rows, rows, pos, mode, block_size, k_budget,
                     window, k_loc=None, v_loc=None):
    """sparse_attn on the listed rows only (same conventions as full_attn_rows)."""
    rows = np.asarray(rows, dtype=np.int32).reshape(-1, 3)
    pos = np.asarray(pos, dtype=np.int64).reshape(-1)
    idx_rows = np.asarray(idx_rows)
    cnt_rows = np.asarray(cnt_rows)
    hq, d = q.shape[1], q.shape[3]
    g = hq // kf.shape[1]
    n = len(rows)
    out = dict(o_g=np.zeros((n, g, d)), lse_g=np.zeros((n, g)), o_l=np.zeros((n, g, d)),
               lse_l=np.zeros((n, g)))
    for (b, u), ns in _units(rows).items():
        ns = np.array(ns)
        ts = pos[ns]
        tmax = int(ts.max())
        q1 = _take_rows(q, b, u * g, (u + 1) * g, rows[ns, 2].astype(np.int64))
        p = Params(1, g, 1, d, len(ns), tmax + 1, mode=mode, block_size=block_size,
                   k=k_budget, window=window)
        sl = lambda t: None if t is None else _f64_any(t[b, u, :tmax + 1][None, None])  # noqa
        r = sparse_attn(p, _f64_any(q1), sl(kf), sl(vf), idx_rows[ns], cnt_rows[ns],
                        rows=[(0, 0, x) for x in range(len(ns))], q_pos=ts, k_loc=sl(k_loc),
                        v_loc=sl(v_loc))
        out["o_g"][ns] = r["o_g"]
        out["lse_g"][ns] = r["lse_g"]
        if k_loc is not None:
            out["o_l"][ns] = r["o_l"]
            out["lse_l"][ns] = r["lse_l"]
    return out


def gather_pages(pool, block_table, page_size):
    """The logical K^F (or V^F) of a paged cache, [b, hkv, max_pages * page_size, d].

    pool [n_pages, hkv, page_size, d] (numpy or torch), block_table [b, max_pages]:
    logical key i of sequence b is row i % page_size of page
    block_table[b, i // page_size] ("HySparse 混合稀疏注意力（一）", 工程实现中的关键约束
    item 2: the index keeps logical token ids, the block table maps them to
    physical pages).  The oracle then runs on this contiguous view.
    """
    pool = _f64_any(pool)
    bt = np.asarray(block_table.cpu() if hasattr(block_table, "cpu") else block_table,
                    dtype=np.int64)
    b, mp = bt.shape
    n_pages, hkv, ps, d = pool.shape
    assert ps == page_size
    out = np.zeros((b, hkv, mp * ps, d))
    for bb in range(b):
        for lp in range(mp):
            out[bb, :, lp * ps:(lp + 1) * ps] = pool[bt[bb, lp]]
    return out


def gate_sink(o_g, lse_g, o_l=None, lse_l=None, sink_g=None, sink_l=None, z_g=None, z_l=None):
    """Sparse-layer output with per-head sinks and sigmoid gates (orc_gate_sink).

    o_* [b, hq, t, d], lse_* and z_* [b, hq, t], sink_* [hq].  Returns
    (o, lse_g', lse_l') with lse_l' None for one branch."""
    o_g = _f64(o_g)
    b, hq, t, d = o_g.shape
    n = b * hq * t
    lse_g = _f64(lse_g).reshape(n)

    def per_entry(s):
        if s is None:
            return None
        return _f64(np.broadcast_to(np.asarray(s, np.float64).reshape(1, hq, 1), (b, hq, t))).reshape(n)

    def opt(a, shape):
        return None if a is None else _f64(a).reshape(shape)

    o_l_, lse_l_ = opt(o_l, (n, d)), opt(lse_l, n)
    s_g_, s_l_ = per_entry(sink_g), per_entry(sink_l)
    z_g_, z_l_ = opt(z_g, n), opt(z_l, n)
    o = np.zeros((n, d))
    lg = np.zeros(n)
    ll = np.zeros(n) if o_l is not None else None
    rc = _load().orc_gate_sink(n, d, _ptr(o_g), _ptr(lse_g), _ptr(s_g_), _ptr(z_g_), _ptr(o_l_),
                               _ptr(lse_l_), _ptr(s_l_), _ptr(z_l_), _ptr(o), _ptr(lg), _ptr(ll))
    if rc != 0:
        raise ValueError(f"orc_gate_sink failed ({rc})")
    return (o.reshape(b, hq, t, d), lg.reshape(b, hq, t),
            None if ll is None else ll.reshape(b, hq, t))
