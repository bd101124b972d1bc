"""The C-ABI library builds, loads and exports every symbol include/hs.h
declares, and its host-side argument checks return the documented codes.

No test here launches a kernel: every call below fails validation on the host
(or only sizes a workspace), so these run without a GPU.
"""
import ctypes
import os
import re

import pytest

from oracle_top_kv_b200 import build as hsbuild
from oracle_top_kv_b200 import hs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    hsbuild.build()
    return hs.load()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "hs.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hs_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert set(hs.EXPORTS) <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    assert hs.hs_status_string(0) == "HS_OK"
    assert hs.hs_status_string(5) == "HS_ERR_BOUNDS"
    assert hs.hs_status_string(99) == "HS_UNKNOWN_STATUS"


def _p(**kw):
    base = dict(batch=2, hq=32, hkv=8, head_dim=128, t_q=256, t_kv=256, dtype="bf16",
                mode="block", block_size=64, k=1024, window=128)
    base.update(kw)
    return hs.make_params(**base)


FAKE = 1 << 20  # 16-byte aligned, never dereferenced: validation fails first


def _full(p, **ptrs):
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, idx=FAKE, idx_count=FAKE)
    args.update(ptrs)
    return hs.load().hs_full_attn_index(ctypes.byref(p), args["q"], args["k"], args["v"],
                                        args["o"], args["lse"], args["idx"], args["idx_count"],
                                        None, None, 0, None)


@pytest.mark.parametrize("bad,code", [
    (dict(hq=30), hs.HS_ERR_INVALID_ARG),            # hq % hkv != 0
    (dict(block_size=48), hs.HS_ERR_INVALID_ARG),     # k % B != 0
    (dict(block_size=8, k=1024), hs.HS_ERR_UNSUPPORTED),  # B not in {16..128}
    (dict(k=8192), hs.HS_ERR_UNSUPPORTED),            # k/B > 64
    (dict(head_dim=96), hs.HS_ERR_UNSUPPORTED),
    (dict(hq=128, hkv=1), hs.HS_ERR_UNSUPPORTED),     # group of 128 heads
    (dict(head_dim=512), hs.HS_ERR_UNSUPPORTED),
    (dict(q_offset=1), hs.HS_ERR_INVALID_ARG),        # rows beyond t_kv
    (dict(mode="token", window=2000, k=1024), hs.HS_ERR_INVALID_ARG),  # w > k
    (dict(mode="token", k=8192, window=128), hs.HS_ERR_UNSUPPORTED),
    (dict(batch=0), hs.HS_ERR_INVALID_ARG),
    (dict(dtype="bf16", scale=-1.0), hs.HS_ERR_INVALID_ARG),
])
def test_full_rejects_bad_params(lib, bad, code):
    assert _full(_p(**bad)) == code


def test_full_rejects_null_and_misaligned_pointers(lib):
    assert _full(_p(), q=0) == hs.HS_ERR_INVALID_ARG
    assert _full(_p(), lse=FAKE + 4) == hs.HS_ERR_INVALID_ARG
    assert hs.load().hs_full_attn_index(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None,
                                        None, 0, None) == hs.HS_ERR_INVALID_ARG


def test_sparse_rejects_local_branch_without_outputs(lib):
    p = _p()
    r = hs.load().hs_sparse_attn_reuse(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                       FAKE, FAKE, None, None, None, 0, None)
    assert r == hs.HS_ERR_INVALID_ARG


def test_decode_checks(lib):
    p = _p(t_q=1, t_kv=4096, mode="token", block_size=1, hq=64, hkv=4)
    L = hs.load()
    need = hs.hs_workspace_size(p, hs.HS_WS_DECODE_FULL)
    assert need >= 2 * 4 * 4096 * 16 * 4  # exported logits of every cached key
    # too small a workspace
    assert L.hs_decode_step(ctypes.byref(p), 0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                            None, FAKE, need - 1, None) == hs.HS_ERR_WORKSPACE
    # decode needs t_q == 1
    p2 = _p(t_q=2, t_kv=4096, mode="token", block_size=1)
    assert L.hs_decode_step(ctypes.byref(p2), 0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                            None, FAKE, need, None) == hs.HS_ERR_INVALID_ARG
    # fp32 and block mode are not implemented for decode
    p3 = _p(t_q=1, t_kv=4096, mode="token", block_size=1, dtype="fp32")
    assert L.hs_decode_step(ctypes.byref(p3), 1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                            None, FAKE, 1 << 30, None) == hs.HS_ERR_UNSUPPORTED
    assert L.hs_decode_step(ctypes.byref(p), 7, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                            None, FAKE, need, None) == hs.HS_ERR_INVALID_ARG


def test_workspace_sizes(lib):
    assert hs.hs_workspace_size(_p(), hs.HS_WS_FULL) == 0
    assert hs.hs_workspace_size(_p(), hs.HS_WS_SPARSE) == 0
    p = _p(t_q=1, t_kv=1024, mode="token", block_size=1)
    assert hs.hs_workspace_size(p, hs.HS_WS_DECODE_SPARSE) == 0  # merged on chip
    assert hs.hs_workspace_size(p, hs.HS_WS_DECODE_FULL) > 0
    with pytest.raises(hs.HsError):
        hs.hs_workspace_size(_p(hq=30), hs.HS_WS_FULL)


def _gate_sink(p, o_g=FAKE, lse_g=FAKE, o_l=None, lse_l=None, s_g=None, s_l=None, z_g=None,
               z_l=None, o=FAKE):
    return hs.load().hs_sparse_gate_sink(ctypes.byref(p), o_g, lse_g, o_l, lse_l, s_g, s_l, z_g,
                                         z_l, o, None)


def test_gate_sink_argument_checks(lib):
    p = _p()
    bad = hs.HS_ERR_INVALID_ARG
    assert _gate_sink(p, o_l=FAKE) == bad                  # local output without its lse
    assert _gate_sink(p, lse_l=FAKE) == bad                # local lse without its output
    assert _gate_sink(p, s_l=FAKE) == bad                  # local sink without a local branch
    assert _gate_sink(p, z_l=FAKE) == bad                  # local gate without a local branch
    assert _gate_sink(p, o=None) == bad                    # no output
    assert _gate_sink(p, o_g=FAKE + 8) == bad              # misaligned
    assert _gate_sink(p, z_g=FAKE + 4) == bad
    assert _gate_sink(_p(head_dim=96)) == hs.HS_ERR_UNSUPPORTED
    assert _gate_sink(_p(t_q=0, t_kv=4)) == hs.HS_OK       # nothing to do, nothing launched


def test_paged_entry_points_check_the_table(lib):
    p = _p(mode="token", block_size=1, t_kv=1024)
    ok = hs.hs_pages(FAKE, 16, 64, 10)
    for bad in (hs.hs_pages(None, 16, 64, 10), hs.hs_pages(FAKE, 0, 64, 10),
                hs.hs_pages(FAKE, 16, 63, 10), hs.hs_pages(FAKE, 16, 64, 0),
                hs.hs_pages(FAKE, 16, 64, 1 << 27)):
        assert lib.hs_sparse_attn_reuse_paged(ctypes.byref(p), ctypes.byref(bad), FAKE, FAKE,
                                              FAKE, FAKE, FAKE, FAKE, FAKE, None) == \
            hs.HS_ERR_INVALID_ARG
    assert lib.hs_sparse_attn_reuse_paged(ctypes.byref(p), None, FAKE, FAKE, FAKE, FAKE, FAKE,
                                          FAKE, FAKE, None) == hs.HS_ERR_INVALID_ARG
    pf = _p(mode="token", block_size=1, t_kv=1024, dtype="fp32")
    assert lib.hs_sparse_attn_reuse_paged(ctypes.byref(pf), ctypes.byref(ok), FAKE, FAKE, FAKE,
                                          FAKE, FAKE, FAKE, FAKE, None) == hs.HS_ERR_UNSUPPORTED
    pd = _p(mode="token", block_size=1, t_kv=1024, t_q=1)
    assert lib.hs_decode_step_paged(ctypes.byref(pd), ctypes.byref(ok), 0, FAKE, FAKE, FAKE,
                                    FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 0, None) == \
        hs.HS_ERR_WORKSPACE


def test_wide_groups_and_head_dim_256_decode_workspace(lib):
    # split-k CUDA-core decode: the full step holds every key's 64 head logits
    # (fp32) plus per-split partials; the sparse step per-split partials
    p = _p(hq=64, hkv=1, head_dim=256, t_q=1, t_kv=4096, mode="token", block_size=1)
    full = hs.hs_workspace_size(p, hs.HS_WS_DECODE_FULL)
    sparse = hs.hs_workspace_size(p, hs.HS_WS_DECODE_SPARSE)
    assert full >= 4096 * 64 * 4 and sparse > 0
    p = _p(hq=64, hkv=1, head_dim=256, t_q=1, t_kv=4096, mode="token", block_size=1)
    pages = hs.hs_pages(FAKE, 16, 256, 10)
    # paged and allocation-free entry points: groups of <= 16 heads, d <= 128
    assert lib.hs_decode_step_paged(ctypes.byref(p), ctypes.byref(pages), 1, FAKE, FAKE, FAKE,
                                    FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 0, None) == \
        hs.HS_ERR_UNSUPPORTED
    assert lib.hs_decode_sparse_noalloc(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                        FAKE, None, None) == hs.HS_ERR_UNSUPPORTED
