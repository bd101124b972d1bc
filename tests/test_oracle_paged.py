"""Pins of the oracle's paged-cache view (gather_pages).

A paged K^F/V^F keeps logical token ids in the index sets and a block table
that maps each sequence's logical pages to physical pages of a pool
("HySparse 混合稀疏注意力（一）", 工程实现中的关键约束 item 2).  The oracle reads a
paged cache by gathering its logical view and running unchanged on it.  The
pins: the gathered view of a pool scattered from a contiguous cache (by the
input generator, with a shuffled table and noise in the unused pages) is that
cache again, bit for bit, for page sizes that do and do not divide the
length; therefore the oracle's paged result equals its contiguous result;
and planted mistakes in the gather are rejected.
"""
import importlib.util
import os
import shutil
import sys

import numpy as np
import pytest
import torch

import oracle
from oracle_top_kv_b200 import workloads as wl


def _kv(b, hkv, T, d, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(b, hkv, T, d, generator=g, dtype=torch.float64),
            torch.randn(b, hkv, T, d, generator=g, dtype=torch.float64))


@pytest.mark.parametrize("page_size", [1, 5, 16, 48])
def test_gathered_view_is_the_contiguous_cache(page_size):
    k, v = _kv(3, 2, 97, 8, seed=page_size)
    kp, vp, bt = wl.paged_pool(k, v, page_size, seed=page_size)
    assert bt.shape == (3, -(-97 // page_size))
    assert len(set(bt.flatten().tolist())) == bt.numel()  # pages are distinct
    for pool, ref in ((kp, k), (vp, v)):
        got = oracle.gather_pages(pool, bt, page_size)
        assert got.shape[2] == bt.shape[1] * page_size
        assert np.array_equal(got[:, :, :97], ref.numpy())


def test_paged_oracle_result_equals_contiguous_result():
    b, hq, hkv, T, d, ps = 2, 8, 2, 90, 16, 7
    g = torch.Generator().manual_seed(3)
    q = torch.randn(b, hq, T, d, generator=g, dtype=torch.float64)
    qs = torch.randn(b, hq, T, d, generator=g, dtype=torch.float64)
    k, v = _kv(b, hkv, T, d, seed=11)
    kp, vp, bt = wl.paged_pool(k, v, ps, seed=1)
    kg, vg = oracle.gather_pages(kp, bt, ps), oracle.gather_pages(vp, bt, ps)
    Tc = kg.shape[2]
    for mode, B, kk, w in (("token", 1, 12, 4), ("block", 4, 16, 0)):
        p = oracle.Params(b, hq, hkv, d, T, T, mode=mode, block_size=B, k=kk, window=w)
        full = oracle.full_attn_index(p, q, k, v)
        pc = oracle.Params(b, hq, hkv, d, T, Tc, mode=mode, block_size=B, k=kk, window=w)
        a = oracle.sparse_attn(p, qs, k, v, full["idx"], full["cnt"])
        c = oracle.sparse_attn(pc, qs, kg, vg, full["idx"], full["cnt"])
        assert np.array_equal(a["o_g"], c["o_g"]) and np.array_equal(a["lse_g"], c["lse_g"])
        # decode rows: the newest token of ragged sequences
        kv_len = np.array([T, 41], np.int32)
        pd = oracle.Params(b, hq, hkv, d, 1, T, mode=mode, block_size=B, k=kk, window=w)
        pdc = oracle.Params(b, hq, hkv, d, 1, Tc, mode=mode, block_size=B, k=kk, window=w)
        fd = oracle.full_attn_index(pd, q[:, :, :1], k, v, kv_len=kv_len)
        fdc = oracle.full_attn_index(pdc, q[:, :, :1], kg, vg, kv_len=kv_len)
        assert np.array_equal(fd["idx"], fdc["idx"]) and np.array_equal(fd["o"], fdc["o"])


MUTANTS = {
    "row_in_page_shifted": ("out[bb, :, lp * ps:(lp + 1) * ps] = pool[bt[bb, lp]]",
                            "out[bb, :, lp * ps:(lp + 1) * ps] = np.roll(pool[bt[bb, lp]], 1, axis=1)"),
    "table_ignored": ("out[bb, :, lp * ps:(lp + 1) * ps] = pool[bt[bb, lp]]",
                      "out[bb, :, lp * ps:(lp + 1) * ps] = pool[bb * mp + lp]"),
    "wrong_sequence_row": ("out[bb, :, lp * ps:(lp + 1) * ps] = pool[bt[bb, lp]]",
                           "out[bb, :, lp * ps:(lp + 1) * ps] = pool[bt[(bb + 1) % b, lp]]"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_paged_pins_reject_mutant(name, tmp_path, monkeypatch):
    before, after = MUTANTS[name]
    here = os.path.dirname(oracle.__file__)
    src = open(os.path.join(here, "__init__.py")).read()
    assert src.count(before) == 1
    pkg = tmp_path / "oracle_mut"
    pkg.mkdir()
    (pkg / "__init__.py").write_text(src.replace(before, after))
    shutil.copy(os.path.join(here, "hs_oracle.c"), pkg / "hs_oracle.c")
    spec = importlib.util.spec_from_file_location("oracle_mut", pkg / "__init__.py")
    mod = importlib.util.module_from_spec(spec)
    monkeypatch.setitem(sys.modules, "oracle_mut", mod)
    spec.loader.exec_module(mod)
    monkeypatch.setattr(oracle, "gather_pages", mod.gather_pages)
    with pytest.raises(AssertionError):
        for ps in (1, 5, 16, 48):
            test_gathered_view_is_the_contiguous_cache(ps)
