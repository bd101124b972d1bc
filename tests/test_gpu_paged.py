"""GPU parity of the paged K^F/V^F entry points.

The index sets keep logical token ids; the kernels translate each row they
load through the block table ("HySparse 混合稀疏注意力（一）", 工程实现中的关键约束
items 2 and 3).  The pools come from the contiguous caches by a seeded
shuffled block table with noise in the unused pages (workloads.paged_pool);
results are checked against the fp64 oracle on the logical view
(oracle.gather_pages) and against the contiguous entry points, with page
sizes that split the 32-row load chunks and blocks across pages.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle_top_kv_b200 import hs
from oracle_top_kv_b200 import workloads as wl
from tests import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"

PREFILL = {
    "token": wl.scaled(wl.WORKLOADS["hysparse2_prefill"], name="paged_token", hq=32, hkv=2,
                       t=700, k=256, window=64),
    "block": wl.scaled(wl.WORKLOADS["hysparse_7b_block"], name="paged_block", batch=2, hq=8,
                       hkv=2, t=640, k=256, window=64, swa_branch=False),
}


def _pages(bt, ps, n_pages):
    return hs.make_pages(bt, ps, n_pages)


@pytest.mark.parametrize("ps", [16, 48])
@pytest.mark.parametrize("mode", sorted(PREFILL))
def test_paged_sparse_prefill(mode, ps):
    w = PREFILL[mode]
    q, k, v, _ = wl.full_layer_inputs(w)
    q, k, v = q.to(DEV), k.to(DEV), v.to(DEV)
    p = P.abi_params(w)
    o, lse, idx, cnt, _ = hs.full_outputs(p)
    hs.hs_full_attn_index(p, q, k, v, o, lse, idx, cnt)
    kp, vp, bt = wl.paged_pool(k, v, ps, seed=ps)
    pages = _pages(bt, ps, kp.shape[0])
    pp = P.abi_params(w)
    pp.t_kv = bt.shape[1] * ps
    qs = wl.sparse_layer_query(w, 0).to(DEV)
    og, lg = torch.empty_like(qs), torch.empty(w.batch, w.hq, w.tq, dtype=torch.float32,
                                                device=DEV)
    hs.hs_sparse_attn_reuse_paged(pp, pages, qs, kp, vp, idx, cnt, og, lg)
    oc, lc = torch.empty_like(qs), torch.empty_like(lg)
    hs.hs_sparse_attn_reuse(p, qs, k, v, idx, cnt, None, None, oc, lc)
    torch.cuda.synchronize()
    assert hs.hs_device_status() == 0
    rows = P.all_rows(w)
    pos = w.q_offset + rows[:, 2]
    g_idx = P.gpu_rows(idx.cpu().numpy(), rows, False)
    g_cnt = P.gpu_rows(cnt.cpu().numpy(), rows, False)
    kg = oracle.gather_pages(kp, bt, ps)
    vg = oracle.gather_pages(vp, bt, ps)
    sp = P.oracle_sparse_rows(w, qs, kg, vg, g_idx, g_cnt, rows, pos)
    g = w.group
    P.check_o(P.gpu_rows(P.f64(og), rows, True, g), sp["o_g"], "bf16", f"paged {mode} o")
    P.check_lse(P.gpu_rows(lg.cpu().double().numpy(), rows, True, g), sp["lse_g"], "bf16",
                f"paged {mode} lse")
    P.check_o(P.f64(og), P.f64(oc), "bf16", f"paged {mode} vs contiguous")


def test_paged_decode_full_and_sparse():
    w = wl.scaled(wl.WORKLOADS["hysparse2_decode"], name="paged_decode", batch=4, hq=32, hkv=2,
                  t=3000, k=256, window=64)
    q, kc, vc, _ = wl.full_layer_inputs(w)
    q, kc, vc = q.to(DEV), kc.to(DEV), vc.to(DEV)
    seq = torch.tensor([3000, 1, 777, 2049], dtype=torch.int32)
    sl = seq.to(DEV)
    ps = 24  # not a divisor of the 32-row chunks: chunks straddle pages
    kp, vp, bt = wl.paged_pool(kc, vc, ps, seed=5)
    pages = _pages(bt, ps, kp.shape[0])
    p = P.abi_params(w, decode=True)
    pp = P.abi_params(w, decode=True)
    pp.t_kv = bt.shape[1] * ps
    ks = p.ksel
    out = {}
    for name, prm, args in (("contig", p, None), ("paged", pp, pages)):
        idx = torch.empty(w.batch, w.hkv, ks, dtype=torch.int32, device=DEV)
        cnt = torch.empty(w.batch, w.hkv, dtype=torch.int32, device=DEV)
        o = torch.empty_like(q)
        lse = torch.empty(w.batch, w.hq, 1, dtype=torch.float32, device=DEV)
        ws = hs.workspace(prm, hs.HS_WS_DECODE_FULL)
        qs = wl.sparse_layer_query(w, 0).to(DEV)
        os_ = torch.empty_like(qs)
        ls = torch.empty_like(lse)
        if args is None:
            hs.hs_decode_step(prm, hs.HS_DECODE_FULL_INDEX, q, kc, vc, sl, idx, cnt, o, lse, None, ws)
            hs.hs_decode_step(prm, hs.HS_DECODE_SPARSE, qs, kc, vc, sl, idx, cnt, os_, ls)
        else:
            hs.hs_decode_step_paged(prm, args, hs.HS_DECODE_FULL_INDEX, q, kp, vp, sl, idx, cnt,
                                    o, lse, None, ws)
            hs.hs_decode_step_paged(prm, args, hs.HS_DECODE_SPARSE, qs, kp, vp, sl, idx, cnt,
                                    os_, ls)
        torch.cuda.synchronize()
        assert hs.hs_device_status() == 0
        out[name] = (idx, cnt, o, lse, os_, ls, qs)
    # the paged step reads the same rows through the table: same index sets
    assert torch.equal(out["paged"][0], out["contig"][0])
    assert torch.equal(out["paged"][1], out["contig"][1])
    idx, cnt, o, lse, os_, ls, qs = out["paged"]
    rows = np.array([[b, u, 0] for b in range(w.batch) for u in range(w.hkv)], np.int32)
    pos = seq.numpy()[rows[:, 0]] - 1
    kg, vg = oracle.gather_pages(kp, bt, ps), oracle.gather_pages(vp, bt, ps)
    orc = P.oracle_full_rows(w, q, kg, vg, rows, pos)
    g = w.group
    P.check_o(P.gpu_rows(P.f64(o), rows, True, g), orc["o"], "bf16", "paged decode o")
    P.check_lse(P.gpu_rows(lse.cpu().double().numpy(), rows, True, g), orc["lse"], "bf16",
                "paged decode lse")
    g_idx = idx.cpu().numpy()[rows[:, 0], rows[:, 1]]
    g_cnt = cnt.cpu().numpy()[rows[:, 0], rows[:, 1]]
    P.check_index(g_idx, g_cnt, orc, "token", w.window, w.k, "paged decode index")
    sp = P.oracle_sparse_rows(w, qs, kg, vg, g_idx, g_cnt, rows, pos)
    P.check_o(P.gpu_rows(P.f64(os_), rows, True, g), sp["o_g"], "bf16", "paged decode sparse")
    P.check_lse(P.gpu_rows(ls.cpu().double().numpy(), rows, True, g), sp["lse_g"], "bf16",
                "paged decode sparse lse")


def test_paged_bad_page_sets_bounds_status():
    w = PREFILL["token"]
    q, k, v, _ = wl.full_layer_inputs(w)
    q, k, v = q.to(DEV), k.to(DEV), v.to(DEV)
    p = P.abi_params(w)
    o, lse, idx, cnt, _ = hs.full_outputs(p)
    hs.hs_full_attn_index(p, q, k, v, o, lse, idx, cnt)
    ps = 16
    kp, vp, bt = wl.paged_pool(k, v, ps, seed=2)
    bt[0, 0] = kp.shape[0] + 5  # every row selects key 0's page: out of the pool
    pp = P.abi_params(w)
    pp.t_kv = bt.shape[1] * ps
    qs = wl.sparse_layer_query(w, 0).to(DEV)
    og = torch.empty_like(qs)
    lg = torch.empty(w.batch, w.hq, w.tq, dtype=torch.float32, device=DEV)
    hs.hs_sparse_attn_reuse_paged(pp, _pages(bt, ps, kp.shape[0]), qs, kp, vp, idx, cnt, og, lg)
    assert hs.hs_device_status() == hs.HS_ERR_BOUNDS
    assert hs.hs_device_status() == 0
