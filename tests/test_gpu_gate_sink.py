"""GPU parity of the sparse-layer output epilogue (hs_sparse_gate_sink): per-head
sinks and the sigmoid-gate fusion of the two branches, against the fp64 oracle
(oracle.gate_sink) on the very branch outputs the library produced.

The branch outputs themselves are checked by test_gpu_parity.py; here they are
inputs, copied exactly (bf16 or fp32 -> fp64) to the oracle, so the comparison
isolates the epilogue.  Bars as in tests/parity.py.
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


def _branches(w):
    """Full layer, then sparse layer 0 of w through the library: o/lse of both branches."""
    q, k, v, _ = wl.full_layer_inputs(w)
    q, k, v = [t.to(DEV) for t in (q, k, v)]
    p = P.abi_params(w)
    o, lse, idx, cnt, _ = hs.full_outputs(p, DEV)
    hs.hs_full_attn_index(p, q, k, v, o, lse, idx, cnt)
    qs = wl.sparse_layer_query(w, 0).to(DEV)
    og = torch.empty_like(qs)
    lg = torch.empty(w.batch, w.hq, w.tq, dtype=torch.float32, device=DEV)
    kl = vl = ol = ll = None
    if w.swa_branch:
        kl, vl = [t.to(DEV) for t in wl.sparse_layer_local_kv(w, 0)]
        ol, ll = torch.empty_like(qs), torch.empty_like(lg)
    hs.hs_sparse_attn_reuse(p, qs, k, v, idx, cnt, kl, vl, og, lg, ol, ll)
    torch.cuda.synchronize()
    assert hs.hs_device_status() == 0
    return p, og, lg, ol, ll


def _knobs(w, seed):
    g = torch.Generator().manual_seed(seed)
    sink = lambda: (torch.randn(w.hq, generator=g) * 2.0).to(DEV)  # noqa: E731
    gate = lambda: (torch.randn(w.batch, w.hq, w.tq, generator=g) * 3.0).to(DEV)  # noqa: E731
    return sink(), sink(), gate(), gate()


def _expect(og, lg, ol, ll, sg, sl, zg, zl):
    f = lambda t: None if t is None else P.f64(t)  # noqa: E731
    return oracle.gate_sink(f(og), f(lg), f(ol), f(ll), f(sg), f(sl), f(zg), f(zl))


@pytest.mark.parametrize("in_place", [False, True])
def test_two_branches_block_bf16(in_place):
    w = wl.scaled(wl.WORKLOADS["hysparse_7b_block"], name="gs_block", hq=8, hkv=2, t=300, k=256,
                  window=64)
    p, og, lg, ol, ll = _branches(w)
    sg, sl, zg, zl = _knobs(w, 11)
    o_want, lg_want, ll_want = _expect(og, lg, ol, ll, sg, sl, zg, zl)
    o = og if in_place else torch.empty_like(og)
    hs.hs_sparse_gate_sink(p, og, lg, o, ol, ll, sg, sl, zg, zl)
    torch.cuda.synchronize()
    assert hs.hs_device_status() == 0
    P.check_o(P.f64(o), o_want, "bf16", "gate_sink o")
    P.check_lse(P.f64(lg), lg_want, "bf16", "gate_sink lse_g")
    P.check_lse(P.f64(ll), ll_want, "bf16", "gate_sink lse_l")


def test_one_branch_token_fp32_in_place():
    w = wl.WORKLOADS["tiny_token"]
    p, og, lg, _, _ = _branches(w)
    sg, _, zg, _ = _knobs(w, 12)
    o_want, lg_want, _ = _expect(og, lg, None, None, sg, None, zg, None)
    hs.hs_sparse_gate_sink(p, og, lg, og, sink_global=sg, gate_global=zg)
    torch.cuda.synchronize()
    assert hs.hs_device_status() == 0
    P.check_o(P.f64(og), o_want, "fp32", "gate_sink o (one branch)")
    P.check_lse(P.f64(lg), lg_want, "fp32", "gate_sink lse_g (one branch)")


def test_sink_only_and_empty_rows_fp32():
    """Rows whose branch kept nothing (o = 0, lse = -inf) end with o = 0 and
    lse = the sink; other rows are only rescaled (no gates)."""
    b, hq, t, d = 2, 4, 37, 64
    p = hs.make_params(b, hq, 2, d, t, t, 0, "fp32", "token", 1, 16, 4)
    g = torch.Generator().manual_seed(13)
    og = torch.randn(b, hq, t, d, generator=g).to(DEV)
    lg = (torch.randn(b, hq, t, generator=g) * 4.0).to(DEV)
    og[:, :, ::5] = 0.0
    lg[:, :, ::5] = float("-inf")
    sg = torch.randn(hq, generator=g).to(DEV)
    o_want, lg_want, _ = _expect(og, lg, None, None, sg, None, None, None)
    o = torch.empty_like(og)
    hs.hs_sparse_gate_sink(p, og, lg, o, sink_global=sg)
    torch.cuda.synchronize()
    P.check_o(P.f64(o), o_want, "fp32", "gate_sink o (sink only)")
    assert torch.all(o[:, :, ::5] == 0)
    np.testing.assert_array_equal(P.f64(lg)[:, :, ::5],
                                  np.broadcast_to(P.f64(sg)[None, :, None], (b, hq, 8)))
    P.check_lse(P.f64(lg), lg_want, "fp32", "gate_sink lse (sink only)")
