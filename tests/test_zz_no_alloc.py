"""The allocation-free sparse decode entry point.

hs_decode_sparse_noalloc serves callers that cannot allocate device memory
(an engine plugin handed only its input and output buffers, or a decode loop
that must not call cudaMalloc).  It runs the sparse decode kernels with a
scratch array that lives inside the library.  These tests call it through the
C ABI twice in a row -- the second call reuses the scratch the first one left
behind -- and compare each output both with hs_decode_step(HS_DECODE_SPARSE)
on the same inputs and with the fp64 oracle on sampled (sequence, group)
units, under the parity tests' bf16 bar; one case fills the scratch array to
its last unit.  The file is named to be collected last, so that a run
stopping at the first failure has run every other test first; it also passes
alone in a fresh process.
"""
import numpy as np
import pytest
import torch

from oracle_top_kv_b200 import hs
from oracle_top_kv_b200 import workloads as wl
from tests import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(w, seq_cpu, units, layers=2):
    q, kc, vc, _ = wl.full_layer_inputs(w)
    q, kc, vc = q.to(DEV), kc.to(DEV), vc.to(DEV)
    seq = seq_cpu.to(DEV)
    p = P.abi_params(w, decode=True)
    idx = torch.empty(w.batch, w.hkv, p.ksel, dtype=torch.int32, device=DEV)
    cnt = torch.empty(w.batch, w.hkv, dtype=torch.int32, device=DEV)
    o = torch.empty_like(q)
    lse = torch.empty(w.batch, w.hq, 1, dtype=torch.float32, device=DEV)
    hs.hs_decode_step(p, hs.HS_DECODE_FULL_INDEX, q, kc, vc, seq, idx, cnt, o, lse, None,
                      hs.workspace(p, hs.HS_WS_DECODE_FULL))
    wss = hs.workspace(p, hs.HS_WS_DECODE_SPARSE)
    rows = np.array([[b, u, 0] for (b, u) in units], np.int32)
    pos = seq_cpu.numpy().astype(np.int64)[rows[:, 0]] - 1
    g = w.group
    for layer in range(layers):  # calls in a row share the library's scratch
        qs = wl.sparse_layer_query(w, layer).to(DEV)
        o_ref = torch.empty_like(qs)
        l_ref = torch.empty(w.batch, w.hq, 1, dtype=torch.float32, device=DEV)
        hs.hs_decode_step(p, hs.HS_DECODE_SPARSE, qs, kc, vc, seq, idx, cnt, o_ref, l_ref, None,
                          wss)
        o_na = torch.full_like(qs, float("nan"))
        l_na = torch.full((w.batch, w.hq, 1), float("nan"), dtype=torch.float32, device=DEV)
        hs.hs_decode_sparse_noalloc(p, qs, kc, vc, seq, idx, cnt, o_na, l_na)
        torch.cuda.synchronize()
        assert hs.hs_device_status() == 0
        # against the entry point that takes a workspace, every row
        P.check_o(P.f64(o_na)[:, :, 0], P.f64(o_ref)[:, :, 0], "bf16", f"noalloc layer {layer}")
        P.check_lse(l_na.cpu().double().numpy(), l_ref.cpu().double().numpy(), "bf16",
                    f"noalloc lse layer {layer}")
        # against the fp64 oracle on the GPU's own index sets, sampled units
        g_idx = idx.cpu().numpy()[rows[:, 0], rows[:, 1]]
        g_cnt = cnt.cpu().numpy()[rows[:, 0], rows[:, 1]]
        sp = P.oracle_sparse_rows(w, qs, kc, vc, g_idx, g_cnt, rows, pos)
        P.check_o(P.gpu_rows(P.f64(o_na), rows, True, g), sp["o_g"], "bf16",
                  f"noalloc vs oracle layer {layer}")
        P.check_lse(P.gpu_rows(l_na.cpu().double().numpy(), rows, True, g), sp["lse_g"], "bf16",
                    f"noalloc lse vs oracle layer {layer}")


def test_noalloc_sparse_decode_matches_workspace_path_and_oracle():
    w = wl.scaled(wl.WORKLOADS["hysparse2_decode"], name="noalloc", batch=8, hq=64, hkv=4,
                  t=20000, k=1024, window=128)
    seq = torch.tensor([20000, 1, 700, 1024, 1025, 19999, 5000, 12345], dtype=torch.int32)
    units = [(0, 0), (1, 3), (2, 1), (3, 2), (4, 0), (6, 3), (7, 1)]
    _run(w, seq, units)


def test_noalloc_at_the_scratch_limit():
    """63 sequences x 4 groups x ceil(1024/64) = 4032 split units: the whole array."""
    w = wl.scaled(wl.WORKLOADS["hysparse2_decode"], name="noalloc_limit", batch=63, hq=64,
                  hkv=4, t=2048, k=1024, window=128)
    seq = torch.full((63,), 2048, dtype=torch.int32)
    seq[5] = 1500
    seq[62] = 1100
    _run(w, seq, [(0, 0), (5, 2), (31, 1), (62, 3)], layers=2)


def test_noalloc_rejects_calls_beyond_its_scratch():
    w = wl.scaled(wl.WORKLOADS["hysparse2_decode"], name="noalloc_big", batch=64, hq=64, hkv=4,
                  t=4096, k=1024, window=128)
    p = P.abi_params(w, decode=True)
    t = torch.empty(16, dtype=torch.int32, device=DEV)
    with pytest.raises(hs.HsError) as e:
        hs.hs_decode_sparse_noalloc(p, t, t, t, t, t, t, t, t)
    assert e.value.code == hs.HS_ERR_WORKSPACE
