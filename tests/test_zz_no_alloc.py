"""The allocation-free sparse decode entry point gives the same result as
the workspace version.

hs_decode_sparse_noalloc serves callers that cannot allocate device memory
(an engine plugin handed only its input and output buffers, or a decode loop
that must not call cudaMalloc).  It runs the sparse decode kernels with a
scratch array that lives inside the library.  This test calls it through the
C ABI twice in a row -- the second call reuses the scratch the first one left
behind -- and compares each output with hs_decode_step(HS_DECODE_SPARSE) on
the same inputs, under the parity tests' bf16 bar.  The file is named to be
collected last, so that a run stopping at the first failure has run every
other test first; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

from oracle_top_kv_b200 import hs
from oracle_top_kv_b200 import workloads as wl
from tests import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_noalloc_sparse_decode_matches_workspace_path():
    w = wl.scaled(wl.WORKLOADS["hysparse2_decode"], name="noalloc", batch=8, hq=64, hkv=4,
                  t=20000, k=1024, window=128)
    q, kc, vc, _ = wl.full_layer_inputs(w)
    q, kc, vc = q.to(DEV), kc.to(DEV), vc.to(DEV)
    seq = torch.tensor([20000, 1, 700, 1024, 1025, 19999, 5000, 12345], dtype=torch.int32,
                       device=DEV)
    p = P.abi_params(w, decode=True)
    idx = torch.empty(w.batch, w.hkv, p.ksel, dtype=torch.int32, device=DEV)
    cnt = torch.empty(w.batch, w.hkv, dtype=torch.int32, device=DEV)
    o = torch.empty_like(q)
    lse = torch.empty(w.batch, w.hq, 1, dtype=torch.float32, device=DEV)
    hs.hs_decode_step(p, hs.HS_DECODE_FULL_INDEX, q, kc, vc, seq, idx, cnt, o, lse, None,
                      hs.workspace(p, hs.HS_WS_DECODE_FULL))
    wss = hs.workspace(p, hs.HS_WS_DECODE_SPARSE)
    for layer in range(2):  # two calls in a row share the library's scratch
        qs = wl.sparse_layer_query(w, layer).to(DEV)
        o_ref = torch.empty_like(qs)
        l_ref = torch.empty(w.batch, w.hq, 1, dtype=torch.float32, device=DEV)
        hs.hs_decode_step(p, hs.HS_DECODE_SPARSE, qs, kc, vc, seq, idx, cnt, o_ref, l_ref, None,
                          wss)
        o_na = torch.empty_like(qs)
        l_na = torch.empty(w.batch, w.hq, 1, dtype=torch.float32, device=DEV)
        hs.hs_decode_sparse_noalloc(p, qs, kc, vc, seq, idx, cnt, o_na, l_na)
        torch.cuda.synchronize()
        assert hs.hs_device_status() == 0
        P.check_o(P.f64(o_na)[:, :, 0], P.f64(o_ref)[:, :, 0], "bf16", f"noalloc layer {layer}")
        P.check_lse(l_na.cpu().double().numpy(), l_ref.cpu().double().numpy(), "bf16",
                    f"noalloc lse layer {layer}")


def test_noalloc_rejects_calls_beyond_its_scratch():
    w = wl.scaled(wl.WORKLOADS["hysparse2_decode"], name="noalloc_big", batch=64, hq=64, hkv=4,
                  t=4096, k=1024, window=128)
    p = P.abi_params(w, decode=True)
    t = torch.empty(16, dtype=torch.int32, device=DEV)
    with pytest.raises(hs.HsError) as e:
        hs.hs_decode_sparse_noalloc(p, t, t, t, t, t, t, t, t)
    assert e.value.code == hs.HS_ERR_WORKSPACE
