"""Bounded waits give up cleanly (failure detection without a GPU fault).

Every wait of a kernel on another role of its CTA is bounded; when the bound
runs out the kernel records HS_ERR_TIMEOUT in the device status word, drains
its in-flight TMA copies and MMAs, frees its tensor memory and returns.  Here
the bound is lowered to a few hundred SM cycles (hs_set_wait_limit), so the
first waits on a TMA copy or an MMA run out on purpose: the full layer (the
tcgen05 attention pipeline, then the token selector; and the block-mode
kernel with its indexer) must report the timeout, and with the default bound
restored the next call on the same device must pass the oracle parity check.
"""
import numpy as np
import pytest
import torch

from oracle_top_kv_b200 import hs
from oracle_top_kv_b200 import workloads as wl
from tests import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = {
    "token": wl.scaled(wl.WORKLOADS["hysparse2_prefill"], name="timeout_token", hq=32, hkv=2,
                       t=1500, k=256, window=64),
    "block": wl.scaled(wl.WORKLOADS["hysparse_7b_block"], name="timeout_block", batch=1, hq=16,
                       hkv=4, t=900, k=512, window=64),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_wait_bound_runs_out_then_the_device_is_usable(name):
    w = CASES[name]
    q, k, v, _ = wl.full_layer_inputs(w)
    q, k, v = q.to(DEV), k.to(DEV), v.to(DEV)
    p = P.abi_params(w)
    o, lse, idx, cnt, _ = hs.full_outputs(p)
    hs.load()
    assert hs.hs_device_status() == 0
    try:
        hs.hs_set_wait_limit(300)
        hs.hs_full_attn_index(p, q, k, v, o, lse, idx, cnt)
        torch.cuda.synchronize()
        assert hs.hs_device_status() == hs.HS_ERR_TIMEOUT
    finally:
        hs.hs_set_wait_limit(0)
    # the same call with the default bound: clean status and oracle parity
    hs.hs_full_attn_index(p, q, k, v, o, lse, idx, cnt)
    torch.cuda.synchronize()
    assert hs.hs_device_status() == 0
    rng = np.random.default_rng(1)
    rows = np.array([(0, int(rng.integers(0, w.hkv)), int(j))
                     for j in sorted(set(rng.integers(0, w.tq, 12).tolist()) | {0, w.tq - 1})],
                    np.int32)
    orc = P.oracle_full_rows(w, q, k, v, rows, w.q_offset + rows[:, 2])
    g = w.group
    P.check_o(P.gpu_rows(P.f64(o), rows, True, g), orc["o"], w.dtype, f"{name} o after timeout")
    P.check_index(P.gpu_rows(idx.cpu().numpy(), rows, False),
                  P.gpu_rows(cnt.cpu().numpy(), rows, False), orc, w.mode, w.window, w.k,
                  f"{name} index after timeout")
