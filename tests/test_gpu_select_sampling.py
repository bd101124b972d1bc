"""The token selectors' sampled start threshold changes how many keys enter
the candidate buffers, never which keys are selected: with it automatic, off,
forced to rank 1 (every position's threshold too high, so each work item is
detected and scanned again) or to a rank that fails only some positions, the
index sets and scores must be bit-identical, and the automatic one must pass
the oracle check ("HySparse2 ..." 4.2: the k - w best of 0..t-w by the
token score, plus the last w)."""
import pytest
import torch

from oracle_top_kv_b200 import hs
from oracle_top_kv_b200 import workloads as wl
from tests import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = {
    # >= 2048 key tiles with a workspace: the wide selector (16 positions per item)
    "wide": (wl.scaled(wl.WORKLOADS["long_1m_chunk"], name="sample_wide", hq=16, hkv=1,
                       t=266240, t_q=40, q_offset=266200, k=1024, window=128,
                       needles="loguniform:16"), True),
    # the same long scan without a workspace: the shared-memory selector's
    # deep-ring configuration (1408-entry buffers, 10 sampled tiles)
    "smem_long": (wl.scaled(wl.WORKLOADS["long_1m_chunk"], name="sample_smem_long", hq=16, hkv=1,
                            t=266240, t_q=40, q_offset=266200, k=1024, window=128,
                            needles="loguniform:16"), False),
    # a shorter scan without a workspace: the shared-memory selector
    "smem": (wl.scaled(wl.WORKLOADS["hysparse2_prefill"], name="sample_smem", hq=32, hkv=2,
                       t=40000, t_q=40, q_offset=39960, k=1024, window=128,
                       needles="frac:0.01"), False),
}


# Many more work items than SMs (2 groups x 150 items of 16 positions): the
# persistent wide selector takes several items per CTA, so forced rescans
# land in the middle of a CTA's item sequence.  Compared across sampling
# ranks only (the oracle check of the same kernel runs on the cases above).
MANY_ITEMS = wl.scaled(wl.WORKLOADS["long_1m_chunk"], name="sample_wide_many", hq=32, hkv=2,
                       t=266240, t_q=2400, q_offset=263840, k=1024, window=128,
                       needles="loguniform:16")


@pytest.fixture(autouse=True)
def _restore():
    hs.load()
    assert hs.hs_device_status() == 0
    yield
    hs.hs_set_select_sampling(-1)


@pytest.mark.parametrize("case", sorted(CASES))
def test_sampled_threshold_never_changes_the_selection(case):
    w, use_ws = CASES[case]
    q, k, v, _ = wl.full_layer_inputs(w)
    q, k, v = (t.to(DEV).contiguous() for t in (q, k, v))
    p = P.abi_params(w)
    ws = hs.workspace(p, hs.HS_WS_FULL) if use_ws else None
    outs = {}
    for rank in (-1, 0, 1, 7, 1000):
        hs.hs_set_select_sampling(rank)
        o, lse, idx, cnt, sel = hs.full_outputs(p, with_scores=True)
        idx.fill_(-7)
        cnt.fill_(-7)
        hs.hs_full_attn_index(p, q, k, v, o, lse, idx, cnt, sel, ws)
        torch.cuda.synchronize()
        assert hs.hs_device_status() == 0, f"{case} rank {rank}"
        outs[rank] = (idx.cpu(), cnt.cpu(), sel.cpu())
    ref = outs[-1]
    for rank, got in outs.items():
        assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1]), \
            f"{case}: index with sampling rank {rank} differs from the automatic one"
        assert torch.equal(got[2], ref[2]), f"{case}: scores with sampling rank {rank}"
    rws = P.all_rows(w)
    orc = P.oracle_full_rows(w, q, k, v, rws, w.q_offset + rws[:, 2])
    P.check_index(P.gpu_rows(ref[0].numpy(), rws, False), P.gpu_rows(ref[1].numpy(), rws, False),
                  orc, w.mode, w.window, w.k, f"{case} index (sampled threshold)")


def test_sampled_threshold_many_items_per_cta():
    w = MANY_ITEMS
    q, k, v, _ = wl.full_layer_inputs(w, device=DEV)
    p = P.abi_params(w)
    ws = hs.workspace(p, hs.HS_WS_FULL)
    assert ws is not None
    outs = {}
    for rank in (-1, 0, 1, 9):
        hs.hs_set_select_sampling(rank)
        o, lse, idx, cnt, _ = hs.full_outputs(p)
        idx.fill_(-7)
        cnt.fill_(-7)
        hs.hs_full_attn_index(p, q, k, v, o, lse, idx, cnt, None, ws)
        torch.cuda.synchronize()
        assert hs.hs_device_status() == 0, f"rank {rank}"
        outs[rank] = (idx.cpu(), cnt.cpu())
    for rank, got in outs.items():
        assert torch.equal(got[0], outs[0][0]) and torch.equal(got[1], outs[0][1]), \
            f"index with sampling rank {rank} differs from the unsampled scan"
    assert int(outs[0][1].min()) == w.k  # every position ranks (t + 1 > k)
