"""GPU parity: the C-ABI CUDA path against the fp64 oracle on the same seeded
inputs, element by element at sizes the oracle finishes in seconds (several
tiles plus ragged tails), and on sampled rows at the workloads' full sizes.
"""
import numpy as np
import pytest
import torch

from oracle_top_kv_b200 import hs
from oracle_top_kv_b200 import workloads as wl
from tests import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    hs.load()
    assert hs.hs_device_status() == 0


def _cuda(*ts):
    return [t.to(DEV).contiguous() for t in ts]


def edge_rows(w, extra_random=24, seed=0):
    """Sampled (b, u, j) rows: the method's edge positions plus random ones."""
    tq, off = w.tq, w.q_offset
    pos = {0, tq - 1}
    for t_abs in (w.window - 1, w.window, w.k - 1, w.k, w.k + 1, w.block_size - 1,
                  w.block_size, 2 * w.block_size + 3, w.t - 1, w.t - 2):
        if off <= t_abs < off + tq:
            pos.add(t_abs - off)
    rng = np.random.default_rng(seed)
    pos |= set(rng.integers(0, tq, size=extra_random).tolist())
    rows = []
    for j in sorted(pos):
        rows.append((int(rng.integers(0, w.batch)), int(rng.integers(0, w.hkv)), j))
    rows.append((w.batch - 1, w.hkv - 1, tq - 1))
    return np.array(rows, dtype=np.int32)


def run_full(w, gen_device="cpu", rows=None, check_scores=True):
    q, k, v, plants = wl.full_layer_inputs(w, device=gen_device)
    q, k, v = _cuda(q, k, v)
    p = P.abi_params(w)
    o, lse, idx, cnt, sel = hs.full_outputs(p, with_scores=True)
    ws = hs.workspace(p, hs.HS_WS_FULL)
    hs.hs_full_attn_index(p, q, k, v, o, lse, idx, cnt, sel, ws)
    torch.cuda.synchronize()
    assert hs.hs_device_status() == 0
    rws = P.all_rows(w) if rows is None else rows
    pos = w.q_offset + rws[:, 2]
    orc = P.oracle_full_rows(w, q, k, v, rws, pos)
    g = w.group
    P.check_o(P.gpu_rows(P.f64(o), rws, True, g), orc["o"], w.dtype, f"{w.name} full o")
    P.check_lse(P.gpu_rows(lse.cpu().double().numpy(), rws, True, g), orc["lse"], w.dtype,
                f"{w.name} full lse")
    g_idx = P.gpu_rows(idx.cpu().numpy(), rws, False)
    g_cnt = P.gpu_rows(cnt.cpu().numpy(), rws, False)
    P.check_index(g_idx, g_cnt, orc, w.mode, w.window, w.k, f"{w.name} index")
    if w.mode == "token":
        # Without score output the selectors take their other finalize paths
        # (id bitmap): same kernel, same arithmetic, so identical index sets.
        # Without the workspace a long scan takes the shared-memory selector
        # instead of the wide one, whose scores round differently (the wide
        # one folds lse into the contraction): that set must pass the oracle
        # check on its own.
        for wsx in ([ws, None] if ws is not None else [None]):
            idx2, cnt2 = torch.full_like(idx, -7), torch.full_like(cnt, -7)
            hs.hs_full_attn_index(p, q, k, v, torch.empty_like(o), torch.empty_like(lse), idx2,
                                  cnt2, None, wsx)
            torch.cuda.synchronize()
            assert hs.hs_device_status() == 0
            if wsx is ws:
                assert torch.equal(idx2, idx) and torch.equal(cnt2, cnt), \
                    f"{w.name}: index without scores"
            else:
                P.check_index(P.gpu_rows(idx2.cpu().numpy(), rws, False),
                              P.gpu_rows(cnt2.cpu().numpy(), rws, False), orc, w.mode, w.window,
                              w.k, f"{w.name} index without workspace")
    if check_scores:
        g_sel = P.gpu_rows(sel.cpu().double().numpy(), rws, False)
        for n in range(len(g_cnt)):
            ids = g_idx[n, :g_cnt[n]]
            want = orc["scores"][n][ids]
            np.testing.assert_allclose(g_sel[n, :g_cnt[n]], want, rtol=2e-3, atol=0,
                                       err_msg=f"{w.name} sel_scores row {n}")
            assert np.all(g_sel[n, g_cnt[n]:] == 0)
    return dict(q=q, k=k, v=v, idx=idx, cnt=cnt, rows=rws, pos=pos, g_idx=g_idx, g_cnt=g_cnt,
                plants=plants)


def run_sparse(w, full, layer, gen_device="cpu"):
    qs = wl.sparse_layer_query(w, layer, device=gen_device).to(DEV)
    p = P.abi_params(w)
    og = torch.empty_like(qs)
    lg = torch.empty(w.batch, w.hq, w.tq, dtype=torch.float32, device=DEV)
    kl = vl = ol = ll = None
    if w.swa_branch:
        kl, vl = _cuda(*wl.sparse_layer_local_kv(w, layer, device=gen_device))
        ol = torch.empty_like(qs)
        ll = torch.empty_like(lg)
    hs.hs_sparse_attn_reuse(p, qs, full["k"], full["v"], full["idx"], full["cnt"], kl, vl, og, lg,
                            ol, ll)
    torch.cuda.synchronize()
    assert hs.hs_device_status() == 0
    rws = full["rows"]
    sp = P.oracle_sparse_rows(w, qs, full["k"], full["v"], full["g_idx"], full["g_cnt"], rws,
                              full["pos"], kl, vl)
    g = w.group
    P.check_o(P.gpu_rows(P.f64(og), rws, True, g), sp["o_g"], w.dtype, f"{w.name} L{layer} o_g")
    P.check_lse(P.gpu_rows(lg.cpu().double().numpy(), rws, True, g), sp["lse_g"], w.dtype,
                f"{w.name} L{layer} lse_g")
    if w.swa_branch:
        P.check_o(P.gpu_rows(P.f64(ol), rws, True, g), sp["o_l"], w.dtype,
                  f"{w.name} L{layer} o_l")
        P.check_lse(P.gpu_rows(ll.cpu().double().numpy(), rws, True, g), sp["lse_l"], w.dtype,
                    f"{w.name} L{layer} lse_l")


# ---------------------------------------------------------------- small cases
SMALL = {
    "tiny_block": wl.WORKLOADS["tiny_block"],
    "tiny_token": wl.WORKLOADS["tiny_token"],
    "bf16_block_g4_B64": wl.scaled(wl.WORKLOADS["hysparse_7b_block"], name="bf16_block_g4_B64",
                                   hq=8, hkv=2, t=300, k=128),
    "bf16_block_g16_B16_d64": wl.scaled(wl.WORKLOADS["hysparse_7b_block"],
                                        name="bf16_block_g16_B16_d64", hq=16, hkv=1,
                                        head_dim=64, t=200, block_size=16, k=64, window=32),
    "bf16_block_g1_B32": wl.scaled(wl.WORKLOADS["hysparse_7b_block"], name="bf16_block_g1_B32",
                                   batch=1, hq=3, hkv=3, t=161, block_size=32, k=64, window=16),
    "bf16_token_g16": wl.scaled(wl.WORKLOADS["hysparse2_prefill"], name="bf16_token_g16",
                                hq=32, hkv=2, t=700, k=256, window=64),
    "bf16_token_g4_d64_w0": wl.scaled(wl.WORKLOADS["hysparse2_prefill"],
                                      name="bf16_token_g4_d64_w0", batch=2, hq=8, hkv=2,
                                      head_dim=64, t=333, k=40, window=0),
    "bf16_token_w_eq_k": wl.scaled(wl.WORKLOADS["hysparse2_prefill"], name="bf16_token_w_eq_k",
                                   hq=4, hkv=1, t=150, k=24, window=24),
    "bf16_token_chunk": wl.scaled(wl.WORKLOADS["long_1m_chunk"], name="bf16_token_chunk",
                                  hq=16, hkv=1, t=1500, t_q=300, q_offset=1200, k=256, window=32),
    # a scan of >= 2048 key tiles: the selector's deep-ring instantiation
    "bf16_token_long_scan": wl.scaled(wl.WORKLOADS["long_1m_chunk"], name="bf16_token_long_scan",
                                      hq=16, hkv=1, t=266240, t_q=40, q_offset=266200, k=1024,
                                      window=128, needles="loguniform:16"),
    # HySparse2's MQA 64/1 at head dim 256 (SIMT kernels), and 64/1 at d = 128
    # (tensor-core attention pass, SIMT selection); a 32-head block-mode group
    # at d = 256 with the window branch
    "bf16_token_mqa64_d256": wl.scaled(wl.WORKLOADS["hysparse2_prefill"],
                                       name="bf16_token_mqa64_d256", hq=64, hkv=1, head_dim=256,
                                       t=600, k=256, window=64),
    "bf16_token_mqa64_d128": wl.scaled(wl.WORKLOADS["hysparse2_prefill"],
                                       name="bf16_token_mqa64_d128", hq=64, hkv=1, t=700, k=256,
                                       window=64),
    "bf16_block_g32_d256": wl.scaled(wl.WORKLOADS["hysparse_7b_block"], name="bf16_block_g32_d256",
                                     batch=1, hq=32, hkv=1, head_dim=256, t=400, k=256, window=64),
    "bf16_select_all": wl.scaled(wl.WORKLOADS["hysparse2_prefill"], name="bf16_select_all",
                                 hq=4, hkv=2, t=100, k=128, window=16),
    "bf16_single_token": wl.scaled(wl.WORKLOADS["hysparse2_prefill"], name="bf16_single_token",
                                   hq=4, hkv=2, t=1, k=16, window=4, needles="count:0"),
    # block mode, B = 64: the row-grouped tensor-core sparse kernel (group of
    # 16 with a ragged length; group of 2; a chunk at a nonzero offset)
    "bf16_block_g16_B64_ragged": wl.scaled(wl.WORKLOADS["hysparse_7b_block"],
                                           name="bf16_block_g16_B64_ragged", batch=1, hq=32,
                                           hkv=2, t=520, k=1024, window=128),
    "bf16_block_g2_B64": wl.scaled(wl.WORKLOADS["hysparse_7b_block"], name="bf16_block_g2_B64",
                                   hq=4, hkv=2, t=400, k=256, window=64),
    "bf16_block_g4_B64_chunk": wl.scaled(wl.WORKLOADS["hysparse_7b_block"],
                                         name="bf16_block_g4_B64_chunk", batch=1, hq=8, hkv=2,
                                         t=900, t_q=250, q_offset=650, k=512, window=64),
}


@pytest.mark.parametrize("name", sorted(SMALL))
def test_small_full_and_sparse(name):
    w = SMALL[name]
    full = run_full(w)
    for layer in range(min(w.n_sparse, 3)):
        run_sparse(w, full, layer)


def test_needles_selected_by_gpu():
    w = wl.WORKLOADS["tiny_token"]
    full = run_full(w)
    idx = full["idx"].cpu().numpy()
    cnt = full["cnt"].cpu().numpy()
    for (b, u, i, h, j) in full["plants"]:
        assert i in set(idx[b, u, j, :cnt[b, u, j]].tolist())


def test_bounds_error_sets_status_without_fault():
    w = SMALL["bf16_token_g4_d64_w0"]
    full = run_full(w)
    bad = full["idx"].clone()
    bad[0, 0, 5, 0] = 10_000  # beyond the row's position
    p = P.abi_params(w)
    qs = wl.sparse_layer_query(w, 0).to(DEV)
    og = torch.empty_like(qs)
    lg = torch.empty(w.batch, w.hq, w.tq, dtype=torch.float32, device=DEV)
    hs.hs_sparse_attn_reuse(p, qs, full["k"], full["v"], bad, full["cnt"], None, None, og, lg)
    assert hs.hs_device_status() == hs.HS_ERR_BOUNDS
    assert hs.hs_device_status() == 0  # reading clears it


def test_block_sparse_custom_index_sets():
    """Block mode, B = 64, with index sets made up here rather than by the full
    layer: empty rows, rows of one block, full rows, blocks crossing the row's
    position, and the window branch -- against the oracle's sparse formula."""
    w = wl.scaled(wl.WORKLOADS["hysparse_7b_block"], name="block_custom", batch=2, hq=8, hkv=2,
                  t=700, k=512, window=96)
    q, k, v, _ = wl.full_layer_inputs(w)
    q, k, v = _cuda(q, k, v)
    ks = w.k // w.block_size
    rng = np.random.default_rng(5)
    idx = np.full((w.batch, w.hkv, w.tq, ks), -1, np.int32)
    cnt = np.zeros((w.batch, w.hkv, w.tq), np.int32)
    for b in range(w.batch):
        for u in range(w.hkv):
            for j in range(w.tq):
                nb = j // w.block_size + 1
                kind = rng.integers(0, 4)
                c = 0 if kind == 0 else 1 if kind == 1 else min(ks, nb) if kind == 2 else \
                    int(rng.integers(1, min(ks, nb) + 1))
                ids = np.sort(rng.choice(nb, size=c, replace=False)) if c else np.zeros(0, int)
                if kind == 1:
                    ids = np.array([nb - 1])  # the block holding the row: in-block causal clip
                idx[b, u, j, :c] = ids
                cnt[b, u, j] = c
    p = P.abi_params(w)
    qs = wl.sparse_layer_query(w, 0).to(DEV)
    kl, vl = _cuda(*wl.sparse_layer_local_kv(w, 0))
    og, ol = torch.empty_like(qs), torch.empty_like(qs)
    lg = torch.empty(w.batch, w.hq, w.tq, dtype=torch.float32, device=DEV)
    ll = torch.empty_like(lg)
    hs.hs_sparse_attn_reuse(p, qs, k, v, torch.from_numpy(idx).to(DEV),
                            torch.from_numpy(cnt).to(DEV), kl, vl, og, lg, ol, ll)
    torch.cuda.synchronize()
    assert hs.hs_device_status() == 0
    rws = P.all_rows(w)
    pos = w.q_offset + rws[:, 2]
    g_idx = idx[rws[:, 0], rws[:, 1], rws[:, 2]]
    g_cnt = cnt[rws[:, 0], rws[:, 1], rws[:, 2]]
    sp = P.oracle_sparse_rows(w, qs, k, v, g_idx, g_cnt, rws, pos, kl, vl)
    g = w.group
    P.check_o(P.gpu_rows(P.f64(og), rws, True, g), sp["o_g"], w.dtype, "custom o_g")
    P.check_lse(P.gpu_rows(lg.cpu().double().numpy(), rws, True, g), sp["lse_g"], w.dtype,
                "custom lse_g")
    P.check_o(P.gpu_rows(P.f64(ol), rws, True, g), sp["o_l"], w.dtype, "custom o_l")
    P.check_lse(P.gpu_rows(ll.cpu().double().numpy(), rws, True, g), sp["lse_l"], w.dtype,
                "custom lse_l")
    # empty rows: o = 0, lse = -inf
    e = np.argwhere(cnt == 0)[0]
    for hh in range(g):
        h = e[1] * g + hh
        assert torch.all(og[e[0], h, e[2]] == 0)
        assert lg[e[0], h, e[2]].item() == -np.inf


def test_block_sparse_bounds_status():
    w = SMALL["bf16_block_g4_B64"]
    full = run_full(w)
    bad = full["idx"].clone()
    bad[0, 0, 5, 0] = 7  # block 7 starts beyond position 5
    p = P.abi_params(w)
    qs = wl.sparse_layer_query(w, 0).to(DEV)
    og = torch.empty_like(qs)
    lg = torch.empty(w.batch, w.hq, w.tq, dtype=torch.float32, device=DEV)
    hs.hs_sparse_attn_reuse(p, qs, full["k"], full["v"], bad, full["cnt"], None, None, og, lg)
    assert hs.hs_device_status() == hs.HS_ERR_BOUNDS
    assert hs.hs_device_status() == 0


# -------------------------------------------------------------------- decode
def run_decode(w, seq_len, layers=2, gen_device="cpu", units=None, use_ws=True):
    q, kc, vc, _ = wl.full_layer_inputs(w, device=gen_device)
    q, kc, vc = _cuda(q, kc, vc)
    sl = seq_len.to(DEV).to(torch.int32)
    p = P.abi_params(w, decode=True)
    ksel = p.ksel
    idx = torch.empty(w.batch, w.hkv, ksel, dtype=torch.int32, device=DEV)
    cnt = torch.empty(w.batch, w.hkv, dtype=torch.int32, device=DEV)
    sel = torch.empty(w.batch, w.hkv, ksel, dtype=torch.float32, device=DEV)
    o = torch.empty_like(q)
    lse = torch.empty(w.batch, w.hq, 1, dtype=torch.float32, device=DEV)
    ws = hs.workspace(p, hs.HS_WS_DECODE_FULL) if use_ws else None
    hs.hs_decode_step(p, hs.HS_DECODE_FULL_INDEX, q, kc, vc, sl, idx, cnt, o, lse, sel, ws)
    torch.cuda.synchronize()
    assert hs.hs_device_status() == 0
    lens = seq_len.cpu().numpy().astype(np.int32)
    if units is None:
        rows = np.array([[b, u, 0] for b in range(w.batch) for u in range(w.hkv)], np.int32)
    else:
        rows = np.array([[b, u, 0] for (b, u) in units], np.int32)
    pos = lens[rows[:, 0]] - 1
    orc = P.oracle_full_rows(w, q, kc, vc, rows, pos)
    g = w.group
    P.check_o(P.gpu_rows(P.f64(o), rows, True, g), orc["o"], w.dtype, f"{w.name} decode o")
    P.check_lse(P.gpu_rows(lse.cpu().double().numpy(), rows, True, g), orc["lse"], w.dtype,
                f"{w.name} decode lse")
    g_idx = idx.cpu().numpy()[rows[:, 0], rows[:, 1]]
    g_cnt = cnt.cpu().numpy()[rows[:, 0], rows[:, 1]]
    P.check_index(g_idx, g_cnt, orc, "token", w.window, w.k, f"{w.name} decode index")
    g_sel = sel.cpu().double().numpy()[rows[:, 0], rows[:, 1]]
    for n in range(len(g_cnt)):
        ids = g_idx[n, :g_cnt[n]]
        np.testing.assert_allclose(g_sel[n, :g_cnt[n]], orc["scores"][n][ids], rtol=2e-3)
    wss = hs.workspace(p, hs.HS_WS_DECODE_SPARSE) if use_ws else None
    for layer in range(layers):
        qs = wl.sparse_layer_query(w, layer, device=gen_device).to(DEV)
        os_ = torch.empty_like(qs)
        ls = torch.empty(w.batch, w.hq, 1, dtype=torch.float32, device=DEV)
        hs.hs_decode_step(p, hs.HS_DECODE_SPARSE, qs, kc, vc, sl, idx, cnt, os_, ls, None, wss)
        torch.cuda.synchronize()
        assert hs.hs_device_status() == 0
        sp = P.oracle_sparse_rows(w, qs, kc, vc, g_idx, g_cnt, rows, pos)
        P.check_o(P.gpu_rows(P.f64(os_), rows, True, g), sp["o_g"], w.dtype,
                  f"{w.name} decode sparse L{layer}")
        P.check_lse(P.gpu_rows(ls.cpu().double().numpy(), rows, True, g), sp["lse_g"], w.dtype,
                    f"{w.name} decode sparse lse L{layer}")


def test_decode_small_ragged():
    w = wl.scaled(wl.WORKLOADS["hysparse2_decode"], name="decode_small", batch=4, hq=32, hkv=2,
                  t=5000, k=256, window=64)
    run_decode(w, torch.tensor([5000, 1, 200, 4097], dtype=torch.int32))


def test_decode_single_sequence_two_level_merge():
    # one sequence and one KV group: the selector splits the cache into 35
    # slices, so their candidates are merged in two levels
    w = wl.scaled(wl.WORKLOADS["hysparse2_decode"], name="decode_one_seq", batch=1, hq=16, hkv=1,
                  t=70000, k=512, window=64)
    run_decode(w, torch.tensor([69999], dtype=torch.int32), layers=1)


def test_decode_small_g4_d64():
    w = wl.scaled(wl.WORKLOADS["hysparse2_decode"], name="decode_g4", batch=2, hq=8, hkv=2,
                  head_dim=64, t=3000, k=100, window=10)
    run_decode(w, torch.tensor([2999, 3000], dtype=torch.int32))


def test_decode_mqa64_d256():
    """HySparse2's MQA 64/1 at head dim 256 (split-k CUDA-core decode)."""
    w = wl.scaled(wl.WORKLOADS["hysparse2_decode"], name="decode_mqa64_d256", batch=3, hq=64,
                  hkv=1, head_dim=256, t=2500, k=256, window=64)
    run_decode(w, torch.tensor([2500, 1, 1300], dtype=torch.int32))


def test_decode_mqa64_d256_without_workspace():
    """The same shape without a workspace: one CTA per sequence and group."""
    w = wl.scaled(wl.WORKLOADS["hysparse2_decode"], name="decode_mqa64_d256_nows", batch=2, hq=64,
                  hkv=1, head_dim=256, t=1500, k=256, window=64)
    run_decode(w, torch.tensor([1500, 700], dtype=torch.int32), layers=1, use_ws=False)


def test_decode_wide_groups_split():
    """Groups of 64 heads at d = 128, 32 at d = 64, 18 at d = 128 and 4 at d =
    256 (split-k CUDA-core decode; splits of 512 keys with a ragged last one,
    short and 1-key caches)."""
    w = wl.scaled(wl.WORKLOADS["hysparse2_decode"], name="decode_g64_d128", batch=2, hq=128,
                  hkv=2, head_dim=128, t=1700, k=300, window=32)
    run_decode(w, torch.tensor([1700, 513], dtype=torch.int32), layers=1)
    w = wl.scaled(wl.WORKLOADS["hysparse2_decode"], name="decode_g32_d64", batch=2, hq=32,
                  hkv=1, head_dim=64, t=900, k=128, window=16)
    run_decode(w, torch.tensor([1, 900], dtype=torch.int32), layers=1)
    # 18 heads: warps own 3 or 2 heads, logit rows not 16-byte multiples
    w = wl.scaled(wl.WORKLOADS["hysparse2_decode"], name="decode_g18", batch=1, hq=18, hkv=1,
                  head_dim=128, t=600, k=128, window=16)
    run_decode(w, torch.tensor([600], dtype=torch.int32), layers=1)
    # 4 heads at d = 256: half the warps own no head
    w = wl.scaled(wl.WORKLOADS["hysparse2_decode"], name="decode_g4_d256", batch=2, hq=8, hkv=2,
                  head_dim=256, t=800, k=128, window=16)
    run_decode(w, torch.tensor([800, 129], dtype=torch.int32), layers=1)


def test_decode_bad_length_sets_status():
    w = wl.scaled(wl.WORKLOADS["hysparse2_decode"], name="decode_bad", batch=2, hq=8, hkv=2,
                  t=512, k=64, window=8)
    q, kc, vc, _ = wl.full_layer_inputs(w)
    q, kc, vc = _cuda(q, kc, vc)
    p = P.abi_params(w, decode=True)
    sl = torch.tensor([512, 513], dtype=torch.int32, device=DEV)  # 513 > capacity
    idx = torch.empty(2, 2, 64, dtype=torch.int32, device=DEV)
    cnt = torch.empty(2, 2, dtype=torch.int32, device=DEV)
    o = torch.empty_like(q)
    lse = torch.empty(2, 8, 1, dtype=torch.float32, device=DEV)
    hs.hs_decode_step(p, hs.HS_DECODE_FULL_INDEX, q, kc, vc, sl, idx, cnt, o, lse, None,
                      hs.workspace(p, hs.HS_WS_DECODE_FULL))
    assert hs.hs_device_status() == hs.HS_ERR_BOUNDS
    assert int(cnt[1, 0]) == 0 and int(cnt[0, 0]) == 64


# ------------------------------------------------------- full-size workloads
@pytest.mark.parametrize("name", ["hysparse_7b_block", "hysparse2_prefill", "long_1m_chunk"])
def test_full_size_prefill_sampled_rows(name):
    w = wl.WORKLOADS[name]
    rows = edge_rows(w)
    full = run_full(w, gen_device=DEV, rows=rows)
    run_sparse(w, full, 0, gen_device=DEV)
    del full
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["hysparse2_decode", "long_1m_decode"])
def test_full_size_decode_sampled_units(name):
    w = wl.WORKLOADS[name]
    rng = np.random.default_rng(3)
    units = sorted({(int(rng.integers(0, w.batch)), int(rng.integers(0, w.hkv)))
                    for _ in range(6)} | {(w.batch - 1, w.hkv - 1)})
    run_decode(w, wl.decode_seq_lens(w, ragged=w.batch > 1), layers=1, gen_device=DEV,
               units=units)
    torch.cuda.empty_cache()
