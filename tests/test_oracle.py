"""Pins of the fp64 oracle against facts that do not come from the oracle.

Each test checks one function of ``oracle/`` against a library routine, a
closed form, an invariant the pages state, or brute force on tiny inputs:

* attention and lse      -- torch's own scaled_dot_product_attention and
                            logsumexp in float64 ("HySparse 混合稀疏注意力（一）",
                            exact attention formulas);
* block / token scores   -- a materialised probability matrix from
                            torch.softmax, reduced by torch.amax (block max,
                            then max over the GQA group);
* top-k                  -- exhaustive enumeration of every candidate subset;
* cardinality            -- |I_t| = k/B (16 at B=64, k=1024, printed on the page);
* forced window          -- every window token is selected ("HySparse2 ..." 4.2);
* sparse == dense        -- when the budget covers every visible token;
* retained mass          -- o_full = a o_S + (1-a) o_notS and the 2(1-a)V_max bound;
* closed forms           -- equal keys give uniform attention and the lowest ids.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def _rand(shape, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g, dtype=torch.float64) * std).numpy()


def _mk(b=1, hq=4, hkv=2, T=29, d=16, seed=0, std=1.0, t_q=None):
    t_q = T if t_q is None else t_q
    q = _rand((b, hq, t_q, d), seed, std)
    k = _rand((b, hkv, T, d), seed + 1, std)
    v = _rand((b, hkv, T, d), seed + 2, std)
    return q, k, v


def _library_attention(q, k, v, q_offset=0, scale=None):
    """torch SDPA (float64, math backend) with the causal mask of a query chunk."""
    b, hq, tq, d = q.shape
    hkv, T = k.shape[1], k.shape[2]
    g = hq // hkv
    qt = torch.from_numpy(q)
    kt = torch.from_numpy(k).repeat_interleave(g, dim=1)
    vt = torch.from_numpy(v).repeat_interleave(g, dim=1)
    pos = torch.arange(tq)[:, None] + q_offset
    mask = torch.arange(T)[None, :] <= pos
    sc = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=sc)
    logits = torch.einsum("bhqd,bhkd->bhqk", qt, kt) * sc
    logits = logits.masked_fill(~mask, float("-inf"))
    lse = torch.logsumexp(logits, dim=-1)
    p = torch.softmax(logits, dim=-1)
    return o.numpy(), lse.numpy(), p.numpy()


def _per_row(arr_bh, rows, g):
    """Pick [n, g, ...] out of a [b, hq, tq, ...] library result for oracle rows."""
    out = []
    for (b, u, j) in rows:
        out.append(np.stack([arr_bh[b, u * g + hh, j] for hh in range(g)]))
    return np.stack(out)


@pytest.mark.parametrize("mode", ["block", "token"])
@pytest.mark.parametrize("q_offset,t_q", [(0, None), (9, 20)])
def test_attention_and_lse_match_library(mode, q_offset, t_q):
    T = 29
    q, k, v = _mk(b=2, hq=4, hkv=2, T=T, d=16, seed=3, t_q=t_q)
    p = oracle.Params(2, 4, 2, 16, q.shape[2], T, mode=mode, block_size=4, k=8, window=3,
                      q_offset=q_offset)
    r = oracle.full_attn_index(p, q, k, v)
    o_ref, lse_ref, _ = _library_attention(q, k, v, q_offset=q_offset)
    np.testing.assert_allclose(r["o"], _per_row(o_ref, r["rows"], 2), rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["lse"], _per_row(lse_ref, r["rows"], 2), rtol=0, atol=1e-12)


@pytest.mark.parametrize("B", [1, 4, 5, 8])
def test_block_scores_are_group_max_of_block_max_probability(B):
    """S_{t,r} = max_{i in B_r} p_{t,i}, then max over the GQA group (materialised P)."""
    T, g = 23, 3
    q, k, v = _mk(b=1, hq=6, hkv=2, T=T, d=8, seed=11)
    p = oracle.Params(1, 6, 2, 8, T, T, mode="block", block_size=B, k=2 * B, window=0)
    r = oracle.full_attn_index(p, q, k, v, want_scores=True)
    _, _, P = _library_attention(q, k, v)
    nb = -(-T // B)
    for n, (b, u, j) in enumerate(r["rows"]):
        probs = torch.from_numpy(P[b, u * g:(u + 1) * g, j])  # [g, T], zeros past j
        padded = torch.nn.functional.pad(probs, (0, nb * B - T), value=-1.0)
        blockmax = padded.view(g, nb, B).amax(dim=-1).amax(dim=0).numpy()
        visible = -(-(j + 1) // B)
        np.testing.assert_allclose(r["scores"][n, :visible], blockmax[:visible], rtol=1e-12,
                                   atol=0)
        assert np.all(r["scores"][n, visible:] == -1.0)


def _beats(a, b):
    """(score, id) order of the pages' top-k with the lower-index tie-break."""
    return a[0] > b[0] or (a[0] == b[0] and a[1] < b[1])


def _brute_topk(scores, cand_ids, K):
    """The unique subset of size K whose members all beat all non-members."""
    found = []
    for sub in itertools.combinations(cand_ids, K):
        s = set(sub)
        ins = [(scores[i], i) for i in sub]
        outs = [(scores[i], i) for i in cand_ids if i not in s]
        if all(_beats(x, y) for x in ins for y in outs):
            found.append(sorted(sub))
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_block_topk_equals_exhaustive_enumeration(seed):
    T, B, K = 24, 3, 3  # 8 blocks, choose 3
    q, k, v = _mk(b=1, hq=2, hkv=1, T=T, d=4, seed=20 + seed)
    # force exact ties between blocks so the tie-break is exercised
    k[0, 0, 6:9] = k[0, 0, 0:3]
    k[0, 0, 15:18] = k[0, 0, 0:3]
    p = oracle.Params(1, 2, 1, 4, T, T, mode="block", block_size=B, k=K * B, window=0)
    r = oracle.full_attn_index(p, q, k, v, want_scores=True)
    for n, (_, _, j) in enumerate(r["rows"]):
        nb = -(-(j + 1) // B)
        cnt = r["cnt"][n]
        if nb <= K:
            assert cnt == nb and list(r["idx"][n, :cnt]) == list(range(nb))
            continue
        want = _brute_topk(r["scores"][n], list(range(nb)), K)
        assert cnt == K and list(r["idx"][n, :cnt]) == want
        assert np.all(r["idx"][n, cnt:] == -1)


@pytest.mark.parametrize("w", [0, 2, 5])
def test_token_topk_equals_exhaustive_enumeration_with_forced_window(w):
    T, K = 14, 6
    q, k, v = _mk(b=1, hq=2, hkv=1, T=T, d=4, seed=31)
    p = oracle.Params(1, 2, 1, 4, T, T, mode="token", block_size=1, k=K, window=w)
    r = oracle.full_attn_index(p, q, k, v, want_scores=True)
    for n, (_, _, t) in enumerate(r["rows"]):
        got = list(r["idx"][n, :r["cnt"][n]])
        if t + 1 <= K:
            assert got == list(range(t + 1))
            continue
        window = list(range(t - w + 1, t + 1))
        outside = list(range(0, t - w + 1))
        want = sorted(_brute_topk(r["scores"][n], outside, K - w) + window)
        assert got == want


def test_cardinality_printed_example():
    """|I_t| = k/B = 16 at B=64, k=1024 once t+1 >= k; min(k/B, ceil((t+1)/B)) before."""
    T = 1100
    q, k, v = _mk(b=1, hq=1, hkv=1, T=T, d=4, seed=5)
    rows = np.array([[0, 0, t] for t in (0, 63, 64, 500, 1022, 1023, 1099)])
    p = oracle.Params(1, 1, 1, 4, T, T, mode="block", block_size=64, k=1024, window=128)
    r = oracle.full_attn_index(p, q, k, v, rows=rows)
    for n, (_, _, t) in enumerate(rows):
        assert r["cnt"][n] == min(16, -(-(t + 1) // 64))
    assert r["cnt"][-1] == 16 and r["cnt"][-2] == 16


def test_token_cardinality_and_window():
    T = 300
    q, k, v = _mk(b=1, hq=2, hkv=1, T=T, d=8, seed=6)
    p = oracle.Params(1, 2, 1, 8, T, T, mode="token", block_size=1, k=40, window=16)
    r = oracle.full_attn_index(p, q, k, v)
    for n, (_, _, t) in enumerate(r["rows"]):
        ids = r["idx"][n, :r["cnt"][n]]
        assert r["cnt"][n] == min(40, t + 1)
        assert set(range(max(0, t - 15), t + 1)) <= set(ids.tolist())
        assert np.all(np.diff(ids) > 0) and ids.max() <= t


def test_block_size_one_equals_token_mode_without_window():
    T = 40
    q, k, v = _mk(b=1, hq=4, hkv=2, T=T, d=8, seed=8)
    pb = oracle.Params(1, 4, 2, 8, T, T, mode="block", block_size=1, k=7, window=0)
    pt = oracle.Params(1, 4, 2, 8, T, T, mode="token", block_size=1, k=7, window=0)
    rb = oracle.full_attn_index(pb, q, k, v)
    rt = oracle.full_attn_index(pt, q, k, v)
    assert np.array_equal(rb["idx"], rt["idx"]) and np.array_equal(rb["cnt"], rt["cnt"])


def test_equal_keys_closed_form_and_lowest_index_tie_break():
    """All keys equal: p = 1/(t+1), o = mean(v[0..t]), lse = a + log(t+1); all scores tie."""
    T, d = 50, 8
    q, _, v = _mk(b=1, hq=2, hkv=1, T=T, d=d, seed=9)
    k = np.repeat(_rand((1, 1, 1, d), 99), T, axis=2)
    for mode, B, K, w in (("block", 4, 12, 0), ("token", 1, 10, 3)):
        p = oracle.Params(1, 2, 1, d, T, T, mode=mode, block_size=B, k=K, window=w)
        r = oracle.full_attn_index(p, q, k, v)
        for n, (_, _, t) in enumerate(r["rows"]):
            mean_v = v[0, 0, :t + 1].mean(axis=0)
            np.testing.assert_allclose(r["o"][n], np.stack([mean_v, mean_v]), atol=1e-12)
            a = q[0, :, t] @ k[0, 0, 0] / math.sqrt(d)
            np.testing.assert_allclose(r["lse"][n], a + math.log(t + 1), atol=1e-12)
            ids = list(r["idx"][n, :r["cnt"][n]])
            if mode == "block":
                assert ids == list(range(min(3, -(-(t + 1) // B))))
            elif t + 1 <= K:
                assert ids == list(range(t + 1))
            else:
                assert ids == list(range(K - w)) + list(range(t - w + 1, t + 1))


def test_sparse_equals_dense_when_budget_covers_everything():
    T = 33
    q, k, v = _mk(b=1, hq=4, hkv=2, T=T, d=8, seed=12)
    for mode, B in (("token", 1), ("block", 8)):
        p = oracle.Params(1, 4, 2, 8, T, T, mode=mode, block_size=B, k=40, window=4)
        full = oracle.full_attn_index(p, q, k, v)
        qs = _rand(q.shape, 77)
        sp = oracle.sparse_attn(p, qs, k, v, full["idx"], full["cnt"], rows=full["rows"])
        o_ref, lse_ref, _ = _library_attention(qs, k, v)
        np.testing.assert_allclose(sp["o_g"], _per_row(o_ref, sp["rows"], 2), atol=1e-12)
        np.testing.assert_allclose(sp["lse_g"], _per_row(lse_ref, sp["rows"], 2), atol=1e-12)


def test_block_sparse_masks_future_keys_inside_a_selected_block():
    """A selected block that crosses t contributes only keys <= t."""
    T, B = 20, 8
    q, k, v = _mk(b=1, hq=1, hkv=1, T=T, d=8, seed=13)
    p = oracle.Params(1, 1, 1, 8, T, T, mode="block", block_size=B, k=8, window=0)
    rows = np.array([[0, 0, 10]])
    sp = oracle.sparse_attn(p, q, k, v, np.array([[1]]), np.array([1]), rows=rows)
    # keys 8..10 only: library attention over that slice
    qt = torch.from_numpy(q[0, 0, 10][None, None, None])
    kt = torch.from_numpy(k[0, 0, 8:11][None, None])
    vt = torch.from_numpy(v[0, 0, 8:11][None, None])
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt).numpy()[0, 0, 0]
    np.testing.assert_allclose(sp["o_g"][0, 0], ref, atol=1e-12)


def test_local_window_branch_matches_banded_library_attention():
    T, w = 26, 5
    q, _, _ = _mk(b=1, hq=4, hkv=2, T=T, d=8, seed=14)
    kl, vl = _rand((1, 2, T, 8), 15), _rand((1, 2, T, 8), 16)
    p = oracle.Params(1, 4, 2, 8, T, T, mode="block", block_size=4, k=8, window=w)
    idx = np.zeros((2 * T, 2), dtype=np.int32); cnt = np.ones(2 * T, dtype=np.int32)
    sp = oracle.sparse_attn(p, q, kl, vl, idx, cnt, k_loc=kl, v_loc=vl)
    qt = torch.from_numpy(q)
    kt = torch.from_numpy(kl).repeat_interleave(2, dim=1)
    vt = torch.from_numpy(vl).repeat_interleave(2, dim=1)
    i = torch.arange(T)
    band = (i[None, :] <= i[:, None]) & (i[None, :] > i[:, None] - w)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=band).numpy()
    np.testing.assert_allclose(sp["o_l"], _per_row(ref, sp["rows"], 2), atol=1e-12)


def test_retained_mass_decomposition_and_bound():
    """o_full = a o_S + (1-a) o_notS;  |o_full - o_S| <= 2 (1-a) V_max."""
    T = 60
    q, k, v = _mk(b=1, hq=2, hkv=1, T=T, d=8, seed=17)
    p = oracle.Params(1, 2, 1, 8, T, T, mode="token", block_size=1, k=12, window=3)
    full = oracle.full_attn_index(p, q, k, v)
    qs = _rand(q.shape, 18)
    sp = oracle.sparse_attn(p, qs, k, v, full["idx"], full["cnt"], rows=full["rows"])
    o_ref, _, P = _library_attention(qs, k, v)
    vmax = np.linalg.norm(v[0, 0], axis=-1).max()
    for n, (_, _, t) in enumerate(full["rows"]):
        S = full["idx"][n, :full["cnt"][n]]
        notS = np.setdiff1d(np.arange(t + 1), S)
        for hh in range(2):
            alpha = P[0, hh, t, S].sum()
            o_full = o_ref[0, hh, t]
            o_s = sp["o_g"][n, hh]
            if len(notS):
                pn = oracle.Params(1, 2, 1, 8, T, T, mode="token", block_size=1, k=T, window=0)
                ids = np.full((1, T), -1, dtype=np.int32); ids[0, :len(notS)] = notS
                comp = oracle.sparse_attn(pn, qs, k, v, ids, np.array([len(notS)]),
                                          rows=np.array([[0, 0, t]]))["o_g"][0, hh]
                np.testing.assert_allclose(alpha * o_s + (1 - alpha) * comp, o_full, atol=1e-12)
            else:
                assert abs(alpha - 1) < 1e-12
            assert np.linalg.norm(o_full - o_s) <= 2 * (1 - alpha) * vmax + 1e-12


def test_decode_row_equals_prefill_last_row():
    T, L = 40, 31
    q, k, v = _mk(b=2, hq=4, hkv=2, T=T, d=8, seed=19)
    lens = np.array([L, T], dtype=np.int32)
    pd = oracle.Params(2, 4, 2, 8, 1, T, mode="token", block_size=1, k=9, window=2)
    qd = q[:, :, :1]
    rd = oracle.full_attn_index(pd, qd, k, v, kv_len=lens)
    for bi, Lb in enumerate(lens):
        qp = np.zeros_like(q[bi:bi + 1, :, :Lb]); qp[:, :, Lb - 1] = qd[bi, :, 0]
        pp = oracle.Params(1, 4, 2, 8, Lb, T, mode="token", block_size=1, k=9, window=2)
        rows = np.array([[0, u, Lb - 1] for u in range(2)])
        rp = oracle.full_attn_index(pp, qp, k[bi:bi + 1], v[bi:bi + 1], rows=rows)
        for u in range(2):
            n = bi * 2 + u
            np.testing.assert_allclose(rd["o"][n], rp["o"][u], atol=1e-13)
            assert list(rd["idx"][n]) == list(rp["idx"][u])


def test_needles_are_selected_for_their_query():
    from oracle_top_kv_b200 import workloads as wl
    w = wl.WORKLOADS["tiny_block"]
    q, k, v, plants = wl.full_layer_inputs(w)
    p = oracle.Params(w.batch, w.hq, w.hkv, w.head_dim, w.t, w.t, mode="block",
                      block_size=w.block_size, k=w.k, window=w.window)
    rows = np.array([[b, u, j] for (b, u, i, h, j) in plants])
    r = oracle.full_attn_index(p, q.double().numpy(), k.double().numpy(), v.double().numpy(),
                               rows=rows)
    for n, (b, u, i, h, j) in enumerate(plants):
        assert i // w.block_size in set(r["idx"][n, :r["cnt"][n]].tolist())


# ------------------------------------------------------------- gate and sink
def test_sink_is_an_extra_key_with_zero_value():
    """A per-head sink bias s_h is one more logit in the softmax whose value
    vector is zero: attention over the keys plus such a key (built so that
    tau q_h . k_s = s_h for both heads of the group) must give gate_sink's o'
    and lse' applied to attention over the keys alone."""
    d, L = 8, 11
    q = _rand((1, 2, 1, d), 31)
    k = _rand((1, 1, L, d), 32)
    v = _rand((1, 1, L, d), 33)
    s = np.array([0.7, -1.3])
    tau = 1.0 / math.sqrt(d)
    Q = q[0, :, 0, :]                                     # [2, d]
    k_s = Q.T @ np.linalg.solve(Q @ Q.T, s / tau)         # tau * Q k_s = s
    np.testing.assert_allclose(tau * Q @ k_s, s, atol=1e-12)
    k_aug = np.concatenate([k_s.reshape(1, 1, 1, d), k], axis=2)
    v_aug = np.concatenate([np.zeros((1, 1, 1, d)), v], axis=2)
    pa = oracle.Params(1, 2, 1, d, 1, L + 1, mode="token", block_size=1, k=L + 1, window=1,
                       q_offset=L)
    ra = oracle.full_attn_index(pa, q, k_aug, v_aug)
    pr = oracle.Params(1, 2, 1, d, 1, L, mode="token", block_size=1, k=L, window=1,
                       q_offset=L - 1)
    rr = oracle.full_attn_index(pr, q, k, v)
    o_g = rr["o"][0][None, :, None, :]                     # [1, 2, 1, d]
    lse_g = rr["lse"][0][None, :, None]
    o, lse, _ = oracle.gate_sink(o_g, lse_g, sink_g=s)
    np.testing.assert_allclose(o[0, :, 0], ra["o"][0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0, :, 0], ra["lse"][0], rtol=0, atol=1e-12)


def test_gate_identities():
    """sigma(0) = 1/2 on both branches; sigma(z) + sigma(-z) = 1, so equal
    branch outputs with opposite gate logits give that output back; a very
    negative gate logit removes its branch."""
    o_g = _rand((2, 3, 5, 4), 41)
    o_l = _rand((2, 3, 5, 4), 42)
    lse_g = _rand((2, 3, 5), 43)
    lse_l = _rand((2, 3, 5), 44)
    z = _rand((2, 3, 5), 45, std=3.0)
    zero = np.zeros((2, 3, 5))
    o, lg, ll = oracle.gate_sink(o_g, lse_g, o_l, lse_l, z_g=zero, z_l=zero)
    np.testing.assert_allclose(o, 0.5 * (o_g + o_l), rtol=0, atol=1e-14)
    np.testing.assert_array_equal(lg, lse_g)
    np.testing.assert_array_equal(ll, lse_l)
    o, _, _ = oracle.gate_sink(o_g, lse_g, o_g, lse_g, z_g=z, z_l=-z)
    np.testing.assert_allclose(o, o_g, rtol=0, atol=1e-14)
    o, _, _ = oracle.gate_sink(o_g, lse_g, o_l, lse_l, z_g=z, z_l=np.full_like(z, -800.0))
    np.testing.assert_allclose(o, o_g / (1.0 + np.exp(-z))[..., None], rtol=0, atol=1e-14)


def test_sink_on_an_empty_branch():
    """A branch that kept no key (o = 0, lse = -inf) keeps o' = 0 and gets
    lse' = s: the sink is then the whole softmax mass."""
    o_g = np.zeros((1, 2, 3, 4))
    lse_g = np.full((1, 2, 3), -np.inf)
    o, lse, _ = oracle.gate_sink(o_g, lse_g, sink_g=[0.25, -2.0])
    assert np.all(o == 0.0)
    np.testing.assert_array_equal(lse[0, :, 0], [0.25, -2.0])
