"""The benchmark's work formulas reproduce the numbers the pages print."""
import json
import os

import pytest

from oracle_top_kv_b200 import accounting as A

G = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_numbers.json")))


def test_kv_cache_sizes():
    for key in ("one_full_layer_kv_mib", "full_model_kv_mib"):
        assert A.kv_cache_bytes(**G[key]["args"]) / A.MIB == G[key]["value"]
    hy = A.hysparse_cache_bytes(**G["hysparse_kv_mib"]["args"]) / A.MIB
    assert round(hy) == G["hysparse_kv_mib"]["value"]
    full = A.kv_cache_bytes(**G["full_model_kv_mib"]["args"]) / A.MIB
    assert round(full / hy, 2) == G["hysparse_reduction"]["value"]


def test_prefill_ratio():
    g = G["prefill_cost_ratio"]
    a = g["args"]
    L = a["F"] + a["S"]
    # the page prints both terms and their sum to 3 places ("about")
    assert abs(a["F"] / L - g["terms"][0]) < 1e-3
    assert abs(a["S"] / L * (a["k"] + a["w"]) / a["T"] - g["terms"][1]) < 1e-3
    assert abs(A.prefill_cost_ratio(**a) - g["value"]) < 1e-3


def test_decode_reads():
    hy = A.decode_token_reads(**G["decode_reads_hysparse"]["args"])
    full = A.decode_token_reads(**G["decode_reads_full"]["args"])
    assert hy == G["decode_reads_hysparse"]["value"] and full == G["decode_reads_full"]["value"]
    assert round(hy / full, 3) == G["decode_read_ratio"]["value"]


def test_block_scores_and_blocks_per_query():
    n = A.block_score_elements(**G["block_scores_per_head_millions"]["args"])
    assert round(n / 1e6, 2) == G["block_scores_per_head_millions"]["value"]
    a = G["blocks_per_query"]["args"]
    assert a["k"] // a["B"] == G["blocks_per_query"]["value"]


def test_full_layer_flops_matches_pair_count():
    # 7B-shaped prefill: b=2, 32 heads, d=128, T=16384
    f = A.full_layer_flops(2, 32, 128, 16384)
    assert f == 4 * 128 * 32 * 2 * (16384 * 16385 // 2)
    assert abs(f - 4.398e12) / 4.398e12 < 1e-3
    # a chunk at the end of a prefix sees q_offset more keys per row
    assert A.causal_pairs(3, 10) == 11 + 12 + 13


def test_sparse_rows_from_index_block_clipping():
    torch = pytest.importorskip("torch")
    idx = torch.tensor([[[[0, 1], [0, 1], [0, -1]]]], dtype=torch.int32)  # t = 4, 5, 6 with B=4
    cnt = torch.tensor([[[2, 2, 1]]], dtype=torch.int32)
    # row t=4: block0 (4 keys) + block1 keys 4..4 (1); t=5: 4 + 2; t=6: 4
    assert A.sparse_rows_from_index(idx, cnt, "block", 4, q_offset=4) == 5 + 6 + 4
    assert A.window_rows(1, 1, 3, 2, q_offset=0) == 1 + 2 + 2


def test_sparse_useful_flops_brute_force():
    """The block-sparse roofline's work: 4*d per (query head, kept key), where a
    row keeps the keys <= t of its selected blocks and, with the window branch,
    the keys t-w+1..t of its own K'/V'; counted here by enumerating pairs."""
    torch = pytest.importorskip("torch")
    import importlib
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    bench = importlib.import_module("bench")
    from oracle_top_kv_b200 import workloads as wl
    w = wl.scaled(wl.WORKLOADS["hysparse_7b_block"], name="tiny", batch=2, hq=6, hkv=2, t=40,
                  block_size=8, k=24, window=5)
    g = torch.Generator().manual_seed(7)
    b, hkv, tq, ks = w.batch, w.hkv, w.tq, w.ksel
    idx = torch.full((b, hkv, tq, ks), -1, dtype=torch.int32)
    cnt = torch.zeros(b, hkv, tq, dtype=torch.int32)
    for bb in range(b):
        for u in range(hkv):
            for t in range(tq):
                nb = t // w.block_size + 1
                c = int(torch.randint(0, min(ks, nb) + 1, (1,), generator=g))
                sel = torch.randperm(nb, generator=g)[:c].sort().values
                idx[bb, u, t, :c] = sel.to(torch.int32)
                cnt[bb, u, t] = c

    class Blk:
        pass
    blk = Blk()
    blk.idx, blk.cnt = idx, cnt
    pairs = 0
    for bb in range(b):
        for u in range(hkv):
            for t in range(tq):
                keys = set()
                for x in range(int(cnt[bb, u, t])):
                    r = int(idx[bb, u, t, x])
                    keys |= {i for i in range(r * w.block_size, (r + 1) * w.block_size) if i <= t}
                window = {i for i in range(max(0, t - w.window + 1), t + 1)} if w.swa_branch else set()
                pairs += (len(keys) + len(window)) * (w.hq // w.hkv)
    assert bench.sparse_useful_flops(w, blk) == pairs * 4 * w.head_dim


def test_code_hash_ignores_comments_not_code(tmp_path, monkeypatch):
    """The DRAM-traffic table is tied to a kernel's code: a comment or spacing
    edit keeps its hash, any code edit changes it."""
    import importlib
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    bench = importlib.import_module("bench")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    f = tmp_path / "k.cu"
    f.write_text("// header\nint f(int x) { /* twice */ return 2 * x; }\n")
    h0 = bench.code_hash(["k.cu"])
    f.write_text("// a longer header\n\nint f(int x) {\n    // doubled\n    return 2 * x;\n}\n")
    assert bench.code_hash(["k.cu"]) == h0
    f.write_text("// header\nint f(int x) { /* twice */ return 3 * x; }\n")
    assert bench.code_hash(["k.cu"]) != h0


def test_sparse_unique_rows_brute_force():
    """Distinct K/V rows a sparse layer touches (its least memory traffic),
    counted by enumerating every row's kept keys into one set per unit."""
    torch = pytest.importorskip("torch")
    g = torch.Generator().manual_seed(11)
    b, hkv, tq, off = 2, 3, 30, 9
    for mode, B, ks in (("token", 1, 7), ("block", 4, 3)):
        idx = torch.full((b, hkv, tq, ks), -1, dtype=torch.int32)
        cnt = torch.zeros(b, hkv, tq, dtype=torch.int32)
        want = 0
        for bb in range(b):
            for u in range(hkv):
                keys = set()
                for j in range(tq):
                    t = off + j
                    nc = t // B + 1
                    c = int(torch.randint(0, min(ks, nc) + 1, (1,), generator=g))
                    sel = torch.randperm(nc, generator=g)[:c].sort().values
                    idx[bb, u, j, :c] = sel.to(torch.int32)
                    cnt[bb, u, j] = c
                    for r in sel.tolist():
                        keys |= {i for i in range(r * B, (r + 1) * B) if i <= t}
                want += len(keys)
        assert A.sparse_unique_rows_from_index(idx, cnt, mode, B, q_offset=off) == want
        got = A.sparse_layer_unique_bytes(want, b, 6, tq, 8, 2, ks, hkv)
        assert got == want * 2 * 8 * 2 + b * 6 * tq * 8 * 2 + b * 6 * tq * (8 * 2 + 4) + \
            b * hkv * tq * (ks + 1) * 4
