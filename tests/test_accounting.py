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
