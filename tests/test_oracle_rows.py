"""Pins of the oracle's sampled-row helpers (full_attn_rows, sparse_attn_rows).

Every GPU parity test evaluates only sampled rows: the helpers hand the C
oracle just those rows' query vectors with explicit positions (the q_pos path
of orc_position) and each (batch, group)'s K/V prefix 0..max(position).  Here
they are checked, on the CPU, against

* the whole-array oracle (rows = every row, positions from q_offset / kv_len,
  no q_pos), itself pinned to library attention and brute force in
  test_oracle.py, to 1e-13 -- outputs, lse, index sets, counts and scores;
* torch's float64 scaled_dot_product_attention directly, for o and lse.

The definition both must preserve is the row-wise one of "HySparse 混合稀疏注意力
（一）", "从精确注意力里提取块级分数": each query row sees keys 0..t of its own
group, independent of the other rows evaluated with it.
"""
import importlib.util
import math
import os
import shutil
import sys

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def _rand(shape, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g, dtype=torch.float64) * std).numpy()


def _inputs(b, hq, hkv, tq, T, d, seed):
    q = _rand((b, hq, tq, d), seed)
    k = _rand((b, hkv, T, d), seed + 1)
    v = _rand((b, hkv, T, d), seed + 2)
    # a few sharp keys so that the index sets are not all near-ties
    rng = np.random.default_rng(seed)
    for _ in range(6):
        bb, u = rng.integers(b), rng.integers(hkv)
        i, h, j = rng.integers(T), rng.integers(hq // hkv), rng.integers(tq)
        k[bb, u, i] = 3.0 * q[bb, u * (hq // hkv) + h, j]
    return q, k, v


def _row_sample(b, hkv, tq, n, seed):
    """n random (b, u, j) rows mixing units, plus the first and last row of each unit."""
    rng = np.random.default_rng(seed)
    rows = [(int(rng.integers(b)), int(rng.integers(hkv)), int(rng.integers(tq)))
            for _ in range(n)]
    for bb in range(b):
        for u in range(hkv):
            rows += [(bb, u, 0), (bb, u, tq - 1)]
    rng.shuffle(rows)
    return np.array(rows, np.int32)


def _whole_index(res, rows, p, decode=False):
    """Map each sampled row to its row number in the whole-array result."""
    tq = 1 if decode else p.t_q
    return [(int(b) * p.hkv + int(u)) * tq + int(j) for (b, u, j) in rows]


CASES = [
    # mode, b, hq, hkv, tq, T, d, q_offset, B, k, w
    ("block", 2, 6, 2, 37, 37, 8, 0, 4, 12, 0),
    ("token", 2, 6, 2, 37, 37, 8, 0, 1, 9, 3),
    ("block", 1, 8, 2, 20, 53, 8, 33, 4, 16, 0),   # a prefill chunk at an offset
    ("token", 1, 8, 2, 20, 53, 8, 33, 1, 12, 5),
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}_off{c[7]}" for c in CASES])
def test_full_rows_equal_whole_array_oracle(case):
    mode, b, hq, hkv, tq, T, d, off, B, kb, w = case
    q, k, v = _inputs(b, hq, hkv, tq, T, d, seed=41)
    p = oracle.Params(b, hq, hkv, d, tq, T, mode=mode, block_size=B, k=kb, window=w,
                      q_offset=off)
    whole = oracle.full_attn_index(p, q, k, v, want_scores=True)
    rows = _row_sample(b, hkv, tq, 25, seed=3)
    got = oracle.full_attn_rows(q, k, v, rows, off + rows[:, 2], mode, B, kb, w)
    at = _whole_index(whole, rows, p)
    np.testing.assert_allclose(got["o"], whole["o"][at], rtol=0, atol=1e-13)
    np.testing.assert_allclose(got["lse"], whole["lse"][at], rtol=0, atol=1e-13)
    assert np.array_equal(got["idx"], whole["idx"][at])
    assert np.array_equal(got["cnt"], whole["cnt"][at])
    for x, n in enumerate(at):
        s = got["scores"][x]
        ref = whole["scores"][n][:len(s)]
        np.testing.assert_allclose(s, ref, rtol=0, atol=1e-13)
        # past the row's prefix the whole-array scores are "no candidate"
        assert np.all(whole["scores"][n][len(s):] == -1.0)


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}_off{c[7]}" for c in CASES])
def test_sparse_rows_equal_whole_array_oracle(case):
    mode, b, hq, hkv, tq, T, d, off, B, kb, w = case
    q, k, v = _inputs(b, hq, hkv, tq, T, d, seed=43)
    qs = _rand((b, hq, tq, d), 90)
    kl, vl = _rand((b, hkv, T, d), 91), _rand((b, hkv, T, d), 92)
    p = oracle.Params(b, hq, hkv, d, tq, T, mode=mode, block_size=B, k=kb, window=max(w, 3),
                      q_offset=off)
    whole_f = oracle.full_attn_index(p, q, k, v)
    local = mode == "block"
    whole = oracle.sparse_attn(p, qs, k, v, whole_f["idx"], whole_f["cnt"],
                               k_loc=kl if local else None, v_loc=vl if local else None)
    rows = _row_sample(b, hkv, tq, 25, seed=5)
    at = _whole_index(whole, rows, p)
    got = oracle.sparse_attn_rows(qs, k, v, whole_f["idx"][at], whole_f["cnt"][at], rows,
                                  off + rows[:, 2], mode, B, kb, max(w, 3),
                                  kl if local else None, vl if local else None)
    np.testing.assert_allclose(got["o_g"], whole["o_g"][at], rtol=0, atol=1e-13)
    np.testing.assert_allclose(got["lse_g"], whole["lse_g"][at], rtol=0, atol=1e-13)
    if local:
        np.testing.assert_allclose(got["o_l"], whole["o_l"][at], rtol=0, atol=1e-13)
        np.testing.assert_allclose(got["lse_l"], whole["lse_l"][at], rtol=0, atol=1e-13)


def test_decode_rows_with_ragged_lengths_equal_whole_array_oracle():
    """Decode: one query per sequence at t = kv_len[b] - 1, lengths ragged."""
    b, hq, hkv, T, d = 4, 8, 2, 61, 8
    q, k, v = _inputs(b, hq, hkv, 1, T, d, seed=47)
    kv_len = np.array([61, 17, 40, 1], np.int32)
    for mode, B, kb, w in (("token", 1, 12, 4), ("block", 4, 8, 0)):
        p = oracle.Params(b, hq, hkv, d, 1, T, mode=mode, block_size=B, k=kb, window=w)
        whole = oracle.full_attn_index(p, q, k, v, kv_len=kv_len, want_scores=True)
        rows = np.array([(bb, u, 0) for bb in (3, 0, 2, 1) for u in (1, 0)], np.int32)
        pos = kv_len[rows[:, 0]] - 1
        got = oracle.full_attn_rows(q, k, v, rows, pos, mode, B, kb, w)
        at = _whole_index(whole, rows, p, decode=True)
        np.testing.assert_allclose(got["o"], whole["o"][at], rtol=0, atol=1e-13)
        np.testing.assert_allclose(got["lse"], whole["lse"][at], rtol=0, atol=1e-13)
        assert np.array_equal(got["idx"], whole["idx"][at])
        assert np.array_equal(got["cnt"], whole["cnt"][at])
        qs = _rand((b, hq, 1, d), 93)
        sw = oracle.sparse_attn(p, qs, k, v, whole["idx"], whole["cnt"], kv_len=kv_len)
        sg = oracle.sparse_attn_rows(qs, k, v, whole["idx"][at], whole["cnt"][at], rows, pos,
                                     mode, B, kb, w)
        np.testing.assert_allclose(sg["o_g"], sw["o_g"][at], rtol=0, atol=1e-13)
        np.testing.assert_allclose(sg["lse_g"], sw["lse_g"][at], rtol=0, atol=1e-13)


def test_full_rows_match_library_attention():
    """o and lse of sampled rows against torch's float64 SDPA on the whole chunk."""
    b, hq, hkv, tq, T, d, off = 2, 6, 3, 19, 45, 8, 26
    q, k, v = _inputs(b, hq, hkv, tq, T, d, seed=53)
    g = hq // hkv
    qt = torch.from_numpy(q)
    kt = torch.from_numpy(k).repeat_interleave(g, dim=1)
    vt = torch.from_numpy(v).repeat_interleave(g, dim=1)
    mask = torch.arange(T)[None, :] <= (torch.arange(tq)[:, None] + off)
    sc = 1.0 / math.sqrt(d)
    o_ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask,
                                                             scale=sc).numpy()
    logits = (torch.einsum("bhqd,bhkd->bhqk", qt, kt) * sc).masked_fill(~mask, float("-inf"))
    lse_ref = torch.logsumexp(logits, dim=-1).numpy()
    rows = _row_sample(b, hkv, tq, 20, seed=7)
    got = oracle.full_attn_rows(q, k, v, rows, off + rows[:, 2], "token", 1, 8, 2)
    for x, (bb, u, j) in enumerate(rows):
        for hh in range(g):
            np.testing.assert_allclose(got["o"][x, hh], o_ref[bb, u * g + hh, j], rtol=0,
                                       atol=1e-12)
            np.testing.assert_allclose(got["lse"][x, hh], lse_ref[bb, u * g + hh, j], rtol=0,
                                       atol=1e-12)


def test_rows_accept_torch_tensors():
    """The helpers take torch tensors (the GPU tests pass device tensors) as numpy."""
    b, hq, hkv, tq, T, d = 1, 4, 2, 15, 15, 8
    q, k, v = _inputs(b, hq, hkv, tq, T, d, seed=59)
    rows = _row_sample(b, hkv, tq, 8, seed=9)
    a = oracle.full_attn_rows(q, k, v, rows, rows[:, 2], "token", 1, 6, 2)
    t = oracle.full_attn_rows(torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
                              rows, rows[:, 2], "token", 1, 6, 2)
    assert np.array_equal(a["o"], t["o"]) and np.array_equal(a["idx"], t["idx"])


# ------------------------------------------------------ planted mistakes
ROW_PINS = [
    lambda: test_full_rows_equal_whole_array_oracle(CASES[1]),
    lambda: test_full_rows_equal_whole_array_oracle(CASES[2]),
    lambda: test_sparse_rows_equal_whole_array_oracle(CASES[0]),
    lambda: test_decode_rows_with_ragged_lengths_equal_whole_array_oracle(),
    lambda: test_full_rows_match_library_attention(),
]

PY_MUTANTS = {
    # head range of a unit shifted by one head
    "take_rows_head_range": ("q[b, h0:h1][:, js][None]", "q[b, h0 + 1:h1 + 1][:, js][None]"),
    # K/V prefix cut one key short of the latest row's position
    "prefix_cut_short": ("_f64_any(k[b, u, :tmax + 1][None, None])",
                         "_f64_any(k[b, u, :tmax][None, None])"),
    # rows' positions taken from the storage row, not the explicit position
    "rows_lose_positions": ("rows=[(0, 0, x) for x in range(len(ns))], q_pos=ts, want_scores=True",
                            "rows=[(0, 0, x) for x in range(len(ns))], q_pos=ts - 1, "
                            "want_scores=True"),
    # sparse helper's head range
    "sparse_take_rows_group": ("q1 = _take_rows(q, b, u * g, (u + 1) * g,",
                               "q1 = _take_rows(q, b, 0, g,"),
}

C_MUTANTS = {
    "q_pos_off_by_one": ("if (q_pos) return q_pos[n];", "if (q_pos) return q_pos[n] - 1;"),
    "q_pos_first_only": ("if (q_pos) return q_pos[n];", "if (q_pos) return q_pos[0];"),
}


def _caught():
    for pin in ROW_PINS:
        try:
            pin()
        except Exception:
            return True
    return False


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_row_pins_reject_python_mutant(name, tmp_path, monkeypatch):
    before, after = PY_MUTANTS[name]
    here = os.path.dirname(oracle.__file__)
    src = open(os.path.join(here, "__init__.py")).read()
    assert src.count(before) == 1, f"mutation site for {name} not unique"
    pkg = tmp_path / "oracle_mut"
    pkg.mkdir()
    (pkg / "__init__.py").write_text(src.replace(before, after))
    shutil.copy(os.path.join(here, "hs_oracle.c"), pkg / "hs_oracle.c")
    spec = importlib.util.spec_from_file_location("oracle_mut", pkg / "__init__.py")
    mod = importlib.util.module_from_spec(spec)
    monkeypatch.setitem(sys.modules, "oracle_mut", mod)  # dataclasses look the module up
    spec.loader.exec_module(mod)
    # route the row helpers of this module through the mutated copy
    monkeypatch.setattr(oracle, "full_attn_rows", mod.full_attn_rows)
    monkeypatch.setattr(oracle, "sparse_attn_rows", mod.sparse_attn_rows)
    assert _caught(), f"no pin rejects mutant {name}"


@pytest.mark.parametrize("name", sorted(C_MUTANTS))
def test_row_pins_reject_c_mutant(name, tmp_path):
    import subprocess
    before, after = C_MUTANTS[name]
    src = open(os.path.join(os.path.dirname(oracle.__file__), "hs_oracle.c")).read()
    assert src.count(before) == 1
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(before, after))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o",
                           str(lib), str(mutated), "-lm"])
    with oracle.use_library(str(lib)):
        assert _caught(), f"no pin rejects mutant {name}"
