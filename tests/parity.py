"""Shared helpers of the GPU parity tests: run the C-ABI path and the fp64
oracle on the same seeded inputs and compare them under the stated bars.

Bars (written here once, used by every parity test):
  * index sets: identical, except candidates whose fp64 group score lies
    within 1e-3 relative of the k-th ranked score (near-ties);
  * attention outputs: max-abs error <= 1e-4 for fp32 inputs; for bf16,
    every element of a head's output vector at a query row is within
    1.5e-2 * RMS(that vector of the fp64 result) plus half a bf16 ulp of the
    fp64 value -- the bar applies to the computed value, and storing it as
    bf16 adds up to half an ulp that no bf16 output can avoid;
  * lse: |err| <= 1e-4 (fp32) / 2e-3 (bf16) -- the fp32 log-sum-exp of
    logits computed from the same (bf16-exact) inputs.
The sparse layers are checked on the GPU's own index set (the oracle
evaluates the sparse formula on exactly the rows the GPU selected).
"""
import numpy as np
import torch

import oracle
from oracle_top_kv_b200 import hs

INDEX_REL = 1e-3
O_TOL_FP32 = 1e-4
O_TOL_BF16_REL_RMS = 1.5e-2
LSE_TOL = {"fp32": 1e-4, "bf16": 2e-3}


def oracle_params(w, t_q=None, t_kv=None, q_offset=None):
    return oracle.Params(w.batch, w.hq, w.hkv, w.head_dim, w.tq if t_q is None else t_q,
                         w.t if t_kv is None else t_kv, mode=w.mode, block_size=w.block_size,
                         k=w.k, window=w.window,
                         q_offset=w.q_offset if q_offset is None else q_offset)


def abi_params(w, decode=False):
    return hs.make_params(w.batch, w.hq, w.hkv, w.head_dim, 1 if decode else w.tq, w.t,
                          0 if decode else w.q_offset, w.dtype, w.mode, w.block_size, w.k,
                          w.window)


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def half_ulp_bf16(x):
    """Half the spacing of bf16 numbers at |x| (8 significant bits)."""
    _, e = np.frexp(np.abs(x))
    return np.where(x == 0, 0.0, np.ldexp(1.0, e - 9))


def check_o(got, want, dtype, what):
    """got / want: [..., d] output vectors (one per query row and head)."""
    got = np.asarray(got, dtype=np.float64)
    if not got.size:
        return 0.0
    err = np.abs(got - want)
    if dtype == "fp32":
        e = err.max()
        assert e <= O_TOL_FP32, f"{what}: max-abs {e:.3e} > {O_TOL_FP32}"
        return e
    rms = np.sqrt(np.mean(want ** 2, axis=-1, keepdims=True))
    bound = O_TOL_BF16_REL_RMS * rms + half_ulp_bf16(want)
    # an exact match passes even where the bound is 0 (an all-zero output
    # vector: a row with an empty index set)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(err == 0, 0.0, err / bound)
    worst = np.unravel_index(np.argmax(ratio), ratio.shape)
    assert ratio.max() <= 1.0, (
        f"{what}: element {worst} err {err[worst]:.3e} > bound {bound[worst]:.3e} "
        f"(row rms {rms[worst[:-1]].item():.3e}, got {got[worst]:.5e}, want {want[worst]:.5e}); "
        f"{int((ratio > 1).sum())} of {ratio.size} elements out")
    with np.errstate(divide="ignore", invalid="ignore"):
        rel = np.where(err == 0, 0.0, err / rms)
    return float(rel.max())


def check_lse(got, want, dtype, what):
    got = np.asarray(got, dtype=np.float64)
    fin = np.isfinite(want)
    assert np.array_equal(np.isfinite(got), fin), f"{what}: -inf pattern differs"
    err = np.abs(got[fin] - want[fin]).max() if fin.any() else 0.0
    assert err <= LSE_TOL[dtype], f"{what}: lse max-abs {err:.3e}"


def check_index(g_idx, g_cnt, orc, mode, window, k, what):
    """g_idx [n, ksel], g_cnt [n]: GPU rows in the oracle's row order."""
    n_amb = 0
    for n in range(len(g_cnt)):
        oc = int(orc["cnt"][n])
        gc = int(g_cnt[n])
        assert gc == oc, f"{what} row {n}: count {gc} != {oc}"
        gi = g_idx[n]
        assert np.all(np.diff(gi[:gc]) > 0), f"{what} row {n}: not ascending"
        assert np.all(gi[gc:] == -1), f"{what} row {n}: padding"
        o_ids = set(orc["idx"][n, :oc].tolist())
        g_ids = set(gi[:gc].tolist())
        diff = o_ids ^ g_ids
        if not diff:
            continue
        sc = orc["scores"][n]
        ranked = sorted(o_ids)
        if mode == "token":
            t = int(orc["_t"][n])
            ranked = [i for i in ranked if i <= t - window]
        kth = min(sc[i] for i in ranked)
        for i in diff:
            assert abs(sc[i] - kth) <= INDEX_REL * kth, (
                f"{what} row {n}: id {i} (score {sc[i]:.6e}) differs, k-th {kth:.6e}")
        n_amb += 1
    return n_amb


def gpu_rows(arr, rows, per_head, g=None):
    """Gather GPU outputs at oracle rows (b, u, j).  per_head: arr is
    [b, hq, tq, ...] -> [n, g, ...]; else [b, hkv, tq, ...] -> [n, ...]."""
    b, u, j = rows[:, 0], rows[:, 1], rows[:, 2]
    if per_head:
        heads = u[:, None] * g + np.arange(g)[None, :]
        return arr[b[:, None], heads, j[:, None]]
    return arr[b, u, j]


def oracle_full_rows(w, q, k, v, rows, pos):
    return oracle.full_attn_rows(q, k, v, rows, pos, w.mode, w.block_size, w.k, w.window)


def oracle_sparse_rows(w, qs, kf, vf, idx_rows, cnt_rows, rows, pos, kl=None, vl=None):
    return oracle.sparse_attn_rows(qs, kf, vf, idx_rows, cnt_rows, rows, pos, w.mode,
                                   w.block_size, w.k, w.window, kl, vl)


def all_rows(w):
    b, u, j = np.meshgrid(np.arange(w.batch), np.arange(w.hkv), np.arange(w.tq), indexing="ij")
    return np.stack([b.ravel(), u.ravel(), j.ravel()], axis=1).astype(np.int32)
