"""Algorithmic work of the hot path: the FLOPs and bytes the method itself
requires, used as roofline numerators by the benchmark.

Formulas (titles of the pages the method is described on):
  * KV cache size M_full = 2 b T L h_kv d_h s and the HySparse cache
    2 b h_kv d_h s (F T + S w)          -- "HySparse 混合稀疏注意力（一）",
    "从“少算注意力”到“少存 KV”" and "为什么局部分支不能也复用同一份 KV";
  * prefill cost ratio F/L + (S/L)(k+w)/T and decode reads F T + S (k+w)
                                        -- same page, "成本模型";
  * block-score tensor size T x ceil(T/B) -- same page, "还有三笔容易漏掉的开销".
The full-attention FLOPs count QK^T and PV of every causal (query, key) pair:
4 d per pair and head.  The sparse layers' bytes count every K and V row the
index set makes a query read (the pages' "reads k+w tokens"), plus the
layer's own query, its outputs and the index rows.
"""
from __future__ import annotations

import math

MIB = 1 << 20


def kv_cache_bytes(b, T, L, hkv, d, s):
    """M_full = 2 b T L h_kv d s (K and V of L full-attention layers)."""
    return 2 * b * T * L * hkv * d * s


def hysparse_cache_bytes(b, hkv, d, s, F, S, T, w):
    """2 b h_kv d s (F T + S w): F full layers keep T tokens, S sparse layers a window."""
    return 2 * b * hkv * d * s * (F * T + S * w)


def prefill_cost_ratio(F, S, k, w, T):
    L = F + S
    return F / L + (S / L) * (k + w) / T


def decode_token_reads(F, S, T, k, w):
    """Token-KV pairs one decode step reads: F T + S (k + w)."""
    return F * T + S * (k + w)


def block_score_elements(T, B):
    return T * math.ceil(T / B)


def causal_pairs(t_q, q_offset=0):
    """Sum over query rows of visible keys: sum_{j < t_q} (q_offset + j + 1)."""
    return t_q * q_offset + t_q * (t_q + 1) // 2


def full_layer_flops(batch, hq, d, t_q, q_offset=0):
    """QK^T and PV of every causal pair: 4 d flops per (pair, head)."""
    return 4 * d * hq * batch * causal_pairs(t_q, q_offset)


def decode_full_bytes(batch, hkv, d, seq_lens, elt=2):
    """Full-layer decode step: the whole K and V cache of every sequence."""
    return sum(int(L) for L in seq_lens) * hkv * 2 * d * elt


def sparse_rows_from_index(idx, cnt, mode, block_size, q_offset=0):
    """Number of K/V rows the sparse layer reads, from an index set.

    idx [b, hkv, t_q, ksel] and cnt [b, hkv, t_q] (torch tensors).  Block mode
    counts each selected block's keys clipped to the row's position.
    """
    import torch
    if mode == "token":
        return int(cnt.sum().item())
    b, hkv, tq, ksel = idx.shape
    t = (torch.arange(tq, device=idx.device) + q_offset).view(1, 1, tq, 1)
    start = idx.long() * block_size
    n = (t - start + 1).clamp(min=0, max=block_size)
    valid = torch.arange(ksel, device=idx.device).view(1, 1, 1, ksel) < cnt.unsqueeze(-1)
    return int((n * valid).sum().item())


def window_rows(batch, hkv, t_q, w, q_offset=0):
    """Rows of the local window branch: sum_t min(w, t+1)."""
    tot = 0
    for j in range(t_q):
        tot += min(w, q_offset + j + 1)
    return batch * hkv * tot


def sparse_layer_bytes(kv_rows, batch, hq, t_q, d, elt, ksel, hkv, local_rows=0):
    """K+V rows gathered, plus q' read, o (and o_local) written, lse, index read."""
    kv = (kv_rows + local_rows) * 2 * d * elt
    q = batch * hq * t_q * d * elt
    outs = (2 if local_rows else 1) * batch * hq * t_q * (d * elt + 4)
    index = batch * hkv * t_q * (ksel + 1) * 4
    return kv + q + outs + index


def sparse_unique_rows_from_index(idx, cnt, mode, block_size, q_offset=0):
    """Distinct K/V rows the sparse layer's queries keep, summed over (batch,
    group) units: the least it must read from memory, however its queries
    share them.

    idx [b, hkv, t_q, ksel] and cnt [b, hkv, t_q] (torch tensors).  Token
    mode: the distinct token ids.  Block mode: the union of the kept keys, a
    selected block kept up to the latest position among the rows selecting it.
    """
    import torch
    b, hkv, tq, ksel = idx.shape
    valid = torch.arange(ksel, device=idx.device).view(1, 1, 1, ksel) < cnt.unsqueeze(-1)
    pos = (torch.arange(tq, device=idx.device) + q_offset).view(tq, 1).expand(tq, ksel)
    total = 0
    for bb in range(b):
        for u in range(hkv):
            m = valid[bb, u]
            ids = idx[bb, u][m].long()
            if ids.numel() == 0:
                continue
            if mode == "token":
                total += int(torch.unique(ids).numel())
                continue
            # latest position selecting each block, then its keys up to there
            last = torch.full((int(ids.max()) + 1,), -1, dtype=torch.long, device=idx.device)
            last.scatter_reduce_(0, ids, pos[m].long(), reduce="amax")
            blk = torch.arange(last.numel(), device=idx.device)
            keep = (last - blk * block_size + 1).clamp(min=0, max=block_size)
            total += int(keep[last >= 0].sum().item())
    return total


def sparse_layer_unique_bytes(unique_rows, batch, hq, t_q, d, elt, ksel, hkv, local_unique=0,
                              local=False):
    """Least memory traffic of a sparse layer: every distinct K/V row touched
    once, q' read, o (and o_local) and lse written, the index rows read."""
    kv = (unique_rows + local_unique) * 2 * d * elt
    q = batch * hq * t_q * d * elt
    outs = (2 if local else 1) * batch * hq * t_q * (d * elt + 4)
    index = batch * hkv * t_q * (ksel + 1) * 4
    return kv + q + outs + index
