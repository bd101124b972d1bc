"""Seeded synthetic workloads for the HySparse / HySparse2 hot path.

This module only draws inputs: Gaussian Q/K/V of the shapes the pages use,
with a few keys planted as scaled copies of queries ("needles") so that the
oracle selection has sharp, checkable peaks.  It contains none of the method's
arithmetic and is the one module that both the oracle side and the CUDA side
take their inputs from.

Shapes follow the pages' model configurations ("HySparse 混合稀疏注意力（一）",
configuration table: 7B dense 32/8 heads, 80B-A3B MoE 64/4 heads, head dim
128, B=64, k=1024, w=128; "HySparse2 ..." 4.2: 128 forced + token top-k).

Every tensor is drawn from a torch.Generator seeded with
``1000 * config_id + stream`` (stream 0 = full layer, 1+l = sparse layer l,
100+l = the local K'/V' of sparse layer l), then rounded once to the
workload's dtype.  Needles: key i of kv group u becomes ``c * q[h, j]`` for a
query position j that sees i (j > i in prefill, the new token in decode) and a
uniform head h of the group.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    hq: int
    hkv: int
    head_dim: int
    t: int                 # prefill tokens, or decode cache length
    dtype: str             # "fp32" | "bf16"
    mode: str              # "block" (HySparse) | "token" (HySparse2)
    block_size: int
    k: int
    window: int
    n_sparse: int          # sparse layers per full layer
    swa_branch: bool       # HySparse sparse layers carry their own window K'/V'
    std: float             # Gaussian std of Q, K, V
    needle_scale: float    # c in k_i := c * q_{h,j}
    needles: str           # "count:N" | "frac:F" | "decode:N" | "loguniform:N"
    decode: bool = False
    t_q: int = 0           # query rows (0: = t);  chunked prefill uses fewer
    q_offset: int = 0
    config_id: int = 0
    page_size: int = 0     # > 0: the K^F/V^F cache is paged (decode workloads)
    extra: dict = field(default_factory=dict)

    @property
    def group(self) -> int:
        return self.hq // self.hkv

    @property
    def ksel(self) -> int:
        return self.k // self.block_size if self.mode == "block" else self.k

    @property
    def tq(self) -> int:
        return 1 if self.decode else (self.t_q or self.t)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16


_S128 = 1.0 / math.sqrt(128.0)

WORKLOADS = {
    # Tiny oracle case: 4 query heads on 1 kv head, d=64, fp32, 8 needles (x3).
    "tiny_block": Workload("tiny_block", 1, 4, 1, 64, 512, "fp32", "block", 16, 64, 32, 3,
                           True, 1.0, 3.0, "count:8", config_id=1),
    "tiny_token": Workload("tiny_token", 1, 4, 1, 64, 512, "fp32", "token", 1, 64, 32, 3,
                           False, 1.0, 3.0, "count:8", config_id=1),
    # HySparse 7B-dense-shaped block-level prefill, 1 full : 3 sparse (+ own window K'/V').
    "hysparse_7b_block": Workload("hysparse_7b_block", 2, 32, 8, 128, 16384, "bf16", "block",
                                  64, 1024, 128, 3, True, _S128, 8.0 / _S128, "frac:0.01",
                                  config_id=2),
    # HySparse2 token-level prefill, 80B-shaped heads 64/4, 1 full : 11 sparse.
    "hysparse2_prefill": Workload("hysparse2_prefill", 1, 64, 4, 128, 65536, "bf16", "token",
                                  1, 1024, 128, 11, False, _S128, 8.0 / _S128, "frac:0.01",
                                  config_id=3),
    # HySparse2 decode: 32 sequences with a 131072-token cache, 16 needles each.
    "hysparse2_decode": Workload("hysparse2_decode", 32, 64, 4, 128, 131072, "bf16", "token",
                                 1, 1024, 128, 11, False, _S128, 8.0 / _S128, "decode:16",
                                 decode=True, config_id=4),
    # 1M context: (a) one 8192-query chunk at the end of the 2^20 prefix.
    "long_1m_chunk": Workload("long_1m_chunk", 1, 64, 4, 128, 1 << 20, "bf16", "token", 1,
                              1024, 128, 11, False, _S128, 8.0 / _S128, "loguniform:64",
                              t_q=8192, q_offset=(1 << 20) - 8192, config_id=5),
    # 1M context: (b) decode steps at the end of the 2^20 cache.
    "long_1m_decode": Workload("long_1m_decode", 1, 64, 4, 128, 1 << 20, "bf16", "token", 1,
                               1024, 128, 11, False, _S128, 8.0 / _S128, "loguniform:64",
                               decode=True, config_id=5),
    # The HySparse2 decode case over a paged cache: 64-token pages, shuffled
    # block table ("HySparse 混合稀疏注意力（一）", 工程实现中的关键约束 item 2).
    "hysparse2_decode_paged": Workload("hysparse2_decode_paged", 32, 64, 4, 128, 131072, "bf16",
                                       "token", 1, 1024, 128, 11, False, _S128, 8.0 / _S128,
                                       "decode:16", decode=True, config_id=4, page_size=64),
    # HySparse2's MQA 64/1 at head dim 256 ("HySparse2 ...", 6.4): a prefill
    # and a decode case at reduced lengths (CUDA-core kernels).
    "mqa64_d256_prefill": Workload("mqa64_d256_prefill", 1, 64, 1, 256, 8192, "bf16", "token",
                                   1, 1024, 128, 11, False, 1.0 / 16.0, 8.0 * 16.0, "frac:0.01",
                                   config_id=6),
    "mqa64_d256_decode": Workload("mqa64_d256_decode", 8, 64, 1, 256, 32768, "bf16", "token", 1,
                                  1024, 128, 11, False, 1.0 / 16.0, 8.0 * 16.0, "decode:16",
                                  decode=True, config_id=7),
}


def scaled(w: Workload, **kw) -> Workload:
    """The same workload with some fields replaced (reduced-size replicas)."""
    return replace(w, **kw)


def _gen(w: Workload, stream: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(1000 * w.config_id + stream)
    return g


def _randn(shape, gen, std, dtype, device) -> torch.Tensor:
    x = torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def _plant(w: Workload, q: torch.Tensor, k: torch.Tensor, gen: torch.Generator) -> list:
    """Overwrite some keys with scaled copies of queries that can see them.

    Returns the list of (b, u, key_pos, head, query_row) plants.
    """
    kind, _, arg = w.needles.partition(":")
    T, tq, g = w.t, w.tq, w.group
    plants = []
    cpu = torch.Generator().manual_seed(int(torch.randint(0, 2**31 - 1, (1,), generator=gen,
                                                          device=gen.device).item()))
    for b in range(w.batch):
        for u in range(w.hkv):
            if kind == "frac" or kind == "count":
                n = int(round(float(arg) * T)) if kind == "frac" else int(arg)
                # key positions 0..T-2 (so a later query exists), later query j in (i, T)
                hi = min(T - 1, w.q_offset + tq - 1)
                pos = torch.randperm(hi, generator=cpu)[:n]
                for i in pos.tolist():
                    lo_j = max(i + 1, w.q_offset)
                    j_abs = int(torch.randint(lo_j, w.q_offset + tq, (1,), generator=cpu))
                    h = u * g + int(torch.randint(0, g, (1,), generator=cpu))
                    plants.append((b, u, i, h, j_abs - w.q_offset))
            elif kind == "decode":
                n = int(arg)
                pos = torch.randperm(T - 1, generator=cpu)[:n]
                for i in pos.tolist():
                    h = u * g + int(torch.randint(0, g, (1,), generator=cpu))
                    plants.append((b, u, i, h, 0))
            elif kind == "loguniform":
                n = int(arg)
                for _ in range(n):
                    j_row = int(torch.randint(0, tq, (1,), generator=cpu))
                    t_abs = (T - 1) if w.decode else (w.q_offset + j_row)
                    delta = int(math.floor(math.exp(float(torch.rand(1, generator=cpu)) *
                                                    math.log(max(t_abs, 2)))))
                    i = max(0, t_abs - max(delta, 1))
                    h = u * g + int(torch.randint(0, g, (1,), generator=cpu))
                    plants.append((b, u, i, h, 0 if w.decode else j_row))
            else:
                raise ValueError(w.needles)
    for (b, u, i, h, j) in plants:
        k[b, u, i] = (q[b, h, j].float() * w.needle_scale).to(k.dtype)
    return plants


def full_layer_inputs(w: Workload, device="cpu"):
    """Q [b,hq,tq,d], K^F and V^F [b,hkv,T,d] of the full-attention layer."""
    gen = _gen(w, 0, device)
    dt = w.torch_dtype
    q = _randn((w.batch, w.hq, w.tq, w.head_dim), gen, w.std, dt, device)
    k = _randn((w.batch, w.hkv, w.t, w.head_dim), gen, w.std, dt, device)
    v = _randn((w.batch, w.hkv, w.t, w.head_dim), gen, w.std, dt, device)
    plants = _plant(w, q, k, gen)
    return q, k, v, plants


def sparse_layer_query(w: Workload, layer: int, device="cpu") -> torch.Tensor:
    """The own query Q' [b,hq,tq,d] of sparse layer ``layer`` (0-based)."""
    gen = _gen(w, 1 + layer, device)
    return _randn((w.batch, w.hq, w.tq, w.head_dim), gen, w.std, w.torch_dtype, device)


def sparse_layer_local_kv(w: Workload, layer: int, device="cpu"):
    """The own window K', V' [b,hkv,T,d] of a HySparse sparse layer."""
    gen = _gen(w, 100 + layer, device)
    dt = w.torch_dtype
    k = _randn((w.batch, w.hkv, w.t, w.head_dim), gen, w.std, dt, device)
    v = _randn((w.batch, w.hkv, w.t, w.head_dim), gen, w.std, dt, device)
    return k, v


def decode_seq_lens(w: Workload, ragged: bool = False, device="cpu") -> torch.Tensor:
    """Per-sequence cache lengths (new token included).  Ragged: uniform in [T/2, T]."""
    if not ragged:
        return torch.full((w.batch,), w.t, dtype=torch.int32, device=device)
    gen = torch.Generator().manual_seed(1000 * w.config_id + 7)
    lens = torch.randint(w.t // 2, w.t + 1, (w.batch,), generator=gen, dtype=torch.int32)
    lens[0] = w.t
    return lens.to(device)


def paged_pool(k: torch.Tensor, v: torch.Tensor, page_size: int, seed: int = 0,
               extra_pages: int = 3):
    """Scatter contiguous K, V [b, hkv, T, d] into page pools.

    Pools are [n_pages, hkv, page_size, d]; the block table [b, ceil(T/ps)]
    int32 maps logical page i of sequence b to a physical page drawn from a
    seeded permutation, so consecutive logical pages land anywhere in the pool.
    Unused pages (extra_pages of them, and the tail of a last partial page)
    hold noise that a correct reader never sees.  Pure data movement.
    """
    b, hkv, T, d = k.shape
    mp = -(-T // page_size)
    n_pages = b * mp + extra_pages
    dev = k.device
    gen = torch.Generator().manual_seed(7919 + seed)
    perm = torch.randperm(n_pages, generator=gen)[: b * mp].view(b, mp)
    noise = torch.Generator(device=dev).manual_seed(104729 + seed)
    kp = (torch.randn(n_pages, hkv, page_size, d, generator=noise, device=dev) * 0.5).to(k.dtype)
    vp = (torch.randn(n_pages, hkv, page_size, d, generator=noise, device=dev) * 0.5).to(v.dtype)
    pad = mp * page_size - T
    for pool, src in ((kp, k), (vp, v)):
        x = torch.nn.functional.pad(src, (0, 0, 0, pad)) if pad else src
        # [b, hkv, mp, ps, d] -> one [hkv, ps, d] page per (b, logical page)
        pages = x.reshape(b, hkv, mp, page_size, d).permute(0, 2, 1, 3, 4).reshape(b * mp, hkv,
                                                                                 page_size, d)
        if pad:  # the tail of a last partial page keeps its noise
            keep = pool[perm[:, -1].to(dev)].clone()
            pool[perm.reshape(-1).to(dev)] = pages
            tail = pool[perm[:, -1].to(dev)]
            tail[:, :, page_size - pad:] = keep[:, :, page_size - pad:]
            pool[perm[:, -1].to(dev)] = tail
        else:
            pool[perm.reshape(-1).to(dev)] = pages
    return kp, vp, perm.to(torch.int32).to(dev)
