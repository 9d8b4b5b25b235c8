"""Seeded synthetic workloads for CoSA block-sparse prefill attention.

This module only draws random inputs (host tensors, bf16) with the shapes and
structure of the long-context prefill workloads that the CoSA pages describe
(GQA 32/8 heads, d=128, contexts from 2K to 128K tokens, chunked prefill over a
paged KV cache).  It holds none of the method's arithmetic: no pooling, no
scores, no softmax.  Both the CPU oracle (``oracle/``) and the CUDA path
(``block_sparse_attention_kap_b200``) consume what it returns.

Recipe (every constant below is a choice made here; the pages give no
data distribution, they measure on RULER / LongBench-v2, which are not
available here, so these synthetic inputs stand in for their shapes only):

* ``z`` denotes i.i.d. N(0, 1) per element.
* ``u_h``: one unit direction per query head (a normalised N(0, I) draw);
  ``ubar_g``: the normalised mean of the ``u_h`` of the G query heads that
  share KV head ``g``.
* Q = z + Q_DIR * u_h.
* K = z + mu_{g,blk}, with one offset mu ~ N(0, MU_STD^2 I) per (kv-head,
  KV block of 128 tokens).
* sinks: tokens 0..3 get K += SINK_SCALE * sqrt(d) * ubar_g.
* needles: n_needle KV blocks per kv-head (uniform, never block 0) get
  K += NEEDLE_SCALE * sqrt(d) * ubar_g on every token of the block.
* local window (128K-context workloads only): Q and K both get, in dims
  0..15, 8 sinusoid pairs a*(cos 2 pi t / P_k, sin 2 pi t / P_k) with a=2 and
  P_k = 2048 * 2^(k/2); their product peaks at lag 0 and decays over a few
  blocks.
* V = z.
* recipe "planned" (``Workload.recipe``), a weaker structure drawn from the
  same noise: Q_DIR_PLANNED = 2 instead of 16, and needle blocks get
  K += NEEDLE_SCALE * ubar_g (no sqrt(d) factor); sinks as above.  Attention
  is then far less concentrated, and the in-kernel skip test fires less.
* the integer grid variant draws Q, K, V uniformly from {-2,...,2}; every
  pooled value and every logit is then exact in bf16 / fp32.  With structure
  on, a per-kv-head integer direction w_g in {-1, 0, 1}^d (nonzero on dims
  0..15) is added as Q += 4 w_g and, on the sink tokens and needle blocks,
  K += 4 w_g: values stay in {-6..6}, so pooled scores and logits stay exact,
  while sink and needle logits sit ~200 above the rest and in-kernel skips
  occur.

All values are rounded to bf16 with round-to-nearest-even (torch's
float32 -> bfloat16 conversion).  Seeds: 1000 * workload id + tensor id.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

Q_DIR = 16.0
Q_DIR_PLANNED = 2.0
MU_STD = 0.5
SINK_SCALE = 3.0
NEEDLE_SCALE = 3.0
N_SINK_TOKENS = 4
LOCAL_AMP = 2.0
LOCAL_PAIRS = 8

TENSOR_Q, TENSOR_K, TENSOR_V, TENSOR_DIR, TENSOR_MU, TENSOR_NEEDLE, TENSOR_PAGES = range(1, 8)


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and structure of one synthetic prefill-attention problem."""

    name: str
    wid: int                 # workload id (seeds = 1000 * wid + tensor id)
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nkv: int
    d: int = 128
    bq: int = 128
    bk: int = 128
    stride: int = 16
    paged: bool = False
    structured: bool = True  # sinks / needles / per-block offsets
    n_needle: int = 0
    local_window: bool = False
    budgets: tuple = (0.1,)
    eps: float = 1e-4
    recipe: str = "default"  # "default" or "planned" (weaker query direction and needles, see above)

    @property
    def n_qblocks(self) -> int:
        return -(-self.Nq // self.bq)

    @property
    def n_kblocks(self) -> int:
        return -(-self.Nkv // self.bk)

    @property
    def num_pages(self) -> int:
        return self.B * self.n_kblocks if self.paged else 0

    def dense_causal_flops(self) -> float:
        """4*B*Hq*d*(number of causal (query, key) pairs)."""
        off = self.Nkv - self.Nq
        pairs = self.Nq * off + self.Nq * (self.Nq + 1) // 2
        return 4.0 * self.B * self.Hq * self.d * pairs

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads of the benchmark plan, named by what they are.
WORKLOADS = {
    "single_head_2k": Workload("single_head_2k", 1, B=1, Hq=1, Hkv=1, Nq=2048, Nkv=2048,
                               bq=64, bk=64, structured=False, budgets=(0.25, 1.0)),
    "gqa_32k": Workload("gqa_32k", 2, B=1, Hq=32, Hkv=8, Nq=32768, Nkv=32768,
                        n_needle=8, budgets=(0.1,)),
    "gqa_128k": Workload("gqa_128k", 3, B=1, Hq=32, Hkv=8, Nq=131072, Nkv=131072,
                         n_needle=32, local_window=True, budgets=(0.05, 0.1)),
    "chunked_128k_paged": Workload("chunked_128k_paged", 4, B=1, Hq=32, Hkv=8, Nq=4096,
                                   Nkv=131072, bq=128, bk=64, paged=True, n_needle=32,
                                   local_window=True, budgets=(0.1,)),
    "sweep_64k_b2": Workload("sweep_64k_b2", 5, B=2, Hq=32, Hkv=8, Nq=65536, Nkv=65536,
                             n_needle=16, budgets=(1.0, 0.5, 0.2, 0.1, 0.05, 0.02)),
}


def _gen(wid: int, tid: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(1000 * wid + tid)
    return g


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True)


@dataclasses.dataclass
class Inputs:
    """Host tensors of one workload instance (bf16, contiguous).

    q: [B, Hq, Nq, d]; k, v: [B, Hkv, Nkv, d] when not paged, else the paged
    cache [num_pages, Hkv, bk, d] with ``page_table`` [B, n_kblocks] (int32)
    mapping logical KV block -> physical page.
    """

    wl: Workload
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    page_table: Optional[torch.Tensor] = None


def _local_window(n: int, t0: int, d: int) -> torch.Tensor:
    t = torch.arange(t0, t0 + n, dtype=torch.float64)
    cols = []
    for k in range(LOCAL_PAIRS):
        period = 2048.0 * 2.0 ** (k / 2.0)
        ang = 2.0 * math.pi * t / period
        cols += [LOCAL_AMP * torch.cos(ang), LOCAL_AMP * torch.sin(ang)]
    out = torch.zeros(n, d, dtype=torch.float32)
    out[:, : 2 * LOCAL_PAIRS] = torch.stack(cols, dim=1).float()
    return out


def generate(wl: Workload, grid: bool = False, rank: int = 0) -> Inputs:
    """Draw the inputs of ``wl`` (CPU, bf16).  ``rank`` shifts every seed, so
    replicas on several GPUs see different but equally distributed data."""
    wid = wl.wid + 100 * rank
    B, Hq, Hkv, Nq, Nkv, d = wl.B, wl.Hq, wl.Hkv, wl.Nq, wl.Nkv, wl.d
    G = Hq // Hkv
    if grid:
        q = torch.randint(-2, 3, (B, Hq, Nq, d), generator=_gen(wid, TENSOR_Q), dtype=torch.int8)
        k = torch.randint(-2, 3, (B, Hkv, Nkv, d), generator=_gen(wid, TENSOR_K), dtype=torch.int8)
        v = torch.randint(-2, 3, (B, Hkv, Nkv, d), generator=_gen(wid, TENSOR_V), dtype=torch.int8)
        if wl.structured:
            w = torch.randint(-1, 2, (B, Hkv, d), generator=_gen(wid, TENSOR_DIR), dtype=torch.int8)
            w[..., 16:] = 0
            q += 4 * w.repeat_interleave(G, dim=1)[:, :, None, :]
            k[:, :, :N_SINK_TOKENS] += 4 * w[:, :, None, :]
            nblk128 = -(-Nkv // 128)
            gn = _gen(wid, TENSOR_NEEDLE)
            for b in range(B):
                for g in range(Hkv):
                    if wl.n_needle > 0 and nblk128 > 1:
                        picks = torch.randperm(nblk128 - 1, generator=gn)[: wl.n_needle] + 1
                        for blk in picks.tolist():
                            k[b, g, blk * 128:(blk + 1) * 128] += 4 * w[b, g]
        q, k, v = q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)
    else:
        q = torch.empty(B, Hq, Nq, d, dtype=torch.bfloat16)
        k = torch.empty(B, Hkv, Nkv, d, dtype=torch.bfloat16)
        v = torch.empty(B, Hkv, Nkv, d, dtype=torch.bfloat16)
        gq, gk, gv = _gen(wid, TENSOR_Q), _gen(wid, TENSOR_K), _gen(wid, TENSOR_V)
        if wl.structured:
            u = _unit_rows(torch.randn(B, Hq, d, generator=_gen(wid, TENSOR_DIR)))
            ubar = _unit_rows(u.view(B, Hkv, G, d).mean(dim=2))
            nblk128 = -(-Nkv // 128)
            mu = MU_STD * torch.randn(B, Hkv, nblk128, d, generator=_gen(wid, TENSOR_MU))
            gn = _gen(wid, TENSOR_NEEDLE)
        loc_q = _local_window(Nq, Nkv - Nq, d) if (wl.structured and wl.local_window) else None
        loc_k = _local_window(Nkv, 0, d) if (wl.structured and wl.local_window) else None
        sq = math.sqrt(d)
        for b in range(B):
            for h in range(Hq):
                x = torch.randn(Nq, d, generator=gq)
                if wl.structured:
                    x += (Q_DIR_PLANNED if wl.recipe == "planned" else Q_DIR) * u[b, h]
                    if loc_q is not None:
                        x += loc_q
                q[b, h] = x.to(torch.bfloat16)
            for g in range(Hkv):
                x = torch.randn(Nkv, d, generator=gk)
                if wl.structured:
                    x += mu[b, g].repeat_interleave(128, dim=0)[:Nkv]
                    x[:N_SINK_TOKENS] += SINK_SCALE * sq * ubar[b, g]
                    n_blk = nblk128
                    if wl.n_needle > 0 and n_blk > 1:
                        picks = torch.randperm(n_blk - 1, generator=gn)[: wl.n_needle] + 1
                        for blk in picks.tolist():
                            x[blk * 128:(blk + 1) * 128] += \
                                NEEDLE_SCALE * (1.0 if wl.recipe == "planned" else sq) * ubar[b, g]
                    if loc_k is not None:
                        x += loc_k
                k[b, g] = x.to(torch.bfloat16)
                v[b, g] = torch.randn(Nkv, d, generator=gv).to(torch.bfloat16)
    if not wl.paged:
        return Inputs(wl, q.contiguous(), k.contiguous(), v.contiguous())
    return _to_paged(wl, q, k, v, wid)


def _to_paged(wl: Workload, q, k, v, wid: int) -> Inputs:
    """Scatter the logical KV sequence into a shuffled page pool.

    Physical page pt[b, p] holds logical tokens [p*bk, (p+1)*bk) of batch b for
    every kv-head (layout [num_pages, Hkv, bk, d]); the page table is a seeded
    permutation of all pages."""
    B, Hkv, Nkv, d, bk = wl.B, wl.Hkv, wl.Nkv, wl.d, wl.bk
    npg = -(-Nkv // bk)
    total = B * npg
    perm = torch.randperm(total, generator=_gen(wid, TENSOR_PAGES)).to(torch.int32)
    pt = perm.view(B, npg).contiguous()
    kc = torch.zeros(total, Hkv, bk, d, dtype=torch.bfloat16)
    vc = torch.zeros(total, Hkv, bk, d, dtype=torch.bfloat16)
    pad = npg * bk - Nkv
    kl = torch.nn.functional.pad(k, (0, 0, 0, pad)) if pad else k
    vl = torch.nn.functional.pad(v, (0, 0, 0, pad)) if pad else v
    for b in range(B):
        idx = pt[b].long()
        kc[idx] = kl[b].view(Hkv, npg, bk, d).permute(1, 0, 2, 3)
        vc[idx] = vl[b].view(Hkv, npg, bk, d).permute(1, 0, 2, 3)
    return Inputs(wl, q.contiguous(), kc.contiguous(), vc.contiguous(), pt)


def logical_kv(inp: Inputs):
    """Return (k, v) in the logical [B, Hkv, Nkv, d] layout (un-paging if needed)."""
    wl = inp.wl
    if not wl.paged:
        return inp.k, inp.v
    B, Hkv, Nkv, d, bk = wl.B, wl.Hkv, wl.Nkv, wl.d, wl.bk
    npg = inp.page_table.shape[1]
    ks, vs = [], []
    for b in range(B):
        idx = inp.page_table[b].long()
        ks.append(inp.k[idx].permute(1, 0, 2, 3).reshape(Hkv, npg * bk, d)[:, :Nkv])
        vs.append(inp.v[idx].permute(1, 0, 2, 3).reshape(Hkv, npg * bk, d)[:, :Nkv])
    return torch.stack(ks), torch.stack(vs)
