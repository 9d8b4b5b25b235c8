"""ctypes front end of the CoSA CPU oracle (test infrastructure only).

Only tests/, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
import this package.  The product path (``block_sparse_attention_kap_b200``)
never imports, calls or links it.

Every function takes host torch tensors (bf16 inputs as produced by
``synth``) and returns host tensors.  Semantics: see cosa_oracle.c; each
step cites the CoSA technical summary (Sec. 2.1-2.3).  Beyond the C
library: ``block_union`` (CompactAttention's selection stage, Python sets),
``decode_kap`` / ``decode_osk`` (one decode step: the single-row reading of
Sec. 2.2/2.3), ``round_bf16`` (fp64 -> nearest bf16).  All are pinned in
tests/test_oracle_pins.py against hand-worked examples, independent
formulations (the C prefill proxy, torch SDPA, brute force) or properties.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

from . import build as _build

_LIB = None


class OrShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in
                ("B", "Hq", "Hkv", "Nq", "Nkv", "d", "bq", "bk", "s", "paged", "num_pages")]


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P, I, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        S = ctypes.POINTER(OrShape)
        L.oracle_kap.argtypes = [S, P, P, P, D, P, I, I, P, P, P, P, P, I]
        L.oracle_osk.argtypes = [S, P, P, P, P, P, I, P, P, I, D, P, P, P, P, I]
        L.oracle_dense.argtypes = [S, P, P, P, P, P, I, P, P, I, P, P, I]
        L.oracle_kmax.argtypes = [S, D]
        L.oracle_causal_blocks.argtypes = [S, I]
        L.oracle_budget_blocks.argtypes = [I, D]
        L.oracle_skip_threshold.argtypes = [D, I]
        L.oracle_skip_threshold.restype = ctypes.c_float
        L.oracle_pool.argtypes = [P, I, I, I, P]
        L.oracle_num_threads.restype = I
        _LIB = L
    return _LIB


def round_bf16(x: torch.Tensor) -> torch.Tensor:
    """Round fp64 values to the nearest bf16 value, ties to even, directly
    from fp64 (no intermediate fp32 rounding), returned as fp64.  The
    kernels store their fp32 outputs as bf16 with round-to-nearest-even, so
    this is the closest a bf16 output can be to the exact result."""
    x = x.double()
    m, e = torch.frexp(x)                       # x = m * 2^e, 0.5 <= |m| < 1
    # bf16 keeps 8 significant bits; below 2^-126 the spacing stays 2^-133
    step = torch.ldexp(torch.ones_like(x), torch.clamp(e - 8, min=-133))
    r = torch.round(x / step) * step            # torch.round: half to even
    return torch.where(torch.isfinite(x), r, x)


def block_union(wl, order: torch.Tensor, count: torch.Tensor):
    """Block union of CompactAttention's selection stage ("CompactAttention:
    Accelerating Chunked Prefill with Block-Union KV Selection", method): the
    KV block table of (batch b, kv-head g) is the set of blocks that any
    Q-block of any query head h with h // G == g selected, in ascending
    order.  order [B*Hq*nQB, kmax] and count [B*Hq*nQB] in (b, h, I)
    row-major order.  Returns (tables: list over (b, g) of sorted lists,
    per-row visible prefixes: list over (b, h, I) rows)."""
    B, Hq, Hkv, nqb, nkb = wl.B, wl.Hq, wl.Hkv, wl.n_qblocks, wl.n_kblocks
    G = Hq // Hkv
    order = order.view(B, Hq, nqb, -1)
    count = count.view(B, Hq, nqb)
    kmax_ = order.shape[-1]
    tables = []
    for b in range(B):
        for g in range(Hkv):
            chosen = set()
            for h in range(g * G, (g + 1) * G):
                for I in range(nqb):
                    c = min(max(int(count[b, h, I]), 0), kmax_)
                    for j in order[b, h, I, :c].tolist():
                        if 0 <= j < nkb:
                            chosen.add(j)
            tables.append(sorted(chosen))
    rows = []
    for b in range(B):
        for h in range(Hq):
            tab = tables[b * Hkv + h // G]
            for I in range(nqb):
                lim = lib().oracle_causal_blocks(ctypes.byref(shape_of(wl)), I)   # blocks 0..lim-1 visible
                rows.append([j for j in tab if j < lim])
    return tables, rows


def decode_kap(q: torch.Tensor, k: torch.Tensor, bk: int, stride: int, budget: float):
    """The Kernel-Aware Proxy for one decode step (CoSA technical summary
    Sec. 2.2 with a single query row; the pages leave decoding to future
    work, Sec. 4): the query of each head, at position Nkv-1, is not pooled
    (a row of one token); the keys are pooled as in prefill (mean of
    `stride` consecutive keys, bf16).  Scores S[c] = q . Kp[c] (all pooled
    keys are visible to the last position), MaxPool over each block's pooled
    keys, MaxNorm (minus the row max), HRM = first block holding the row max,
    order = (HRM desc, score desc, block asc), k = max(1, ceil(nKB * bp /
    1e4)).  Products are summed in fp64 and rounded to fp32 before every
    comparison, like the prefill steps.
    q [B, Hq, d] bf16; k logical [B, Hkv, Nkv, d] bf16 (Nkv a multiple of
    stride).  Returns dict(order [B*Hq, k] int32, count [B*Hq], hrm_count,
    score [B*Hq, nKB] fp32, hrm [B*Hq, nKB] uint8)."""
    B, Hq, d = q.shape
    Hkv, Nkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    nkb = -(-Nkv // bk)
    kpb = bk // stride
    kp = pool(k.reshape(B * Hkv * Nkv, d), stride).view(B, Hkv, Nkv // stride, d).double()
    sc = torch.einsum("bhd,bhcd->bhc", q.double(), kp.repeat_interleave(G, dim=1)).float()
    nkp = sc.shape[-1]
    pad = nkb * kpb - nkp
    bs = torch.nn.functional.pad(sc, (0, pad), value=float("-inf")).view(B, Hq, nkb, kpb).amax(-1)
    bs = bs.reshape(B * Hq, nkb)
    rowmax = bs.amax(-1, keepdim=True)
    jstar = torch.argmax((bs == rowmax).to(torch.int8), dim=-1)      # first block holding the max
    z = bs - rowmax                                                 # fp32 subtraction
    hrm = torch.zeros_like(bs, dtype=torch.uint8)
    hrm[torch.arange(B * Hq), jstar] = 1
    bp = int(round(budget * 10000))
    kk = max(1, min(nkb, -(-nkb * bp // 10000)))
    order = torch.empty(B * Hq, kk, dtype=torch.int32)
    for i in range(B * Hq):
        keys = sorted(range(nkb), key=lambda j: (-int(hrm[i, j]), -float(z[i, j]), j))
        order[i] = torch.tensor(keys[:kk], dtype=torch.int32)
    return dict(order=order, count=torch.full((B * Hq,), kk, dtype=torch.int32),
                hrm_count=hrm.sum(-1).to(torch.int32), score=z, hrm=hrm)


def decode_osk(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, order: torch.Tensor, count: torch.Tensor,
               bk: int, eps: float):
    """The Ordered-Skipping Kernel for one decode step: OSK (Sec. 2.3) with a
    single query row, so the tile-wide vote is that row's own test (no
    bucket effect).  It is oracle_osk on the shape Nq = 1, bq = 1 (stride 1:
    nothing is pooled here).  q [B, Hq, d]; k, v logical [B, Hkv, Nkv, d].
    Returns osk()'s dict with out [B*Hq, 1, d]."""
    B, Hq, d = q.shape
    Hkv, Nkv = k.shape[1], k.shape[2]
    sh = OrShape(B, Hq, Hkv, 1, Nkv, d, 1, bk, 1, 0, 0)
    n = B * Hq
    km = order.shape[1]
    out = torch.empty(n, 1, d, dtype=torch.float64)
    lse = torch.empty(n, 1, dtype=torch.float64)
    skipped = torch.empty(n, km, dtype=torch.uint8)
    margin = torch.empty(n, km, dtype=torch.float64)
    qq = q.contiguous().view(B, Hq, 1, d)
    rc = lib().oracle_osk(ctypes.byref(sh), _p(qq.view(torch.int16)), _p(k.contiguous().view(torch.int16)),
                          _p(v.contiguous().view(torch.int16)), None, None, 0, _p(order.contiguous()),
                          _p(count.contiguous()), km, eps, _p(out), _p(lse), _p(skipped), _p(margin), 0)
    if rc != 0:
        raise ValueError(f"oracle_osk failed ({rc})")
    return dict(out=out, lse=lse, skipped=skipped, margin=margin)


def shape_of(wl) -> OrShape:
    return OrShape(wl.B, wl.Hq, wl.Hkv, wl.Nq, wl.Nkv, wl.d, wl.bq, wl.bk, wl.stride,
                   1 if wl.paged else 0, wl.num_pages)


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    assert t.device.type == "cpu" and t.is_contiguous()
    return ctypes.c_void_p(t.data_ptr())


def _sel(sel: Optional[Sequence]) -> Optional[torch.Tensor]:
    if sel is None:
        return None
    return torch.tensor([list(x) for x in sel], dtype=torch.int32).reshape(-1, 3).contiguous()


def num_threads() -> int:
    return lib().oracle_num_threads()


def kmax(wl, budget: float) -> int:
    return lib().oracle_kmax(ctypes.byref(shape_of(wl)), budget)


def causal_blocks(wl, I: int) -> int:
    return lib().oracle_causal_blocks(ctypes.byref(shape_of(wl)), I)


def budget_blocks(n: int, budget: float) -> int:
    return lib().oracle_budget_blocks(n, budget)


def skip_threshold(eps: float, d: int) -> float:
    return lib().oracle_skip_threshold(eps, d)


def pool(x: torch.Tensor, s: int) -> torch.Tensor:
    """Pool a [rows, d] bf16 matrix with stride s (fp32 token-order sum, x 1/s, bf16 RNE)."""
    x = x.contiguous()
    rows, d = x.shape
    out = torch.empty(rows // s, d, dtype=torch.bfloat16)
    lib().oracle_pool(_p(x), rows, d, s, _p(out))
    return out


def kap(inp, budget: float, sel=None, kmax_: Optional[int] = None, want_scores: bool = False,
        threads: int = 0):
    """Stage 1 (KAP).  Returns dict(order [n,kmax] int32 padded -1, count [n],
    hrm_count [n], and optionally score [n,nKB] fp32, hrm [n,nKB] uint8).
    With sel=None, n = B*Hq*nQB in (b, h, I) row-major order."""
    wl = inp.wl
    sh = shape_of(wl)
    km = kmax_ if kmax_ is not None else kmax(wl, budget)
    selt = _sel(sel)
    n = selt.shape[0] if selt is not None else wl.B * wl.Hq * wl.n_qblocks
    order = torch.full((n, max(km, 1)), -1, dtype=torch.int32)
    count = torch.zeros(n, dtype=torch.int32)
    hrmc = torch.zeros(n, dtype=torch.int32)
    score = torch.empty(n, wl.n_kblocks, dtype=torch.float32) if want_scores else None
    hrm = torch.empty(n, wl.n_kblocks, dtype=torch.uint8) if want_scores else None
    rc = lib().oracle_kap(ctypes.byref(sh), _p(inp.q.view(torch.int16)), _p(inp.k.view(torch.int16)),
                          _p(inp.page_table), budget, _p(selt), n if selt is not None else 0,
                          max(km, 1), _p(order), _p(count), _p(hrmc), _p(score), _p(hrm), threads)
    if rc != 0:
        raise ValueError(f"oracle_kap failed ({rc})")
    out = dict(order=order, count=count, hrm_count=hrmc)
    if want_scores:
        out.update(score=score, hrm=hrm)
    return out


def osk(inp, order: torch.Tensor, count: torch.Tensor, eps: float, sel=None, threads: int = 0):
    """Stage 2 (OSK).  Returns dict(out [n,bq,d] fp64, lse [n,bq] fp64,
    skipped [n,kmax] uint8, margin [n,kmax] fp64: per visit the largest row
    value of fp32(m_loc - m_run) - T, negative iff the block was skipped)."""
    wl = inp.wl
    sh = shape_of(wl)
    order = order.to(torch.int32).contiguous()
    count = count.to(torch.int32).contiguous()
    selt = _sel(sel)
    n = order.shape[0]
    km = order.shape[1]
    out = torch.empty(n, wl.bq, wl.d, dtype=torch.float64)
    lse = torch.empty(n, wl.bq, dtype=torch.float64)
    skipped = torch.zeros(n, km, dtype=torch.uint8)
    margin = torch.empty(n, km, dtype=torch.float64)
    rc = lib().oracle_osk(ctypes.byref(sh), _p(inp.q.view(torch.int16)), _p(inp.k.view(torch.int16)),
                          _p(inp.v.view(torch.int16)), _p(inp.page_table), _p(selt),
                          n if selt is not None else 0, _p(order), _p(count), km, eps,
                          _p(out), _p(lse), _p(skipped), _p(margin), threads)
    if rc != 0:
        raise ValueError(f"oracle_osk failed ({rc})")
    return dict(out=out, lse=lse, skipped=skipped, margin=margin)


def dense(inp, sel=None, order: Optional[torch.Tensor] = None, count: Optional[torch.Tensor] = None,
          threads: int = 0):
    """Textbook causal attention (fp64), optionally restricted to the blocks
    listed in order/count.  Returns dict(out [n,bq,d], lse [n,bq])."""
    wl = inp.wl
    sh = shape_of(wl)
    selt = _sel(sel)
    n = selt.shape[0] if selt is not None else wl.B * wl.Hq * wl.n_qblocks
    km = 0
    if order is not None:
        order = order.to(torch.int32).contiguous()
        count = count.to(torch.int32).contiguous()
        km = order.shape[1]
    out = torch.empty(n, wl.bq, wl.d, dtype=torch.float64)
    lse = torch.empty(n, wl.bq, dtype=torch.float64)
    rc = lib().oracle_dense(ctypes.byref(sh), _p(inp.q.view(torch.int16)), _p(inp.k.view(torch.int16)),
                            _p(inp.v.view(torch.int16)), _p(inp.page_table), _p(selt),
                            n if selt is not None else 0, _p(order), _p(count), km,
                            _p(out), _p(lse), threads)
    if rc != 0:
        raise ValueError(f"oracle_dense failed ({rc})")
    return dict(out=out, lse=lse)


def rows_of(out: torch.Tensor, wl) -> torch.Tensor:
    """Reshape a full [B*Hq*nQB, bq, d] result into [B, Hq, Nq, d]."""
    B, Hq, nqb, bq, d = wl.B, wl.Hq, wl.n_qblocks, wl.bq, wl.d
    return out.view(B, Hq, nqb * bq, d)[:, :, : wl.Nq]
