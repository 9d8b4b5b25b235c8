"""Chunked prefill with the pooled keys kept across chunks (cosa_plan_chunk)
against the oracle.

In chunked prefill ("CompactAttention: Accelerating Chunked Prefill with
Block-Union KV Selection", evaluation setup) chunk c of C queries attends to
the (c+1)*C keys cached so far.  cosa_plan_chunk pools only the keys no
earlier chunk pooled and reuses the rest from a caller-owned cache; the plan
of every chunk must still be the plan of that chunk's problem as the oracle
defines it from scratch (pooling of all its keys, Sec. 2.2 of the CoSA
technical summary).  Integer-grid inputs make every pooled value and logit
exact, so plans and skip decisions are compared bit for bit.
"""
import pytest
import torch

import oracle
import synth
from test_gpu_parity import (EPS, check_out, check_skips_and_out, compare_plans, flat, gpu_rows, tiny,
                             _samples)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cosa():
    import block_sparse_attention_kap_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


CHUNK_CASES = [
    dict(B=1, Hq=4, Hkv=2, C=256, n_chunks=4, bq=128, bk=64, paged=True),
    dict(B=2, Hq=4, Hkv=1, C=384, n_chunks=3, bq=128, bk=128, paged=False),
    dict(B=1, Hq=2, Hkv=1, C=208, n_chunks=3, bq=64, bk=64, paged=True),     # chunks end inside a page
]


def _chunk_inputs(inp_full, c, C):
    """The problem chunk c solves, in the oracle's contiguous layout."""
    wl = inp_full.wl
    k, v = synth.logical_kv(inp_full)
    nkv = (c + 1) * C
    wl_c = wl.replace(Nq=C, Nkv=nkv, paged=False)
    q = inp_full.q[:, :, c * C:(c + 1) * C].contiguous()
    return synth.Inputs(wl_c, q, k[:, :, :nkv].contiguous(), v[:, :, :nkv].contiguous())


def _pooled(k, s):
    """oracle.pool over the token axis of [B, H, N, d]."""
    B, H, N, d = k.shape
    return oracle.pool(k.reshape(B * H * N, d), s).view(B, H, N // s, d)


@pytest.mark.parametrize("case", CHUNK_CASES)
@pytest.mark.parametrize("budget", [0.3, 1.0])
def test_chunk_sequence_bit_exact(cosa, case, budget):
    case = dict(case)
    C, n_chunks, paged = case.pop("C"), case.pop("n_chunks"), case.pop("paged")
    total = C * n_chunks
    wl = tiny(Nq=total, Nkv=total, structured=True, n_needle=2, **case)
    inp = synth.generate(wl, grid=True)
    full = synth._to_paged(wl.replace(paged=True), inp.q, inp.k, inp.v, wid=11) if paged else inp
    kd = full.k.cuda()
    vd = full.v.cuda()
    pt = full.page_table.cuda() if paged else None
    cap = total // wl.stride
    cache = torch.zeros(wl.B, wl.Hkv, cap, wl.d, dtype=torch.bfloat16, device="cuda")
    skipped = 0
    for c in range(n_chunks):
        ci = _chunk_inputs(full, c, C)
        nkv = (c + 1) * C
        shape = cosa.make_shape(wl.B, wl.Hq, wl.Hkv, C, nkv, wl.d, wl.bq, wl.bk, wl.stride, paged,
                                full.page_table.numel() if paged else 0)
        m = cosa.CoSA(shape)
        q = ci.q.cuda()
        if paged:
            k_arg, v_arg = kd, vd
        else:
            k_arg, v_arg = ci.k.cuda(), ci.v.cuda()
        pt_c = pt[:, : m.nkb].contiguous() if paged else None
        before = cache[:, :, : c * C // wl.stride].clone()
        plan = m.plan_chunk(q, k_arg, budget, cache, c * C // wl.stride, page_table=pt_c, scores=True)
        torch.cuda.synchronize()
        assert m.device_status() == 0
        # rows pooled by earlier chunks are read, never rewritten
        assert torch.equal(cache[:, :, : c * C // wl.stride], before)
        ref = oracle.kap(ci, budget, want_scores=True)
        km = ref["order"].shape[1]
        assert torch.equal(flat(plan["order"])[:, :km], ref["order"])
        assert torch.equal(flat(plan["count"]).view(-1), ref["count"])
        assert torch.equal(flat(plan["block_score"]), ref["score"])
        assert torch.equal(flat(plan["hrm"]), ref["hrm"])
        res = m.attend(q, k_arg, v_arg, plan["order"], plan["count"], EPS, page_table=pt_c, lse=True,
                       skip_bits=True)
        torch.cuda.synchronize()
        assert m.device_status() == 0
        o = oracle.osk(ci, ref["order"], ref["count"], EPS)
        bits = cosa.unpack_skip_bits(flat(res["skip_bits"]), km)
        assert torch.equal(bits, o["skipped"])
        skipped += int(bits.sum())
        check_out(gpu_rows(res["out"], ci.wl), o["out"])
    # after the last chunk the cache holds every pooled key
    k_log, _ = synth.logical_kv(full)
    assert torch.equal(cache.cpu(), _pooled(k_log, wl.stride))
    if budget == 1.0:
        assert skipped > 0


def test_chunk_full_size_reuses_cache(cosa):
    """The 4096-query chunk after a 126976-token cache (64-token pages): the
    prefix rows come from the cache, the chunk's 256 pooled rows per head are
    pooled afresh (their cache rows are poisoned first), and the plan equals
    cosa_plan's bit for bit and the oracle's on sampled rows."""
    wl = synth.WORKLOADS["chunked_128k_paged"]
    inp = synth.generate(wl)
    shape = cosa.shape_of_workload(wl)
    m = cosa.CoSA(shape)
    q, k, v, pt = inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.page_table.cuda()
    budget = 0.1
    ref_plan = m.plan(q, k, budget, page_table=pt, scores=True)
    nkp = wl.Nkv // wl.stride
    valid = (wl.Nkv - wl.Nq) // wl.stride
    cache = torch.empty(wl.B, wl.Hkv, nkp, wl.d, dtype=torch.bfloat16, device="cuda")
    m.plan_chunk(q, k, budget, cache, 0, page_table=pt)           # fills every row
    torch.cuda.synchronize()
    cache[:, :, valid:] = float("inf")                             # must be re-pooled
    sentinel = cache[:, :, :valid].clone()
    plan = m.plan_chunk(q, k, budget, cache, valid, page_table=pt, scores=True)
    torch.cuda.synchronize()
    assert m.device_status() == 0
    assert torch.equal(cache[:, :, :valid], sentinel)
    assert bool(torch.isfinite(cache[:, :, valid:].float()).all())
    for key in ("order", "count", "hrm_count", "block_score", "hrm"):
        assert torch.equal(plan[key], ref_plan[key]), key
    sel = _samples(wl, 8, 5)
    idx = [(b * wl.Hq + h) * wl.n_qblocks + I for b, h, I in sel]
    km = plan["order"].shape[-1]
    ref = oracle.kap(inp, budget, sel=sel, kmax_=km, want_scores=True)
    compare_plans(cosa, plan, ref, wl, budget, sel_idx=idx)
    # the chunk's pooled rows against the oracle's pooling of the logical keys
    k_log, _ = synth.logical_kv(inp)
    heads = [0, wl.Hkv - 1]
    exp = _pooled(k_log[:, heads, wl.Nkv - wl.Nq:], wl.stride)
    assert torch.equal(cache[:, heads, valid:].cpu(), exp)
    # and the chunk's attention on that plan, sampled rows
    order = plan["order"].clone().view(-1, km)
    count = plan["count"].clone().view(-1)
    order[idx] = ref["order"].cuda()
    count[idx] = ref["count"].cuda()
    res = m.attend(q, k, v, order.view_as(plan["order"]), count.view_as(plan["count"]), EPS, page_table=pt,
                   lse=True, skip_bits=True)
    torch.cuda.synchronize()
    assert m.device_status() == 0
    o = oracle.osk(inp, ref["order"], ref["count"], EPS, sel=sel)
    check_skips_and_out(cosa, res, o, wl, km, sel_idx=idx)
