"""One decode step (NEXT-4: the pages leave decoding to future work, CoSA
technical summary Sec. 4) against the oracle: the proxy with a single,
unpooled query row (cosa_decode_plan vs oracle.decode_kap) and the
Ordered-Skipping Kernel with that row (cosa_attend on Nq = 1 vs
oracle.decode_osk, where the tile-wide vote is the row's own test).
Integer-grid inputs make logits exact, so orders, scores and skip bits are
compared bit for bit; on real-valued inputs the comparison follows the
prefill tests' tolerances.
"""
import pytest
import torch

import oracle
import synth
from test_gpu_parity import EPS, MARGIN_TOL, SCORE_TOL, check_out, tiny

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cosa():
    import block_sparse_attention_kap_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def _decode_inputs(grid, paged, **kw):
    """The last query row of a prefill workload is a decode query at position
    Nkv-1; keys and values are that workload's cache."""
    wl = tiny(**kw)
    inp = synth.generate(wl, grid=grid)
    q = inp.q[:, :, -1, :].contiguous()                     # [B, Hq, d]
    k, v = inp.k, inp.v
    pt = None
    if paged:
        pinp = synth._to_paged(wl.replace(paged=True), inp.q, inp.k, inp.v, wid=13)
        k, v, pt = pinp.k, pinp.v, pinp.page_table
    return wl, q, inp.k, inp.v, k, v, pt


def _shape(cosa, wl, paged, num_pages):
    return cosa.make_shape(wl.B, wl.Hq, wl.Hkv, 1, wl.Nkv, wl.d, 128, wl.bk, wl.stride, paged, num_pages)


DECODE_SHAPES = [
    dict(B=2, Hq=4, Hkv=2, Nq=2048, Nkv=2048, bk=128),
    dict(B=1, Hq=8, Hkv=2, Nq=1024, Nkv=3072, bk=64),
    dict(B=1, Hq=4, Hkv=2, Nq=1040, Nkv=1040, bk=128),     # ragged cache: one pooled key in the last block
]


@pytest.mark.parametrize("shape", DECODE_SHAPES)
@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("budget", [0.1, 1.0])
def test_decode_step_bit_exact_on_grid(cosa, shape, paged, budget):
    wl, q, k_log, v_log, k, v, pt = _decode_inputs(True, paged, structured=True, n_needle=2, **shape)
    s = _shape(cosa, wl, paged, pt.numel() if paged else 0)
    m = cosa.CoSA(s)
    nkp = wl.Nkv // wl.stride
    cache = torch.zeros(wl.B, wl.Hkv, nkp, wl.d, dtype=torch.bfloat16, device="cuda")
    qd = q.view(wl.B, wl.Hq, 1, wl.d).cuda()
    kd, vd = k.cuda(), v.cuda()
    ptd = pt.cuda() if paged else None
    # the first half of the pooled keys come from a cache filled beforehand
    half = nkp // 2
    m.decode_plan(qd, kd, budget, cache, 0, page_table=ptd)
    torch.cuda.synchronize()
    cache[:, :, half:] = 0
    plan = m.decode_plan(qd, kd, budget, cache, half, page_table=ptd, scores=True)
    torch.cuda.synchronize()
    ref = oracle.decode_kap(q, k_log, wl.bk, wl.stride, budget)
    km = ref["order"].shape[1]
    assert torch.equal(plan["order"].view(-1, plan["order"].shape[-1]).cpu()[:, :km], ref["order"])
    assert torch.equal(plan["count"].view(-1).cpu(), ref["count"])
    assert torch.equal(plan["hrm_count"].view(-1).cpu(), ref["hrm_count"])
    assert torch.equal(plan["block_score"].view(-1, m.nkb).cpu(), ref["score"])
    assert torch.equal(plan["hrm"].view(-1, m.nkb).cpu(), ref["hrm"])
    # the step's attention: cosa_attend with one query row
    for eps in (0.0, EPS, 0.05):
        res = m.attend(qd, kd, vd, plan["order"], plan["count"], eps, page_table=ptd, lse=True, skip_bits=True)
        torch.cuda.synchronize()
        assert m.device_status() == 0
        o = oracle.decode_osk(q, k_log, v_log, ref["order"], ref["count"], wl.bk, eps)
        bits = cosa.unpack_skip_bits(res["skip_bits"].view(-1, res["skip_bits"].shape[-1]).cpu(), km)
        assert torch.equal(bits, o["skipped"])
        if eps == 0.0:
            assert int(bits.sum()) == 0
        check_out(res["out"].view(-1, 1, wl.d).float(), o["out"])


def test_decode_step_skips_on_grid(cosa):
    """The single-row test does skip on structured grids at full budget."""
    shape = DECODE_SHAPES[0]
    wl, q, k_log, v_log, k, v, _ = _decode_inputs(True, False, structured=True, n_needle=2, **shape)
    ref = oracle.decode_kap(q, k_log, wl.bk, wl.stride, 1.0)
    o = oracle.decode_osk(q, k_log, v_log, ref["order"], ref["count"], wl.bk, EPS)
    assert int(o["skipped"].sum()) > 0


def test_decode_step_full_size_sampled(cosa):
    """B=2 decode queries after a 128K-token cache (GQA 32/8, blocks of 128,
    budget 10%): scores within SCORE_TOL of the oracle, the GPU order exact
    for its own scores, and the attention over the oracle's order on sampled
    heads within tolerance (skip decisions may differ only at fragile
    margins)."""
    wl = synth.WORKLOADS["gqa_128k"].replace(B=1, Nq=4096, n_needle=8)
    inp = synth.generate(wl)
    q = inp.q[:, :, -1, :].contiguous()
    s = _shape(cosa, wl, False, 0)
    m = cosa.CoSA(s)
    cache = torch.empty(wl.B, wl.Hkv, wl.Nkv // wl.stride, wl.d, dtype=torch.bfloat16, device="cuda")
    qd = q.view(wl.B, wl.Hq, 1, wl.d).cuda()
    kd, vd = inp.k.cuda(), inp.v.cuda()
    budget = 0.1
    plan = m.decode_plan(qd, kd, budget, cache, 0, scores=True)
    torch.cuda.synchronize()
    ref = oracle.decode_kap(q, inp.k, wl.bk, wl.stride, budget)
    gs = plan["block_score"].view(-1, m.nkb).cpu()
    fin = torch.isfinite(ref["score"])
    assert torch.equal(fin, torch.isfinite(gs))
    assert (gs[fin].double() - ref["score"][fin].double()).abs().max().item() <= SCORE_TOL
    go = plan["order"].view(wl.B * wl.Hq, -1).cpu()
    gh = plan["hrm"].view(-1, m.nkb).cpu()
    kk = int(ref["count"][0])
    for i in range(wl.B * wl.Hq):
        keys = sorted(range(m.nkb), key=lambda j: (-int(gh[i, j]), -float(gs[i, j]), j))
        assert go[i, :kk].tolist() == keys[:kk]
    # attention on the oracle's order, all heads
    order = ref["order"].view(wl.B, wl.Hq, 1, -1).cuda()
    count = ref["count"].view(wl.B, wl.Hq, 1).cuda()
    res = m.attend(qd, kd, vd, order, count, EPS, lse=True, skip_bits=True)
    torch.cuda.synchronize()
    assert m.device_status() == 0
    o = oracle.decode_osk(q, inp.k, inp.v, ref["order"], ref["count"], wl.bk, EPS)
    bits = cosa.unpack_skip_bits(res["skip_bits"].view(wl.B * wl.Hq, -1).cpu(), kk)
    diff = bits != o["skipped"]
    assert bool((~diff | (o["margin"].abs() <= MARGIN_TOL)).all())
    flips = diff.sum(1).double()
    check_out(res["out"].view(-1, 1, wl.d).float(), o["out"], extra_atol=(2 * 6.0 * wl.bk * EPS * flips).view(-1, 1, 1))


# ----------------------------------------------------------------- the decode-step attention kernels

@pytest.mark.parametrize("shape", DECODE_SHAPES)
@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("budget", [0.1, 1.0])
def test_decode_attend_bit_exact_on_grid(cosa, shape, paged, budget):
    """cosa_decode_attend (parallel logits, prefix-max decisions, parallel
    P.V) on integer grids: skip bits bit-exact against the oracle and equal
    to cosa_attend's on the same one-row shape, outputs and lse within
    tolerance, at eps 0, 1e-4 and 0.05."""
    wl, q, k_log, v_log, k, v, pt = _decode_inputs(True, paged, structured=True, n_needle=2, **shape)
    s = _shape(cosa, wl, paged, pt.numel() if paged else 0)
    m = cosa.CoSA(s)
    cache = torch.zeros(wl.B, wl.Hkv, wl.Nkv // wl.stride, wl.d, dtype=torch.bfloat16, device="cuda")
    qd = q.view(wl.B, wl.Hq, 1, wl.d).cuda()
    kd, vd = k.cuda(), v.cuda()
    ptd = pt.cuda() if paged else None
    plan = m.decode_plan(qd, kd, budget, cache, 0, page_table=ptd)
    ref = oracle.decode_kap(q, k_log, wl.bk, wl.stride, budget)
    km = ref["order"].shape[1]
    for eps in (0.0, EPS, 0.05):
        res = m.decode_attend(qd, kd, vd, plan["order"], plan["count"], eps, page_table=ptd, lse=True,
                              skip_bits=True)
        att = m.attend(qd, kd, vd, plan["order"], plan["count"], eps, page_table=ptd, lse=True, skip_bits=True)
        torch.cuda.synchronize()
        assert m.device_status() == 0
        o = oracle.decode_osk(q, k_log, v_log, ref["order"], ref["count"], wl.bk, eps)
        bits = cosa.unpack_skip_bits(res["skip_bits"].view(wl.B * wl.Hq, -1).cpu(), km)
        assert torch.equal(bits, o["skipped"])
        assert torch.equal(bits, cosa.unpack_skip_bits(att["skip_bits"].view(wl.B * wl.Hq, -1).cpu(), km))
        if eps == 0.0:
            assert int(bits.sum()) == 0
        check_out(res["out"].view(-1, 1, wl.d).float(), o["out"])
        assert (res["lse"].view(-1).double().cpu() - o["lse"].view(-1)).abs().max().item() < 1e-3


def test_decode_attend_invalid_entries_and_empty_rows(cosa):
    """Entries that are not blocks count as skipped visits; a row whose
    visits are all such entries, or that has none, outputs 0 with lse -inf."""
    wl, q, k_log, v_log, k, v, _ = _decode_inputs(True, False, structured=True, n_needle=2, **DECODE_SHAPES[0])
    s = _shape(cosa, wl, False, 0)
    m = cosa.CoSA(s)
    nkb = m.nkb
    order = torch.full((wl.B, wl.Hq, 1, 6), -1, dtype=torch.int32)
    count = torch.tensor([[4, 3, 0, 2], [5, 1, 2, 6]], dtype=torch.int32).view(wl.B, wl.Hq, 1)
    rows = [[0, -1, 3, nkb + 2], [nkb, -5, 7], [], [9, 2], [1, 2, 3, 4, 5], [nkb + 1], [0, 15], [4, 3, 2, 1, 0, 11]]
    for i, r in enumerate(rows):
        order.view(-1, 6)[i, :len(r)] = torch.tensor(r, dtype=torch.int32)
    qd, kd, vd = q.view(wl.B, wl.Hq, 1, wl.d).cuda(), k.cuda(), v.cuda()
    res = m.decode_attend(qd, kd, vd, order.cuda(), count.cuda(), EPS, lse=True, skip_bits=True)
    torch.cuda.synchronize()
    bits = cosa.unpack_skip_bits(res["skip_bits"].view(wl.B * wl.Hq, -1).cpu(), 6)
    out = res["out"].view(-1, wl.d).float().cpu()
    lse = res["lse"].view(-1).cpu()
    for i, r in enumerate(rows):
        valid = [j for j in r if 0 <= j < nkb]
        for t, j in enumerate(r):
            if not 0 <= j < nkb:
                assert bits[i, t] == 1
        if not valid:
            assert out[i].abs().max().item() == 0.0 and lse[i].item() == float("-inf")
            continue
        o = oracle.decode_osk(q.view(-1, wl.d)[i].view(1, 1, wl.d), k_log[i // wl.Hq:i // wl.Hq + 1, (i % wl.Hq) // 2:(i % wl.Hq) // 2 + 1].contiguous(),
                              v_log[i // wl.Hq:i // wl.Hq + 1, (i % wl.Hq) // 2:(i % wl.Hq) // 2 + 1].contiguous(),
                              torch.tensor([valid], dtype=torch.int32), torch.tensor([len(valid)], dtype=torch.int32),
                              wl.bk, EPS)
        check_out(out[i].view(1, 1, wl.d), o["out"])


@pytest.mark.parametrize("bk,Nkv", [(64, 1040), (128, 1168), (64, 1101)])
def test_decode_attend_nan_in_ragged_page_tail(cosa, bk, Nkv):
    """The rows of the last page past the end of the cache hold NaN and Inf;
    the decode step must neither read them into a logit nor into P.V."""
    stride = 16 if Nkv % 16 == 0 else 1
    wl = tiny(B=1, Hq=4, Hkv=2, Nq=Nkv, Nkv=Nkv, bk=bk, stride=stride, structured=True, n_needle=2)
    inp = synth.generate(wl, grid=True)
    q = inp.q[:, :, -1, :].contiguous()
    pinp = synth._to_paged(wl.replace(paged=True), inp.q, inp.k, inp.v, wid=17)
    kp, vp = pinp.k.clone(), pinp.v.clone()
    tail = Nkv % bk
    last = int(pinp.page_table[0, -1])
    kp[last, :, tail:] = float("nan")
    vp[last, :, tail:] = float("inf")
    s = _shape(cosa, wl, True, pinp.page_table.numel())
    m = cosa.CoSA(s)
    order, count = m.dense_order()
    qd = q.view(wl.B, wl.Hq, 1, wl.d).cuda()
    for eps in (0.0, EPS):
        res = m.decode_attend(qd, kp.cuda(), vp.cuda(), order, count, eps, page_table=pinp.page_table.cuda(),
                              lse=True, skip_bits=True)
        torch.cuda.synchronize()
        assert bool(torch.isfinite(res["out"].float()).all()) and bool(torch.isfinite(res["lse"]).all())
        km = order.shape[-1]
        o = oracle.decode_osk(q, inp.k, inp.v, order.view(-1, km).cpu(), count.view(-1).cpu(), bk, eps)
        assert torch.equal(cosa.unpack_skip_bits(res["skip_bits"].view(wl.B * wl.Hq, -1).cpu(), km), o["skipped"])
        check_out(res["out"].view(-1, 1, wl.d).float(), o["out"])


def test_decode_attend_full_size(cosa):
    """Decode queries after the 131,072-token cache of the 128K layer (GQA
    32/8, blocks of 128, budget 10%, eps 1e-4), on the oracle's order: skip
    decisions equal the oracle's except at fragile margins, outputs meet the
    acceptance bar as written; and the dense step (every block, eps 0)
    equals the oracle's dense attention of the row."""
    wl = synth.WORKLOADS["gqa_128k"].replace(Nq=4096)     # the cache is the full one; 4096 queries drawn
    inp = synth.generate(wl)
    q = inp.q[:, :, -1, :].contiguous()
    s = _shape(cosa, wl, False, 0)
    m = cosa.CoSA(s)
    qd = q.view(wl.B, wl.Hq, 1, wl.d).cuda()
    kd, vd = inp.k.cuda(), inp.v.cuda()
    ref = oracle.decode_kap(q, inp.k, wl.bk, wl.stride, 0.1)
    kk = ref["order"].shape[1]
    order = ref["order"].view(wl.B, wl.Hq, 1, -1).cuda()
    count = ref["count"].view(wl.B, wl.Hq, 1).cuda()
    res = m.decode_attend(qd, kd, vd, order, count, EPS, lse=True, skip_bits=True)
    torch.cuda.synchronize()
    o = oracle.decode_osk(q, inp.k, inp.v, ref["order"], ref["count"], wl.bk, EPS)
    bits = cosa.unpack_skip_bits(res["skip_bits"].view(wl.B * wl.Hq, -1).cpu(), kk)
    diff = bits != o["skipped"]
    assert bool((~diff | (o["margin"].abs() <= MARGIN_TOL)).all())
    assert int(bits.sum()) > 0
    extra = None if int(diff.sum()) == 0 else (2 * 6.0 * wl.bk * EPS * diff.sum(1).double()).view(-1, 1, 1)
    check_out(res["out"].view(-1, 1, wl.d).float(), o["out"], extra_atol=extra, literal=extra is None)
    d_order, d_count = m.dense_order()
    dres = m.decode_attend(qd, kd, vd, d_order, d_count, 0.0)
    torch.cuda.synchronize()
    dense = oracle.decode_osk(q, inp.k, inp.v, d_order.view(wl.B * wl.Hq, -1).cpu(), d_count.view(-1).cpu(), wl.bk,
                              0.0)
    check_out(dres["out"].view(-1, 1, wl.d).float(), dense["out"], literal=True)
