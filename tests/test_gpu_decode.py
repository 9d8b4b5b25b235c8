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
