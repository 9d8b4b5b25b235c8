"""Parity of the CUDA path (through the C ABI) against the CPU oracle.

Bar: M_KAP (order, count, HRM) and the in-kernel skip
decisions bit-exact on integer-grid inputs, where every pooled value and
logit is exact; outputs within max-abs 1e-2 of the exact result (plus one
bf16 half-ulp of the value, since |out| >= 4 has a bf16 spacing above 2e-2)
and mean-abs 1e-3 from the exact result rounded to bf16 (the outputs are
bf16; rounding alone costs ~ulp/4 on average).
On real-valued inputs the proxy's pooled scores come from tensor-core fp32
sums, so they are compared with a tolerance derived from fp32 accumulation
(SCORE_TOL), the GPU's sort is checked exactly against its own scores, and
skip decisions may differ only where the oracle's margin to the threshold
is within MARGIN_TOL.  Every expected value comes from oracle/; inputs from
synth/ (or the oracle's own orders when both sides must visit the same
blocks).
"""
import math
import random

import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

ATOL, RTOL, MEAN_TOL = 1e-2, 2.0 ** -8, 1e-3
SCORE_TOL = 2e-2        # |pooled score| <= ~600 here; 128-term fp32 sums err < 128 * 2^-24 * 600 per term
MARGIN_TOL = 0.05       # raw-logit units; fp32 tensor-core logits of |S| <= 400 err < 4e-3
EPS = 1e-4
LSE_TOL = 4e-3           # 2 * 2^-9: would cover a row sum over bf16-rounded weights; the kernel sums fp32 ones


@pytest.fixture(scope="module")
def cosa():
    import block_sparse_attention_kap_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def tiny(**kw):
    base = dict(name="t", wid=91, B=1, Hq=2, Hkv=1, Nq=1024, Nkv=1024, d=128, bq=128, bk=128,
                stride=16, structured=False)
    base.update(kw)
    return synth.Workload(**base)


def to_gpu(inp):
    pt = inp.page_table.cuda() if inp.page_table is not None else None
    return inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), pt


def gpu_plan(cosa, inp, budget, scores=True):
    m = cosa.CoSA(cosa.shape_of_workload(inp.wl))
    q, k, v, pt = to_gpu(inp)
    plan = m.plan(q, k, budget, page_table=pt, scores=scores)
    torch.cuda.synchronize()
    assert m.device_status() == 0
    return m, (q, k, v, pt), plan


def gpu_attend(m, dev, order, count, eps):
    q, k, v, pt = dev
    res = m.attend(q, k, v, order, count, eps, page_table=pt, lse=True, skip_bits=True)
    torch.cuda.synchronize()
    assert m.device_status() == 0
    return res


def flat(t):
    return t.reshape(-1, t.shape[-1]).cpu()


def check_out(gpu_rows, ref_rows, extra_atol=None, literal=False):
    """Max error against the exact (fp64) oracle output, allowing half a
    bf16 ulp of the value; mean error against the oracle output rounded to
    bf16 (nearest even), the closest any bf16 output can be -- on outputs of
    magnitude ~2 the rounding alone averages ~1.2e-3.
    literal=True applies the acceptance bar as written instead: max abs
    error <= 1e-2 and mean abs error <= 1e-3, both against the exact oracle
    output (used on the N(0,1) workloads, whose outputs stay below 4, where a
    bf16 value can always be within 1e-2 of the exact one)."""
    g = gpu_rows.double().cpu()
    r = ref_rows.double().cpu()
    err = (g - r).abs()
    if literal:
        assert r.abs().max().item() < 4.0, "an output of 4 or more cannot meet 1e-2 in bf16"
        tol = torch.full_like(r, ATOL)
    else:
        tol = ATOL + RTOL * r.abs()
    if extra_atol is not None:
        tol = tol + extra_atol
    assert bool((err <= tol).all()), f"max abs err {err.max().item():.4g}"
    mean_err = (g - (r if literal else oracle.round_bf16(r))).abs().mean().item()
    assert mean_err <= MEAN_TOL, f"mean abs err (vs {'exact' if literal else 'bf16-rounded'} oracle) {mean_err:.4g}"
    return err.max().item()


def gpu_rows(out, wl):
    """[B,Hq,Nq,d] -> [B*Hq*nQB, bq, d] zero-padded (the oracle's layout)."""
    B, Hq, nqb, bq, d = wl.B, wl.Hq, wl.n_qblocks, wl.bq, wl.d
    pad = nqb * bq - wl.Nq
    o = torch.nn.functional.pad(out.float().cpu(), (0, 0, 0, pad))
    return o.view(B * Hq * nqb, bq, d)


def valid_rows_mask(wl):
    nqb, bq = wl.n_qblocks, wl.bq
    r = torch.arange(nqb * bq).view(nqb, bq) < wl.Nq
    return r.repeat(wl.B * wl.Hq, 1)


GRID_SHAPES = [
    dict(Hq=2, Hkv=1, Nq=1024, Nkv=1024, bq=64, bk=64),
    dict(B=2, Hq=4, Hkv=2, Nq=1168, Nkv=1168, bq=128, bk=128),            # ragged last blocks
    dict(Hq=4, Hkv=1, Nq=384, Nkv=2304, bq=128, bk=64),                   # chunk after a cache, G=4
    dict(Hq=4, Hkv=2, Nq=512, Nkv=1536, bq=128, bk=64, paged=True),       # paged cache
]


def _make(shape, grid, structured=False):
    kw = dict(shape)
    paged = kw.pop("paged", False)
    wl = tiny(structured=structured, n_needle=2 if structured else 0, **kw)
    inp = synth.generate(wl, grid=grid)
    if paged:
        wl = wl.replace(paged=True)
        inp = synth._to_paged(wl, inp.q, inp.k, inp.v, wid=5)
    return inp


@pytest.mark.parametrize("shape", GRID_SHAPES)
@pytest.mark.parametrize("budget", [0.3, 1.0])
@pytest.mark.parametrize("structured", [False, True])
def test_grid_plan_bit_exact(cosa, shape, budget, structured):
    inp = _make(shape, grid=True, structured=structured)
    wl = inp.wl
    _, _, plan = gpu_plan(cosa, inp, budget)
    ref = oracle.kap(inp, budget, want_scores=True)
    km = ref["order"].shape[1]
    assert torch.equal(flat(plan["count"]).view(-1), ref["count"])
    assert torch.equal(flat(plan["order"])[:, :km], ref["order"])
    assert torch.equal(flat(plan["hrm_count"]).view(-1), ref["hrm_count"])
    assert torch.equal(flat(plan["block_score"]), ref["score"])
    assert torch.equal(flat(plan["hrm"]), ref["hrm"])


@pytest.mark.parametrize("shape", GRID_SHAPES)
@pytest.mark.parametrize("budget,eps", [(0.5, EPS), (1.0, EPS), (1.0, 0.0)])
def test_grid_attend_skip_bits_exact(cosa, shape, budget, eps):
    # structured grid: sink and needle logits ~200 above the rest, so blocks
    # really are skipped in-kernel (every decision >= 0.2 from the threshold)
    inp = _make(shape, grid=True, structured=True)
    wl = inp.wl
    m, dev, plan = gpu_plan(cosa, inp, budget, scores=False)
    ref_plan = oracle.kap(inp, budget)
    res = gpu_attend(m, dev, plan["order"], plan["count"], eps)
    ref = oracle.osk(inp, ref_plan["order"], ref_plan["count"], eps)
    km = ref_plan["order"].shape[1]
    bits = cosa.unpack_skip_bits(flat(res["skip_bits"]), km)
    assert torch.equal(bits, ref["skipped"])
    if eps == 0.0:
        assert bits.sum().item() == 0
    elif budget == 1.0:
        assert bits.sum().item() > 0          # the skip path is exercised
    check_out(gpu_rows(res["out"], wl), ref["out"])


@pytest.mark.parametrize("shape", GRID_SHAPES)
def test_dense_path_matches_oracle(cosa, shape):
    inp = _make(shape, grid=False)
    wl = inp.wl
    m = cosa.CoSA(cosa.shape_of_workload(wl))
    q, k, v, pt = to_gpu(inp)
    res = m.dense(q, k, v, page_table=pt, lse=True)
    torch.cuda.synchronize()
    ref = oracle.dense(inp)
    check_out(gpu_rows(res["out"], wl), ref["out"])
    lse_g = torch.nn.functional.pad(res["lse"].double().cpu(), (0, wl.n_qblocks * wl.bq - wl.Nq))
    lse_g = lse_g.view(-1, wl.bq)
    mask = valid_rows_mask(wl)
    # l sums bf16-rounded weights (relative error <= 2^-9 each), so ln(l) is
    # within ~2^-9 of the exact log-sum-exp
    assert (lse_g[mask] - ref["lse"][mask]).abs().max().item() < LSE_TOL


def test_single_head_2k_normal(cosa):
    """single_head_2k (B=1, H=1, N=2048, blocks 64): budget 25% with the skip
    threshold, and budget 100% with threshold 0, which must equal dense."""
    wl = synth.WORKLOADS["single_head_2k"]
    inp = synth.generate(wl)
    m, dev, plan = gpu_plan(cosa, inp, 0.25)
    ref = oracle.kap(inp, 0.25, want_scores=True)
    compare_plans(cosa, plan, ref, wl, 0.25)
    # OSK on the oracle's order on both sides
    order = ref["order"].view(wl.B, wl.Hq, wl.n_qblocks, -1).cuda()
    count = ref["count"].view(wl.B, wl.Hq, wl.n_qblocks).cuda()
    res = gpu_attend(m, dev, order, count, EPS)
    o = oracle.osk(inp, ref["order"], ref["count"], EPS)
    check_skips_and_out(cosa, res, o, wl, ref["order"].shape[1], literal=True)
    # budget 100%, threshold 0 == dense attention
    full = m.plan(dev[0], dev[1], 1.0)
    res = gpu_attend(m, dev, full["order"], full["count"], 0.0)
    check_out(gpu_rows(res["out"], wl), oracle.dense(inp)["out"], literal=True)


def compare_plans(cosa, plan, ref, wl, budget, sel_idx=None):
    """Scores within SCORE_TOL, HRM equal except at near-ties, the GPU sort
    exact for its own (HRM, score) keys, counts exact.  Returns the number of
    positions where the GPU and oracle orders differ."""
    go = flat(plan["order"])
    gc = flat(plan["count"]).view(-1)
    gs = flat(plan["block_score"])
    gh = flat(plan["hrm"])
    ghc = flat(plan["hrm_count"]).view(-1)
    if sel_idx is not None:
        go, gc, gs, gh, ghc = go[sel_idx], gc[sel_idx], gs[sel_idx], gh[sel_idx], ghc[sel_idx]
    assert torch.equal(gc, ref["count"])
    rs, rh = ref["score"], ref["hrm"]
    fin = torch.isfinite(rs)
    assert torch.equal(fin, torch.isfinite(gs))
    diff = (gs[fin].double() - rs[fin].double()).abs()
    assert diff.max().item() <= SCORE_TOL, f"score diff {diff.max().item()}"
    near0 = (rs >= -SCORE_TOL) & (gs >= -SCORE_TOL)
    assert bool(((gh == rh) | near0).all())
    assert torch.equal(ghc, gh.sum(1).to(torch.int32))
    mism = 0
    for i in range(gc.shape[0]):
        k = gc[i].item()
        n = int(fin[i].sum().item())
        keys = sorted(range(n), key=lambda j: (-int(gh[i, j]), -float(gs[i, j]), j))
        assert go[i, :k].tolist() == keys[:k]
        assert bool((go[i, k:] == -1).all())
        # a position where the two orders differ must hold a near-tie: the
        # oracle's scores of the two blocks there within twice the score
        # tolerance (HRM blocks score exactly 0, so an HRM near-tie counts)
        for a, b in zip(go[i, :k].tolist(), ref["order"][i, :k].tolist()):
            if a != b:
                mism += 1
                gap = abs(float(rs[i, a]) - float(rs[i, b]))
                assert gap <= 2 * SCORE_TOL, f"row {i}: blocks {a} / {b} differ by {gap:.4g} in the oracle's score"
    print(f"order positions that differ from the oracle's (all near-ties): {mism}")
    return mism


def check_skips_and_out(cosa, res, o, wl, km, sel_idx=None, eps=EPS, literal=False):
    """Skip bits equal the oracle's except where its margin (pinned against
    the definition in the oracle tests) is within MARGIN_TOL of 0, i.e. where
    fp32 tensor-core logits may fall on the other side of the threshold;
    outputs within tolerance, plus the derived allowance for each flip."""
    bits = cosa.unpack_skip_bits(flat(res["skip_bits"]), km)
    out = gpu_rows(res["out"], wl)
    if sel_idx is not None:
        bits, out = bits[sel_idx], out[sel_idx]
    diff = bits != o["skipped"]
    fragile = o["margin"].abs() <= MARGIN_TOL
    assert bool((~diff | fragile).all()), "a robust skip decision differs"
    # a flipped decision moves a row by at most 2*max|v|*bk*eps
    flips = diff.sum(1).double()
    vmax = 6.0
    extra = (2 * vmax * wl.bk * eps * flips).view(-1, 1, 1)
    n_flip = int(diff.sum())
    print(f"skip decisions that differ from the oracle's (all within the margin): {n_flip} "
          f"of {int(bits.numel())} entries; fragile visits {int(fragile.sum())}")
    if literal and n_flip == 0:
        extra = None
    return check_out(out, o["out"], extra_atol=extra, literal=literal), n_flip


def test_order_invariance_gpu(cosa):
    inp = _make(dict(Hq=2, Hkv=1, Nq=1024, Nkv=1024, bq=128, bk=128), grid=False)
    wl = inp.wl
    m, dev, plan = gpu_plan(cosa, inp, 0.6, scores=False)
    order = plan["order"].clone()
    count = plan["count"]
    g = torch.Generator().manual_seed(7)
    o2 = order.cpu().view(-1, order.shape[-1]).clone()
    for i, c in enumerate(count.cpu().view(-1).tolist()):
        o2[i, :c] = o2[i, :c][torch.randperm(c, generator=g)]
    a = gpu_attend(m, dev, order, count, 0.0)["out"].float()
    b = gpu_attend(m, dev, o2.view_as(order).cuda(), count, 0.0)["out"].float()
    assert (a - b).abs().max().item() < 2e-2
    assert (a - b).abs().mean().item() < 1e-3


def test_paged_equals_contiguous_gpu(cosa):
    flat_inp = _make(dict(Hq=4, Hkv=2, Nq=512, Nkv=1536, bq=128, bk=64), grid=False, structured=True)
    paged = synth._to_paged(flat_inp.wl.replace(paged=True), flat_inp.q, flat_inp.k, flat_inp.v, wid=9)
    m1, d1, p1 = gpu_plan(cosa, flat_inp, 0.2, scores=False)
    m2, d2, p2 = gpu_plan(cosa, paged, 0.2, scores=False)
    assert torch.equal(p1["order"], p2["order"]) and torch.equal(p1["count"], p2["count"])
    r1 = gpu_attend(m1, d1, p1["order"], p1["count"], EPS)
    r2 = gpu_attend(m2, d2, p2["order"], p2["count"], EPS)
    assert torch.equal(r1["out"], r2["out"]) and torch.equal(r1["skip_bits"], r2["skip_bits"])


def test_edge_cases(cosa):
    inp = _make(dict(Hq=2, Hkv=1, Nq=512, Nkv=512, bq=128, bk=128), grid=True)
    wl = inp.wl
    m, dev, plan = gpu_plan(cosa, inp, 1.0, scores=False)
    order = plan["order"].clone()
    count = plan["count"].clone()
    count[0, 0, 1] = 0                           # a Q-block that visits nothing
    order[0, 1, 3, 1] = -1                       # an invalid entry inside count: treated as skipped
    order[0, 1, 2, 0] = 10 ** 6
    res = gpu_attend(m, dev, order, count, 0.0)
    out = res["out"].float().cpu()
    assert out[0, 0, 128:256].abs().max().item() == 0.0
    assert bool(torch.isinf(res["lse"][0, 0, 128:256]).all())
    bits = cosa.unpack_skip_bits(res["skip_bits"].cpu(), order.shape[-1])
    assert bits[0, 1, 3, 1].item() == 1 and bits[0, 1, 2, 0].item() == 1
    # the oracle on the same orders with the invalid entries removed
    o_cpu, c_cpu = order.cpu().view(-1, order.shape[-1]).clone(), count.cpu().view(-1).clone()
    for i in range(o_cpu.shape[0]):
        keep = [j for j in o_cpu[i, : c_cpu[i]].tolist() if 0 <= j < wl.n_kblocks]
        o_cpu[i] = -1
        o_cpu[i, : len(keep)] = torch.tensor(keep, dtype=torch.int32)
        c_cpu[i] = len(keep)
    ref = oracle.osk(inp, o_cpu, c_cpu, 0.0)
    check_out(gpu_rows(res["out"], wl), ref["out"])
    # empty problem: no launch, status OK
    empty = cosa.make_shape(1, 2, 1, 0, 512, 128, 128, 128, 16)
    cosa.cosa_attend(empty, dev[0], dev[1], dev[2], None, order, count, order.shape[-1], 0.0, res["out"])


# ----------------------------------------------------------------- full-size workloads, sampled rows

def _samples(wl, n, seed):
    rng = random.Random(seed)
    picks = {(0, 0, wl.n_qblocks - 1), (wl.B - 1, wl.Hq - 1, 0), (0, wl.Hq // 2, wl.n_qblocks // 2)}
    while len(picks) < n:
        picks.add((rng.randrange(wl.B), rng.randrange(wl.Hq), rng.randrange(wl.n_qblocks)))
    return sorted(picks)


_FULL = {}


def _full_inputs(cosa, name, grid):
    """The workload's inputs on host and device, kept for the next case of
    the same workload (only one workload is held at a time)."""
    key = (name, grid)
    if key not in _FULL:
        _FULL.clear()
        torch.cuda.empty_cache()
        inp = synth.generate(synth.WORKLOADS[name], grid=grid)
        _FULL[key] = (inp, to_gpu(inp))
    return _FULL[key]


# every workload and budget of the benchmark plan, at its own full size: the
# 2K single head at 25%, the 32K layer at 10%, the 128K layer at 10% and 5%,
# the 4096-query chunk after a 128K paged cache at 10%, and the B=2 x 64K
# sweep at 100% (threshold 0: must equal dense attention), 50, 20, 10, 5, 2%
def check_plan_structure(cosa, m, plan, wl, budget):
    """Every row of a full-size plan, not only the sampled ones: a visit order
    cosa_attend may be given (cosa_check_order: causally visible blocks, none
    twice), of exactly k_I = max(1, ceil(n_I * budget)) blocks (the budget
    rule of cosa_kmax), padded with -1 past the count."""
    cosa.cosa_check_order(m.shape, plan["order"], plan["count"])
    nqb, nkb = wl.n_qblocks, cosa.cosa_num_kblocks(m.shape)
    last = torch.clamp((torch.arange(nqb) + 1) * wl.bq, max=wl.Nq) - 1
    n = torch.clamp((wl.Nkv - wl.Nq + last) // wl.bk + 1, max=nkb)
    bp = round(budget * 10000)
    k = torch.minimum(torch.clamp((n * bp + 9999) // 10000, min=1), n).to(torch.int32)
    cnt = plan["count"].cpu().view(-1, nqb)
    assert torch.equal(cnt, k.expand_as(cnt))
    km = plan["order"].shape[-1]
    o = plan["order"].cpu().view(-1, km)
    past = torch.arange(km).view(1, -1) >= cnt.reshape(-1, 1)
    assert bool((o[past] == -1).all())


def check_attend_bounds(res, dev):
    """Every row of a full-size attend: the output is a convex combination
    of V rows (|out| <= max |v| up to the bf16 rounding of P and of out) and
    finite, and the log-sum-exp is finite (every row sees at least one key
    of the blocks it visits, the diagonal one among them)."""
    out = res["out"].float()
    assert bool(torch.isfinite(out).all())
    assert float(out.abs().max()) <= float(dev[2].float().abs().max()) * (1 + 2.0 ** -7)
    assert bool(torch.isfinite(res["lse"]).all())


FULL_CASES = [("single_head_2k", 0.25, EPS), ("gqa_32k", 0.1, EPS), ("gqa_128k", 0.1, EPS), ("gqa_128k", 0.05, EPS),
              ("chunked_128k_paged", 0.1, EPS), ("sweep_64k_b2", 1.0, 0.0), ("sweep_64k_b2", 0.5, EPS),
              ("sweep_64k_b2", 0.2, EPS), ("sweep_64k_b2", 0.1, EPS), ("sweep_64k_b2", 0.05, EPS),
              ("sweep_64k_b2", 0.02, EPS)]


@pytest.mark.parametrize("name,budget,eps", FULL_CASES)
def test_full_size_sampled(cosa, name, budget, eps):
    """N(0,1)-based inputs at full size, in the launch configuration the
    benchmark times (one plan and one attend over the whole problem): on 12
    sampled (b, head, Q-block) rows the plan agrees with the oracle's (scores
    within SCORE_TOL, orders equal up to near-ties), skip bits equal except
    where the margin is within MARGIN_TOL, and outputs meet the acceptance
    bar as written (max abs <= 1e-2, mean abs <= 1e-3 against the exact
    oracle).  At budget 100% with threshold 0 the output is also compared
    with dense causal attention."""
    wl = synth.WORKLOADS[name]
    inp, dev = _full_inputs(cosa, name, False)
    m = cosa.CoSA(cosa.shape_of_workload(wl))
    plan = m.plan(dev[0], dev[1], budget, page_table=dev[3], scores=True)
    torch.cuda.synchronize()
    assert m.device_status() == 0
    check_plan_structure(cosa, m, plan, wl, budget)
    sel = _samples(wl, 12, 3)
    idx = [(b * wl.Hq + h) * wl.n_qblocks + I for b, h, I in sel]
    km = plan["order"].shape[-1]
    ref = oracle.kap(inp, budget, sel=sel, kmax_=km, want_scores=True)
    compare_plans(cosa, plan, ref, wl, budget, sel_idx=idx)
    # both sides visit the oracle's order on the sampled rows
    order = plan["order"].clone().view(-1, km)
    count = plan["count"].clone().view(-1)
    order[idx] = ref["order"].cuda()
    count[idx] = ref["count"].cuda()
    res = gpu_attend(m, dev, order.view_as(plan["order"]), count.view_as(plan["count"]), eps)
    check_attend_bounds(res, dev)
    o = oracle.osk(inp, ref["order"], ref["count"], eps, sel=sel)
    check_skips_and_out(cosa, res, o, wl, km, sel_idx=idx, eps=eps, literal=True)
    if budget == 1.0 and eps == 0.0:
        assert int(cosa.unpack_skip_bits(flat(res["skip_bits"]), km).sum()) == 0
        dense = oracle.dense(inp, sel=sel)
        check_out(gpu_rows(res["out"], wl)[idx], dense["out"], literal=True)


GRID_FULL_CASES = [("single_head_2k", 0.25), ("gqa_32k", 0.1), ("gqa_128k", 0.1), ("gqa_128k", 0.05),
                   ("chunked_128k_paged", 0.1), ("sweep_64k_b2", 1.0), ("sweep_64k_b2", 0.5),
                   ("sweep_64k_b2", 0.2), ("sweep_64k_b2", 0.1), ("sweep_64k_b2", 0.05), ("sweep_64k_b2", 0.02)]


@pytest.mark.parametrize("name,budget", GRID_FULL_CASES)
def test_full_size_grid_bit_exact(cosa, name, budget):
    """Each workload at its own full shape (GQA 32/8 at 32K, 128K and B=2 x
    64K, the paged 128K chunk, the 2K single head) on structured integer-grid
    inputs, where every pooled value and logit is exact: on sampled (b, head,
    Q-block) rows the GPU's order, count, HRM count, block scores and HRM
    flags equal the oracle's bit for bit, and so do the in-kernel skip bits
    of the attend over the GPU's own plan (eps 1e-4; at budget 100% also
    with eps 0, where nothing may be skipped)."""
    wl = synth.WORKLOADS[name]
    inp, dev = _full_inputs(cosa, name, True)
    m = cosa.CoSA(cosa.shape_of_workload(wl))
    plan = m.plan(dev[0], dev[1], budget, page_table=dev[3], scores=True)
    torch.cuda.synchronize()
    assert m.device_status() == 0
    check_plan_structure(cosa, m, plan, wl, budget)
    n_rows = wl.B * wl.Hq * wl.n_qblocks
    sel = _samples(wl, 12, 5) if n_rows > 64 else None
    idx = [(b * wl.Hq + h) * wl.n_qblocks + I for b, h, I in sel] if sel else list(range(n_rows))
    km = plan["order"].shape[-1]
    ref = oracle.kap(inp, budget, sel=sel, kmax_=km, want_scores=True)
    assert torch.equal(flat(plan["count"]).view(-1)[idx], ref["count"])
    assert torch.equal(flat(plan["order"])[idx], ref["order"])
    assert torch.equal(flat(plan["hrm_count"]).view(-1)[idx], ref["hrm_count"])
    assert torch.equal(flat(plan["block_score"])[idx], ref["score"])
    assert torch.equal(flat(plan["hrm"])[idx], ref["hrm"])
    for eps in ((EPS, 0.0) if budget == 1.0 else (EPS,)):
        res = gpu_attend(m, dev, plan["order"], plan["count"], eps)
        o = oracle.osk(inp, ref["order"], ref["count"], eps, sel=sel)
        bits = cosa.unpack_skip_bits(flat(res["skip_bits"]), km)[idx]
        assert torch.equal(bits, o["skipped"])
        if eps == 0.0:
            assert int(bits.sum()) == 0
        check_out(gpu_rows(res["out"], wl)[idx], o["out"])


def test_mass_recall_matches_oracle(cosa):
    """Attention-mass recall of M_KAP (fraction of each row's dense softmax
    mass inside the selected blocks) from the GPU's log-sum-exp outputs:
    exp(lse of OSK on the KAP order with eps 0 - lse of the dense path)."""
    wl = synth.WORKLOADS["gqa_32k"].replace(Nq=4096, Nkv=4096, Hq=4, Hkv=1, n_needle=4)
    inp = synth.generate(wl)
    ref_plan = oracle.kap(inp, 0.2)
    m, dev, _ = gpu_plan(cosa, inp, 0.2, scores=False)
    order = ref_plan["order"].view(wl.B, wl.Hq, wl.n_qblocks, -1).cuda()
    count = ref_plan["count"].view(wl.B, wl.Hq, wl.n_qblocks).cuda()
    sel = gpu_attend(m, dev, order, count, 0.0)
    dense = m.dense(*dev[:3], lse=True)
    torch.cuda.synchronize()
    rec_gpu = torch.exp(sel["lse"].double() - dense["lse"].double()).cpu().view(-1, wl.bq)
    rec_ref = torch.exp(oracle.dense(inp, order=ref_plan["order"], count=ref_plan["count"])["lse"] -
                        oracle.dense(inp)["lse"])
    # each lse is within LSE_TOL of the exact value, so the ratio within ~2*LSE_TOL relative
    assert torch.allclose(rec_gpu, rec_ref, rtol=2 * LSE_TOL, atol=0)


EDGE_SHAPES = [
    dict(Hq=2, Hkv=2, Nq=512, Nkv=512, bq=64, bk=128),                   # small Q-blocks, large KV blocks
    dict(Hq=2, Hkv=1, Nq=48, Nkv=48, bq=128, bk=128),                    # one partial Q-block and KV block
    dict(Hq=4, Hkv=4, Nq=80, Nkv=1040, bq=64, bk=64),                    # short chunk, ragged cache, G=1
    dict(B=2, Hq=4, Hkv=2, Nq=256, Nkv=1280, bq=128, bk=64, paged=True),  # two page tables in one pool
]


@pytest.mark.parametrize("shape", EDGE_SHAPES)
@pytest.mark.parametrize("budget,eps", [(0.01, EPS), (1.0, 0.5), (0.4, 0.999)])
def test_edge_shapes_bit_exact(cosa, shape, budget, eps):
    """Plans and skip decisions bit-exact on grids at the edges: one block per
    Q-block (1% budget), a threshold that skips nearly everything (eps near 1),
    partial blocks, G = 1, two batches sharing one page pool."""
    inp = _make(shape, grid=True, structured=True)
    wl = inp.wl
    m, dev, plan = gpu_plan(cosa, inp, budget)
    ref = oracle.kap(inp, budget, want_scores=True)
    km = ref["order"].shape[1]
    assert torch.equal(flat(plan["order"])[:, :km], ref["order"])
    assert torch.equal(flat(plan["count"]).view(-1), ref["count"])
    assert torch.equal(flat(plan["block_score"]), ref["score"])
    res = gpu_attend(m, dev, plan["order"], plan["count"], eps)
    o = oracle.osk(inp, ref["order"], ref["count"], eps)
    assert torch.equal(cosa.unpack_skip_bits(flat(res["skip_bits"]), km), o["skipped"])
    check_out(gpu_rows(res["out"], wl), o["out"])


def test_visit_list_longer_than_the_staged_order(cosa):
    """One Q-block visiting 1,280 KV blocks (64-key blocks of an 81,920-token
    cache): the kernel stages the first 1,024 order entries in shared memory
    and reads the rest from global memory; dense (eps 0) and eps > 0 both
    match the oracle, skip bits included (integer grid, structured)."""
    wl = tiny(Hq=1, Hkv=1, Nq=128, Nkv=81920, bq=128, bk=64, structured=True, n_needle=2)
    inp = synth.generate(wl, grid=True)
    m = cosa.CoSA(cosa.shape_of_workload(wl))
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    assert m.nkb == 1280
    g = torch.Generator().manual_seed(12)
    order = torch.randperm(m.nkb, generator=g).to(torch.int32).view(1, 1, 1, -1)
    count = torch.full((1, 1, 1), m.nkb, dtype=torch.int32)
    for eps in (0.0, EPS):
        res = m.attend(q, k, v, order.cuda(), count.cuda(), eps, lse=True, skip_bits=True)
        torch.cuda.synchronize()
        assert m.device_status() == 0
        o = oracle.osk(inp, order.view(1, -1), count.view(-1), eps)
        bits = cosa.unpack_skip_bits(flat(res["skip_bits"]), m.nkb)
        assert torch.equal(bits, o["skipped"])
        if eps > 0:
            assert int(bits[0, 1024:].sum()) > 0          # decisions past the staged part
        check_out(gpu_rows(res["out"], wl), o["out"])


STRIDE_SHAPES = [
    dict(Hq=2, Hkv=1, Nq=512, Nkv=1024, bq=128, bk=128, stride=4),      # 32 pooled rows per Q-block, 32 keys per block
    dict(Hq=2, Hkv=2, Nq=768, Nkv=768, bq=128, bk=64, stride=8),        # 16 rows per Q-block, 8 keys per block
    dict(Hq=4, Hkv=2, Nq=512, Nkv=1536, bq=64, bk=128, stride=32),      # 2 rows per Q-block, 4 keys per block
]


@pytest.mark.parametrize("shape", STRIDE_SHAPES)
def test_other_pooling_strides_bit_exact(cosa, shape):
    """Pooling strides other than 16 (every row-per-Q-block and key-per-block
    count the kernels instantiate): plans and skip bits bit-exact on
    structured grids, outputs within tolerance."""
    kw = dict(shape)
    stride = kw.pop("stride")
    wl = tiny(structured=True, n_needle=2, stride=stride, **kw)
    inp = synth.generate(wl, grid=True)
    m, dev, plan = gpu_plan(cosa, inp, 0.4)
    ref = oracle.kap(inp, 0.4, want_scores=True)
    km = ref["order"].shape[1]
    assert torch.equal(flat(plan["order"])[:, :km], ref["order"])
    assert torch.equal(flat(plan["count"]).view(-1), ref["count"])
    assert torch.equal(flat(plan["block_score"]), ref["score"])
    assert torch.equal(flat(plan["hrm"]), ref["hrm"])
    res = gpu_attend(m, dev, plan["order"], plan["count"], EPS)
    o = oracle.osk(inp, ref["order"], ref["count"], EPS)
    assert torch.equal(cosa.unpack_skip_bits(flat(res["skip_bits"]), km), o["skipped"])
    check_out(gpu_rows(res["out"], wl), o["out"])
