"""The group form of OSK (cosa_attend_group): one visit order per (batch,
kv-head, Q-block), shared by the query heads of the GQA group, each K/V
tile loaded once for two heads.

Per head the kernel does cosa_attend's arithmetic in the same order, so its
outputs, log-sum-exps and skip bits must equal cosa_attend's on the same
order given to every head bit for bit, and the oracle's (bit-exact skips on
integer grids, outputs within tolerance).  The orders are CompactAttention's
block unions ("CompactAttention: Accelerating Chunked Prefill with
Block-Union KV Selection", method: Q-block and intra-group unions, executed
per group), random shared orders with invalid entries, and the dense path.
Expected values come from oracle/, inputs from synth/.
"""
import random

import pytest
import torch

import oracle
import synth
from test_gpu_parity import EPS, check_out, flat, gpu_rows, tiny, _samples

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cosa():
    import block_sparse_attention_kap_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def _expand(wl, gorder, gcount):
    """[B, Hkv, nQB, km] group orders -> [B*Hq*nQB, km] per-head rows (the
    oracle's layout), every head of a group given its group's order."""
    G = wl.Hq // wl.Hkv
    o = gorder.repeat_interleave(G, dim=1)
    c = gcount.repeat_interleave(G, dim=1)
    return o.reshape(-1, o.shape[-1]).contiguous(), c.reshape(-1).contiguous()


def _union_orders(wl, inp, budget):
    """The oracle's M_KAP, its block union per (b, kv-head) over the call's
    Q-blocks and the group's heads, and each Q-block's causally visible part
    of the union: [B, Hkv, nQB, nKB] / [B, Hkv, nQB]."""
    plan = oracle.kap(inp, budget)
    _, rows = oracle.block_union(wl, plan["order"], plan["count"])
    G = wl.Hq // wl.Hkv
    order = torch.full((wl.B, wl.Hkv, wl.n_qblocks, wl.n_kblocks), -1, dtype=torch.int32)
    count = torch.zeros(wl.B, wl.Hkv, wl.n_qblocks, dtype=torch.int32)
    for b in range(wl.B):
        for g in range(wl.Hkv):
            for I in range(wl.n_qblocks):
                r = rows[(b * wl.Hq + g * G) * wl.n_qblocks + I]
                order[b, g, I, : len(r)] = torch.tensor(r, dtype=torch.int32)
                count[b, g, I] = len(r)
    return order, count


def _random_group_orders(wl, frac, seed):
    """Random subsets of each Q-block's causal blocks in random order, shared
    by the group, with an out-of-range and a negative entry now and then."""
    rng = random.Random(seed)
    order = torch.full((wl.B, wl.Hkv, wl.n_qblocks, wl.n_kblocks + 1), -1, dtype=torch.int32)
    count = torch.zeros(wl.B, wl.Hkv, wl.n_qblocks, dtype=torch.int32)
    for b in range(wl.B):
        for g in range(wl.Hkv):
            for I in range(wl.n_qblocks):
                n = oracle.causal_blocks(wl, I)
                js = rng.sample(range(n), max(1, int(n * frac)))
                if rng.random() < 0.3:
                    js.insert(rng.randrange(len(js) + 1), rng.choice([-1, wl.n_kblocks + 3]))
                order[b, g, I, : len(js)] = torch.tensor(js, dtype=torch.int32)
                count[b, g, I] = len(js)
    return order, count


def _clean(order, count, nkb):
    """Drop the entries that are not blocks (the kernels count them as
    skipped visits; the oracle takes only real blocks)."""
    o, c = order.clone(), count.clone()
    for i in range(o.shape[0]):
        keep = [j for j in o[i, : c[i]].tolist() if 0 <= j < nkb]
        o[i] = -1
        o[i, : len(keep)] = torch.tensor(keep, dtype=torch.int32)
        c[i] = len(keep)
    return o, c


def _both(cosa, m, dev, gorder, gcount, eps):
    """cosa_attend_group on the group orders and cosa_attend on the same
    orders given to every head."""
    q, k, v, pt = dev
    wl_G = m.shape.Hq // m.shape.Hkv
    grp = m.attend_group(q, k, v, gorder, gcount, eps, page_table=pt, lse=True, skip_bits=True)
    ho = gorder.repeat_interleave(wl_G, dim=1).contiguous()
    hc = gcount.repeat_interleave(wl_G, dim=1).contiguous()
    per = m.attend(q, k, v, ho, hc, eps, page_table=pt, lse=True, skip_bits=True)
    torch.cuda.synchronize()
    assert m.device_status() == 0
    return grp, per


GROUP_SHAPES = [
    dict(Hq=4, Hkv=1, Nq=512, Nkv=1024, bq=128, bk=128),                  # G = 4, queries after a cache
    dict(B=2, Hq=4, Hkv=2, Nq=1168, Nkv=1168, bq=128, bk=128),           # G = 2, ragged last blocks
    dict(Hq=8, Hkv=2, Nq=384, Nkv=2304, bq=128, bk=64),                  # 64-key blocks
    dict(Hq=4, Hkv=1, Nq=512, Nkv=1040, bq=64, bk=64, paged=True),       # paged, ragged last page
]


def _make(shape, seed=5):
    kw = dict(shape)
    paged = kw.pop("paged", False)
    wl = tiny(structured=True, n_needle=2, **kw)
    inp = synth.generate(wl, grid=True)
    if paged:
        wl = wl.replace(paged=True)
        inp = synth._to_paged(wl, inp.q, inp.k, inp.v, wid=seed)
    return inp


def _dev(inp):
    pt = inp.page_table.cuda() if inp.page_table is not None else None
    return inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), pt


@pytest.mark.parametrize("shape", GROUP_SHAPES)
@pytest.mark.parametrize("budget,eps", [(0.3, EPS), (0.3, 0.0), (1.0, EPS)])
def test_group_on_block_union_matches_oracle(cosa, shape, budget, eps):
    """CompactAttention's union orders on structured integer grids: skip
    bits bit-exact against the oracle, outputs within tolerance, and every
    output, lse and skip bit identical to cosa_attend's on the same orders."""
    inp = _make(shape)
    wl = inp.wl
    gorder, gcount = _union_orders(wl, inp, budget)
    m = cosa.CoSA(cosa.shape_of_workload(wl))
    dev = _dev(inp)
    grp, per = _both(cosa, m, dev, gorder.cuda(), gcount.cuda(), eps)
    assert torch.equal(grp["out"], per["out"])
    assert torch.equal(grp["lse"], per["lse"])
    assert torch.equal(grp["skip_bits"], per["skip_bits"])
    ho, hc = _expand(wl, gorder, gcount)
    o = oracle.osk(inp, ho, hc, eps)
    km = ho.shape[1]
    bits = cosa.unpack_skip_bits(flat(grp["skip_bits"]), km)
    assert torch.equal(bits, o["skipped"])
    if eps == 0.0:
        assert int(bits.sum()) == 0
    check_out(gpu_rows(grp["out"], wl), o["out"])


@pytest.mark.parametrize("shape", GROUP_SHAPES)
def test_group_random_orders_with_invalid_entries(cosa, shape):
    """Random shared orders (random subsets in random order, an entry that is
    not a block now and then) on N(0,1)-based inputs: identical to cosa_attend
    on the same orders, and to the oracle within tolerance."""
    kw = dict(shape)
    paged = kw.pop("paged", False)
    wl = tiny(structured=True, n_needle=2, **kw)
    inp = synth.generate(wl)
    if paged:
        wl = wl.replace(paged=True)
        inp = synth._to_paged(wl, inp.q, inp.k, inp.v, wid=6)
    gorder, gcount = _random_group_orders(wl, 0.6, 9)
    m = cosa.CoSA(cosa.shape_of_workload(wl))
    dev = _dev(inp)
    grp, per = _both(cosa, m, dev, gorder.cuda(), gcount.cuda(), EPS)
    assert torch.equal(grp["out"], per["out"])
    assert torch.equal(grp["skip_bits"], per["skip_bits"])
    ho, hc = _clean(*_expand(wl, gorder, gcount), wl.n_kblocks)
    o = oracle.osk(inp, ho, hc, 0.0)
    res0 = m.attend_group(dev[0], dev[1], dev[2], gorder.cuda(), gcount.cuda(), 0.0, page_table=dev[3])
    torch.cuda.synchronize()
    check_out(gpu_rows(res0["out"], wl), o["out"])


@pytest.mark.parametrize("shape", GROUP_SHAPES)
def test_group_dense_path_matches_oracle(cosa, shape):
    """The dense path through the group kernel (every causal block, eps 0):
    equal to the oracle's dense attention within tolerance and bit for bit
    to the per-head dense path."""
    kw = dict(shape)
    paged = kw.pop("paged", False)
    wl = tiny(**kw)
    inp = synth.generate(wl)
    if paged:
        wl = wl.replace(paged=True)
        inp = synth._to_paged(wl, inp.q, inp.k, inp.v, wid=6)
    m = cosa.CoSA(cosa.shape_of_workload(wl))
    q, k, v, pt = _dev(inp)
    a = m.dense(q, k, v, page_table=pt, group=True, lse=True)
    b = m.dense(q, k, v, page_table=pt, lse=True)
    torch.cuda.synchronize()
    assert torch.equal(a["out"], b["out"]) and torch.equal(a["lse"], b["lse"])
    check_out(gpu_rows(a["out"], wl), oracle.dense(inp)["out"], literal=True)


def test_group_of_one_head_runs_the_per_head_kernel(cosa):
    wl = tiny(Hq=2, Hkv=2, Nq=512, Nkv=512, bq=128, bk=128, structured=True, n_needle=1)
    inp = synth.generate(wl, grid=True)
    gorder, gcount = _random_group_orders(wl, 0.7, 3)
    m = cosa.CoSA(cosa.shape_of_workload(wl))
    grp, per = _both(cosa, m, _dev(inp), gorder.cuda(), gcount.cuda(), EPS)
    assert torch.equal(grp["out"], per["out"]) and torch.equal(grp["skip_bits"], per["skip_bits"])


def test_group_rejects_an_odd_group(cosa):
    s = cosa.make_shape(1, 6, 2, 256, 256)
    P = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(cosa.CosaError):
        cosa.cosa_attend_group(s, torch.zeros(6 * 256 * 128, dtype=torch.bfloat16, device="cuda"),
                               torch.zeros(2 * 256 * 128, dtype=torch.bfloat16, device="cuda"),
                               torch.zeros(2 * 256 * 128, dtype=torch.bfloat16, device="cuda"), None, P, P, 2, 0.0,
                               torch.zeros(6 * 256 * 128, dtype=torch.bfloat16, device="cuda"))


def test_group_full_chunk_union(cosa):
    """The 4096-query chunk after a 128K paged cache (64-token pages): M_KAP
    from cosa_plan, its union from cosa_block_union, executed per group:
    identical to cosa_attend on the union orders (eps 0 and eps 1e-4), and on
    sampled rows equal to the oracle's dense attention over the union
    (eps 0)."""
    wl = synth.WORKLOADS["chunked_128k_paged"]
    inp = synth.generate(wl)
    m = cosa.CoSA(cosa.shape_of_workload(wl))
    dev = _dev(inp)
    plan = m.plan(dev[0], dev[1], 0.1, page_table=dev[3])
    un = m.block_union(plan["order"], plan["count"])
    G = wl.Hq // wl.Hkv
    gorder = un["order"].view(wl.B, wl.Hkv, G, wl.n_qblocks, -1)[:, :, 0].contiguous()
    gcount = un["count"].view(wl.B, wl.Hkv, G, wl.n_qblocks)[:, :, 0].contiguous()
    # the union rows of a group's heads are the same
    assert torch.equal(un["order"].view(wl.B, wl.Hkv, G, wl.n_qblocks, -1),
                       gorder.unsqueeze(2).expand(-1, -1, G, -1, -1))
    for eps in (0.0, EPS):
        grp, per = _both(cosa, m, dev, gorder, gcount, eps)
        assert torch.equal(grp["out"], per["out"]) and torch.equal(grp["skip_bits"], per["skip_bits"])
    sel = _samples(wl, 6, 11)
    idx = [(b * wl.Hq + h) * wl.n_qblocks + I for b, h, I in sel]
    ho = flat(un["order"])[idx]
    hc = flat(un["count"]).view(-1)[idx]
    ref = oracle.dense(inp, sel=sel, order=ho, count=hc)
    grp0 = m.attend_group(dev[0], dev[1], dev[2], gorder, gcount, 0.0, page_table=dev[3])
    torch.cuda.synchronize()
    check_out(gpu_rows(grp0["out"], wl)[idx], ref["out"], literal=True)
