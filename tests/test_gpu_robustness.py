"""Robustness of the CUDA path through the C ABI, in forms that fault no GPU.

* Guard bands: every output and scratch buffer the library writes (order,
  count, HRM count, block scores, HRM flags, the workspace, the pooled-key
  cache, out, lse, skip bits, union tables, the status word) is placed inside
  a larger allocation whose bands before and after it hold a byte pattern;
  after the calls the bands must be untouched and the results still equal
  the oracle's.  This stands in for a memory checker on this GPU pool.
* NaN page tails: a paged cache whose last logical page is ragged holds NaN
  (and Inf) in its rows past the end of the cache; no key there is visible,
  so the outputs must stay finite and equal the oracle's, which never reads
  those rows.

Expected values come from oracle/, inputs from synth/.
"""
import pytest
import torch

import oracle
import synth
from test_gpu_parity import EPS, check_out, flat, gpu_rows, tiny

pytestmark = pytest.mark.gpu

BAND = 4096          # bytes of pattern on each side of a buffer
PATTERN = 0xA5


@pytest.fixture(scope="module")
def cosa():
    import block_sparse_attention_kap_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


class Banded:
    """A device tensor of the given shape and dtype inside a byte buffer
    with BAND pattern bytes before and after it (BAND keeps every view
    256-byte aligned)."""

    def __init__(self, shape, dtype, fill=None):
        n = 1
        for x in shape:
            n *= x
        nbytes = n * torch.empty(0, dtype=dtype).element_size()
        self.raw = torch.full((BAND + nbytes + BAND,), PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.raw[BAND:BAND + nbytes].view(dtype).view(*shape)
        if fill is not None:
            self.t.fill_(fill)
        self.nbytes = nbytes

    def bands_intact(self) -> bool:
        head = self.raw[:BAND]
        tail = self.raw[BAND + self.nbytes:]
        return bool((head == PATTERN).all()) and bool((tail == PATTERN).all())


@pytest.mark.parametrize("shape", [
    dict(B=2, Hq=4, Hkv=2, Nq=1168, Nkv=1168, bq=128, bk=128),                     # ragged last blocks
    dict(Hq=4, Hkv=1, Nq=384, Nkv=2304, bq=128, bk=64),                            # chunk after a cache
    dict(Hq=4, Hkv=2, Nq=512, Nkv=1040, bq=64, bk=64, paged=True),                 # paged, ragged last page
])
def test_guard_bands_plan_and_attend(cosa, shape):
    kw = dict(shape)
    paged = kw.pop("paged", False)
    wl = tiny(structured=True, n_needle=2, **kw)
    inp = synth.generate(wl, grid=True)
    if paged:
        wl = wl.replace(paged=True)
        inp = synth._to_paged(wl, inp.q, inp.k, inp.v, wid=5)
    budget = 0.4
    s = cosa.shape_of_workload(wl)
    nqb, nkb = cosa.cosa_num_qblocks(s), cosa.cosa_num_kblocks(s)
    km = cosa.cosa_kmax(s, budget)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    pt = inp.page_table.cuda() if paged else None
    bufs = dict(
        order=Banded((wl.B, wl.Hq, nqb, km), torch.int32),
        count=Banded((wl.B, wl.Hq, nqb), torch.int32),
        hrm=Banded((wl.B, wl.Hq, nqb), torch.int32),
        score=Banded((wl.B, wl.Hq, nqb, nkb), torch.float32),
        flags=Banded((wl.B, wl.Hq, nqb, nkb), torch.uint8),
        ws=Banded((cosa.cosa_plan_workspace_bytes(s),), torch.uint8),
        status=Banded((1,), torch.int32, fill=0),
        out=Banded((wl.B, wl.Hq, wl.Nq, wl.d), torch.bfloat16),
        lse=Banded((wl.B, wl.Hq, wl.Nq), torch.float32),
        bits=Banded((wl.B, wl.Hq, nqb, (km + 31) // 32), torch.int32),
        table=Banded((wl.B, wl.Hkv, nkb), torch.int32),
        table_len=Banded((wl.B, wl.Hkv), torch.int32),
        uorder=Banded((wl.B, wl.Hq, nqb, nkb), torch.int32),
        ucount=Banded((wl.B, wl.Hq, nqb), torch.int32),
    )
    b = {n: x.t for n, x in bufs.items()}
    cosa.cosa_plan(s, q, k, pt, budget, km, b["order"], b["count"], b["hrm"], b["score"], b["flags"], b["ws"],
                   b["status"])
    cosa.cosa_attend(s, q, k, v, pt, b["order"], b["count"], km, EPS, b["out"], b["lse"], b["bits"], b["status"])
    cosa.cosa_block_union(s, b["order"], b["count"], km, b["table"], b["table_len"], b["uorder"], b["ucount"])
    torch.cuda.synchronize()
    assert int(b["status"].item()) == 0
    for name, x in bufs.items():
        assert x.bands_intact(), f"a kernel wrote outside {name}"
    ref = oracle.kap(inp, budget, want_scores=True)
    assert torch.equal(flat(b["order"]), ref["order"])
    assert torch.equal(flat(b["count"]).view(-1), ref["count"])
    assert torch.equal(flat(b["score"]), ref["score"])
    o = oracle.osk(inp, ref["order"], ref["count"], EPS)
    assert torch.equal(cosa.unpack_skip_bits(flat(b["bits"]), km), o["skipped"])
    check_out(gpu_rows(b["out"], wl), o["out"])


def test_guard_bands_chunk_cache_and_decode(cosa):
    """cosa_plan_chunk's pooled-key cache and cosa_decode_plan's outputs."""
    wl = tiny(Hq=4, Hkv=2, Nq=256, Nkv=1024, bq=128, bk=64, structured=True, n_needle=2)
    inp = synth.generate(wl, grid=True)
    s = cosa.shape_of_workload(wl)
    budget = 0.3
    nqb, nkb = cosa.cosa_num_qblocks(s), cosa.cosa_num_kblocks(s)
    km = cosa.cosa_kmax(s, budget)
    q, k = inp.q.cuda(), inp.k.cuda()
    cap = wl.Nkv // wl.stride
    cache = Banded((wl.B, wl.Hkv, cap, wl.d), torch.bfloat16, fill=0)
    order = Banded((wl.B, wl.Hq, nqb, km), torch.int32)
    count = Banded((wl.B, wl.Hq, nqb), torch.int32)
    ws = Banded((cosa.cosa_plan_workspace_bytes(s),), torch.uint8)
    cosa.cosa_plan_chunk(s, q, k, None, cache.t, 0, budget, km, order.t, count.t, workspace=ws.t)
    # one decode step after the cache: the last query row of each head
    ds = cosa.make_shape(wl.B, wl.Hq, wl.Hkv, 1, wl.Nkv, wl.d, 128, wl.bk, wl.stride)
    qd = q[:, :, -1:].contiguous()
    dorder = Banded((wl.B, wl.Hq, 1, nkb), torch.int32)
    dcount = Banded((wl.B, wl.Hq, 1), torch.int32)
    dhrm = Banded((wl.B, wl.Hq, 1), torch.int32)
    dscore = Banded((wl.B, wl.Hq, 1, nkb), torch.float32)
    dflags = Banded((wl.B, wl.Hq, 1, nkb), torch.uint8)
    cosa.cosa_decode_plan(ds, qd, k, None, cache.t, cap, budget, nkb, dorder.t, dcount.t, dhrm.t, dscore.t,
                          dflags.t)
    torch.cuda.synchronize()
    for name, x in dict(cache=cache, order=order, count=count, ws=ws, dorder=dorder, dcount=dcount, dhrm=dhrm,
                        dscore=dscore, dflags=dflags).items():
        assert x.bands_intact(), f"a kernel wrote outside {name}"
    ref = oracle.kap(inp, budget)
    assert torch.equal(flat(order.t), ref["order"])
    pooled = oracle.pool(inp.k.reshape(-1, wl.d), wl.stride).view(wl.B, wl.Hkv, cap, wl.d)
    assert torch.equal(cache.t.cpu(), pooled)
    dref = oracle.decode_kap(qd.view(wl.B, wl.Hq, wl.d).cpu(), inp.k, wl.bk, wl.stride, budget)
    kk = dref["order"].shape[1]
    assert torch.equal(dorder.t.view(wl.B * wl.Hq, -1)[:, :kk].cpu(), dref["order"])
    assert torch.equal(dscore.t.view(wl.B * wl.Hq, -1).cpu(), dref["score"])


@pytest.mark.parametrize("bk,Nkv", [(64, 1040), (128, 1168), (64, 1101)])
@pytest.mark.parametrize("eps", [0.0, EPS])
def test_nan_in_ragged_page_tail(cosa, bk, Nkv, eps):
    """The rows of the last page past the end of the cache hold NaN and Inf
    (stale or uninitialised pool memory in a serving cache).  No query sees
    them, so plan, skip bits and outputs must equal the oracle's and every
    output stay finite.  Nkv = 1101 also leaves a partial 16-key step."""
    Nq = 256
    stride = 16 if Nkv % 16 == 0 else 1        # the proxy needs Nkv to be a multiple of its stride
    wl = tiny(Hq=4, Hkv=2, Nq=Nq, Nkv=Nkv, bq=128, bk=bk, stride=stride, structured=True, n_needle=2)
    grid = synth.generate(wl, grid=True)
    wl = wl.replace(paged=True)
    inp = synth._to_paged(wl, grid.q, grid.k, grid.v, wid=7)
    tail = Nkv % bk
    assert tail > 0
    kp, vp = inp.k.clone(), inp.v.clone()
    for b in range(wl.B):
        last = int(inp.page_table[b, -1])
        kp[last, :, tail:] = float("nan")
        vp[last, :, tail:] = float("nan")
        vp[last, :, tail::3] = float("inf")
    poisoned = synth.Inputs(wl, inp.q, kp, vp, inp.page_table)
    s = cosa.shape_of_workload(wl)
    m = cosa.CoSA(s)
    q, k, v, pt = poisoned.q.cuda(), poisoned.k.cuda(), poisoned.v.cuda(), poisoned.page_table.cuda()
    budget = 1.0
    plan = None
    if stride == 16:
        plan = m.plan(q, k, budget, page_table=pt)
        order, count = plan["order"], plan["count"]
    else:
        order, count = m.dense_order()
    res = m.attend(q, k, v, order, count, eps, page_table=pt, lse=True, skip_bits=True)
    torch.cuda.synchronize()
    assert m.device_status() == 0
    assert bool(torch.isfinite(res["out"].float()).all())
    assert bool(torch.isfinite(res["lse"]).all())
    ref_order, ref_count = flat(order), flat(count).view(-1)
    if plan is not None:
        ref = oracle.kap(inp, budget)          # the un-poisoned pool: the plan must not see the tail
        km = ref["order"].shape[1]
        assert torch.equal(ref_order[:, :km], ref["order"])
        ref_order, ref_count = ref["order"], ref["count"]
    o = oracle.osk(inp, ref_order, ref_count, eps)
    km = ref_order.shape[1]
    assert torch.equal(cosa.unpack_skip_bits(flat(res["skip_bits"]), km), o["skipped"])
    check_out(gpu_rows(res["out"], wl), o["out"])


def test_bounded_wait_gives_up_and_reports(cosa):
    """Failure detection on the GPU without a fault: the test hook makes one
    wait per CTA of the attention kernel wait on a barrier nothing arrives
    at.  Every wait of the kernel is bounded (here by 2 ms), so the kernel
    must end by itself with a timeout code in the status word; CTAs that
    ran write zero rows, CTAs that start after the report exit at once and
    leave their rows untouched, and the context stays usable: the next
    normal call on the same buffers is correct.  512 CTAs, more than the
    GPU holds at once, so both kinds of CTA occur."""
    import time
    wl = tiny(Hq=8, Hkv=2, Nq=8192, Nkv=8192, bq=128, bk=128, structured=True, n_needle=4)
    inp = synth.generate(wl, grid=True)
    m = cosa.CoSA(cosa.shape_of_workload(wl))
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    plan = m.plan(q, k, 1.0)
    km = plan["order"].shape[-1]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full((wl.B, wl.Hq, wl.Nq, wl.d), 7.0, dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    cosa.cosa_test_attend_wait_timeout(m.shape, q, k, v, None, plan["order"], plan["count"], km, out, status,
                                       2_000_000)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    code = int(status.item())
    assert code in (cosa.DEV_TIMEOUT_PIPE, cosa.DEV_TIMEOUT_MMA), hex(code)
    assert elapsed < 5.0
    blocks = out.float().view(wl.B * wl.Hq * wl.n_qblocks, wl.bq * wl.d)
    zero = (blocks == 0).all(1)
    kept = (blocks == 7).all(1)
    assert bool((zero | kept).all())
    assert int(zero.sum()) > 0 and int(kept.sum()) > 0
    # the same context and buffers, a normal call: correct on sampled rows
    m.status.zero_()
    res = m.attend(q, k, v, plan["order"], plan["count"], EPS, out=out, skip_bits=True)
    torch.cuda.synchronize()
    assert m.device_status() == 0
    sel = [(0, 0, 63), (0, 3, 17), (0, 7, 0), (0, 5, 40)]
    idx = [(b * wl.Hq + h) * wl.n_qblocks + I for b, h, I in sel]
    ref = oracle.kap(inp, 1.0, sel=sel, kmax_=km)
    assert torch.equal(flat(plan["order"])[idx], ref["order"])
    o = oracle.osk(inp, ref["order"], ref["count"], EPS, sel=sel)
    assert torch.equal(cosa.unpack_skip_bits(flat(res["skip_bits"]), km)[idx], o["skipped"])
    check_out(gpu_rows(res["out"], wl)[idx], o["out"])
