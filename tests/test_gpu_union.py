"""Block union (cosa_block_union, CompactAttention's selection stage) against
the oracle, and the union executed by cosa_attend.

Index work: tables, lengths and the per-Q-block orders are compared bit for
bit.  Inputs are seeded synthetic selections (with padding, negative and
out-of-range entries and counts beyond kmax) or the oracle's own KAP plan;
nothing the GPU computes is fed to the oracle.
"""
import pytest
import torch

import oracle
import synth
from test_gpu_parity import EPS, check_out, flat, gpu_rows, tiny

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cosa():
    import block_sparse_attention_kap_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def _random_selection(wl, km, seed):
    g = torch.Generator().manual_seed(seed)
    n = wl.B * wl.Hq * wl.n_qblocks
    order = torch.randint(-3, wl.n_kblocks + 3, (n, km), generator=g, dtype=torch.int32)
    count = torch.randint(-1, km + 3, (n,), generator=g, dtype=torch.int32)
    return order, count


def _check_union(cosa, wl, order, count):
    m = cosa.CoSA(cosa.shape_of_workload(wl))
    km = order.shape[-1]
    res = m.block_union(order.view(wl.B, wl.Hq, wl.n_qblocks, km).cuda(),
                        count.view(wl.B, wl.Hq, wl.n_qblocks).cuda())
    torch.cuda.synchronize()
    tables, rows = oracle.block_union(wl, order, count)
    tab = res["table"].view(wl.B * wl.Hkv, -1).cpu()
    tlen = res["table_len"].view(-1).cpu()
    for i, t in enumerate(tables):
        assert tlen[i].item() == len(t)
        assert tab[i, : len(t)].tolist() == t
        assert bool((tab[i, len(t):] == -1).all())
    uo = flat(res["order"])
    uc = flat(res["count"]).view(-1)
    for i, r in enumerate(rows):
        assert uc[i].item() == len(r)
        assert uo[i, : len(r)].tolist() == r
        assert bool((uo[i, len(r):] == -1).all())
    return m, res


UNION_SHAPES = [
    dict(B=2, Hq=8, Hkv=2, Nq=384, Nkv=2048, bq=128, bk=64),
    dict(B=1, Hq=4, Hkv=4, Nq=200, Nkv=3000, bq=64, bk=128),        # G = 1, ragged
    dict(B=1, Hq=32, Hkv=8, Nq=4096, Nkv=131072, bq=128, bk=64),    # the chunk after a 127K cache
]


@pytest.mark.parametrize("shape", UNION_SHAPES)
def test_union_random_selection_bit_exact(cosa, shape):
    wl = tiny(**shape)
    order, count = _random_selection(wl, 37, seed=shape["Nkv"])
    _check_union(cosa, wl, order, count)


def test_union_of_kap_plan_executes(cosa):
    """The oracle's KAP plan of a chunk -> union on both sides -> cosa_attend
    over the union order with eps 0 (dense attention over the union, as
    CompactAttention's execution stage runs it) and with eps > 0, against the
    oracle's OSK on the same union order."""
    wl = tiny(Hq=4, Hkv=1, Nq=384, Nkv=2304, bq=128, bk=64, structured=True, n_needle=2)
    inp = synth.generate(wl, grid=True)                  # exact logits: skip decisions compare bit for bit
    budget = 0.2
    ref = oracle.kap(inp, budget)
    m, res = _check_union(cosa, wl, ref["order"], ref["count"])
    _, rows = oracle.block_union(wl, ref["order"], ref["count"])
    km = max(len(r) for r in rows)
    o_ref = torch.full((len(rows), km), -1, dtype=torch.int32)
    c_ref = torch.tensor([len(r) for r in rows], dtype=torch.int32)
    for i, r in enumerate(rows):
        o_ref[i, : len(r)] = torch.tensor(r, dtype=torch.int32)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    for eps in (0.0, EPS):
        out = m.attend(q, k, v, res["order"], res["count"], eps, lse=True, skip_bits=True)
        torch.cuda.synchronize()
        assert m.device_status() == 0
        o = oracle.osk(inp, o_ref, c_ref, eps)
        bits = cosa.unpack_skip_bits(flat(out["skip_bits"]), km)
        assert torch.equal(bits, o["skipped"])
        if eps == 0.0:
            assert int(bits.sum()) == 0
        check_out(gpu_rows(out["out"], wl), o["out"])
    # the union visits at least every block KAP selected for that Q-block
    assert bool((c_ref >= ref["count"]).all())
