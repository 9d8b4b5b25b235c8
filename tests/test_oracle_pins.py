"""Pins of the CPU oracle against what the CoSA pages and mathematics fix.

None of these re-types the oracle's own code: each checks it against a
hand-worked example (tests/golden), exact rational arithmetic, a library
routine (torch's scaled_dot_product_attention in fp64), or an invariant the
pages state (order invariance, HRM holds the row max, flag-grouped order,
budget 100% with threshold 0 equals dense attention).
Pages: CoSA technical summary (gist.science/paper/2607.25291) Sec. 1, 2.1-2.3.
"""
import math
import os
import random

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def tiny(name="t", **kw):
    base = dict(name=name, wid=90, B=1, Hq=2, Hkv=1, Nq=512, Nkv=512, d=32, bq=64, bk=64,
                stride=16, structured=False)
    base.update(kw)
    return synth.Workload(**base)


def inputs_from(wl, q, k, v):
    return synth.Inputs(wl, q.to(torch.bfloat16).contiguous(), k.to(torch.bfloat16).contiguous(),
                        v.to(torch.bfloat16).contiguous())


# ----------------------------------------------------------------- library reference

def sdpa_reference(inp, allowed_blocks=None):
    """fp64 attention through torch's SDPA (math path) with the causal mask
    (key <= Nkv-Nq+query) and, optionally, a per-(b,h,I) set of KV blocks.
    Returns [B, Hq, Nq, d] with rows that see no key set to 0."""
    wl = inp.wl
    k, v = synth.logical_kv(inp)
    G = wl.Hq // wl.Hkv
    q64 = inp.q.double()
    k64 = k.double().repeat_interleave(G, dim=1)
    v64 = v.double().repeat_interleave(G, dim=1)
    off = wl.Nkv - wl.Nq
    qi = torch.arange(wl.Nq)[:, None]
    kc = torch.arange(wl.Nkv)[None, :]
    mask = (kc <= off + qi).expand(wl.B, wl.Hq, wl.Nq, wl.Nkv).clone()
    if allowed_blocks is not None:
        blk = torch.zeros(wl.B, wl.Hq, wl.n_qblocks, wl.n_kblocks, dtype=torch.bool)
        for (b, h, I), js in allowed_blocks.items():
            blk[b, h, I, list(js)] = True
        rowmask = blk.repeat_interleave(wl.bq, dim=2)[:, :, : wl.Nq]
        colmask = rowmask.repeat_interleave(wl.bk, dim=3)[..., : wl.Nkv]
        mask &= colmask
    out = torch.nn.functional.scaled_dot_product_attention(q64, k64, v64, attn_mask=mask)
    none = ~mask.any(dim=-1)
    out[none] = 0.0
    return out


def full_rows(res, wl):
    return oracle.rows_of(res["out"], wl)


# ----------------------------------------------------------------- golden: KAP by hand

def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line)
    return rows


def test_kap_hand_example():
    rows = _read_golden("kap_hand_example.txt")
    qp = [float(x) for x in rows[0].split()[1:]]
    kp = [float(x) for x in rows[1].split()[1:]]
    wl = tiny(Hq=1, Nq=96, Nkv=96, d=2, bq=32, bk=32)
    q = torch.tensor(qp).view(6, 1, 2).expand(6, 16, 2).reshape(1, 1, 96, 2)
    k = torch.tensor(kp).view(6, 1, 2).expand(6, 16, 2).reshape(1, 1, 96, 2)
    inp = inputs_from(wl, q, k, torch.zeros_like(k))
    scores = [[float(x) for x in r.split()[1:]] for r in rows if r.startswith("score")]
    hrms = [[int(x) for x in r.split()[1:]] for r in rows if r.startswith("hrm ")]
    hrm_count = [int(x) for x in [r for r in rows if r.startswith("hrm_count")][0].split()[1:]]
    for r in [r for r in rows if r.startswith("budget")]:
        parts = r.split()
        beta = float(parts[1])
        ks = [int(x) for x in parts[3:6]]
        orders = [[int(x) for x in grp.split()] for grp in " ".join(parts[7:]).split("|")]
        res = oracle.kap(inp, beta, want_scores=True)
        assert res["count"].tolist() == ks
        for I in range(3):
            assert res["order"][I, : ks[I]].tolist() == orders[I]
        assert res["hrm_count"].tolist() == hrm_count
        assert res["score"].tolist() == scores
        assert res["hrm"].tolist() == hrms


# ----------------------------------------------------------------- golden: OSK by hand

def _osk_hand_inputs():
    rows = _read_golden("osk_hand_example.txt")
    vals = {r.split()[0]: [float(x) for x in r.split()[1:]] for r in rows[:3]}
    wl = tiny(Hq=1, Nq=4, Nkv=4, d=1, bq=2, bk=2, stride=2)
    t = lambda x: torch.tensor(x).view(1, 1, 4, 1)
    return wl, inputs_from(wl, t(vals["q"]), t(vals["k"]), t(vals["v"])), rows[3:]


def test_osk_hand_example():
    wl, inp, cases = _osk_hand_inputs()
    e = math.exp
    dense2 = (e(15) - 1 + 4 * e(3)) / (e(15) + 1 + e(3))
    dense3 = (e(10) - 1 + 4 * e(2) + 8 * e(-4)) / (e(10) + 1 + e(2) + e(-4))
    named = {"tanh7.5": math.tanh(7.5), "tanh5": math.tanh(5.0)}
    for line in cases:
        f = dict(kv.split("=") for kv in line.split()[1:])
        order = [int(x) for x in f["order"].split(",")]
        eps = float(f["eps"])
        ordt = torch.tensor([[0, -1], order], dtype=torch.int32)
        cnt = torch.tensor([1, 2], dtype=torch.int32)
        res = oracle.osk(inp, ordt, cnt, eps)
        assert res["skipped"][1].tolist() == [int(x) for x in f["skip"].split(",")]
        o = res["out"]
        assert o[0, 0, 0].item() == pytest.approx(1.0, abs=1e-12)
        assert o[0, 1, 0].item() == pytest.approx(math.tanh(5.0), abs=1e-12)
        exp2 = dense2 if f["out2"] == "dense" else named[f["out2"]]
        exp3 = dense3 if f["out3"] == "dense" else named[f["out3"]]
        assert o[1, 0, 0].item() == pytest.approx(exp2, abs=1e-12)
        assert o[1, 1, 0].item() == pytest.approx(exp3, abs=1e-12)
        # skip margins: mdiff (by hand) minus T, +inf where a row had no running max
        T = float(np.float32(math.log(eps))) if eps > 0 else -math.inf
        want = [math.inf if x == "inf" else float(x) - T for x in f["mdiff"].split(",")]
        mg = res["margin"]
        assert mg[0, 0].item() == math.inf and math.isnan(mg[0, 1].item())
        assert mg[1].tolist() == want
        if eps > 0:
            assert [int(x < 0) for x in want] == res["skipped"][1].tolist()


def test_skip_threshold_value():
    # T = fp32(ln(eps) * sqrt(d)) in raw-logit units
    assert oracle.skip_threshold(1e-4, 128) == np.float32(math.log(1e-4) * math.sqrt(128))
    assert oracle.skip_threshold(0.0, 128) == -math.inf
    assert abs(oracle.skip_threshold(1e-4, 128) + 104.2031) < 1e-3     # -9.21034 * 11.31371


# ----------------------------------------------------------------- pooling

def test_pool_grid_exact():
    g = torch.Generator().manual_seed(5)
    x = torch.randint(-2, 3, (256, 128), generator=g)
    p = oracle.pool(x.to(torch.bfloat16), 16)
    exact = x.view(16, 16, 128).sum(dim=1).double() / 16.0     # integers / 16: exact in bf16
    assert torch.equal(p.double(), exact)


def test_round_bf16_matches_float_conversion():
    """Direct fp64 -> bf16 rounding: on fp32-representable values it must
    agree with the fp32 -> bf16 RNE conversion (no double rounding there);
    ties go to even; the error never exceeds half a bf16 ulp."""
    g = torch.Generator().manual_seed(3)
    x32 = (torch.randn(20000, generator=g) * torch.exp2(torch.randint(-20, 20, (20000,), generator=g).float()))
    ref = x32.to(torch.bfloat16).double()
    assert torch.equal(oracle.round_bf16(x32.double()), ref)
    # exact ties: 1 + 2^-8 sits between 1 and 1 + 2^-7 -> even (1); 1 + 3*2^-8 -> 1 + 2^-6
    t = torch.tensor([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(2 + 2 ** -7), 0.0, float("inf")], dtype=torch.float64)
    assert oracle.round_bf16(t).tolist() == [1.0, 1 + 2 ** -6, -2.0, 0.0, float("inf")]
    # a value just above a tie that fp32 would round onto the tie first
    y = torch.tensor([1 + 2 ** -8 + 2 ** -40], dtype=torch.float64)
    assert oracle.round_bf16(y).item() == 1 + 2 ** -7
    z = torch.randn(5000, generator=g, dtype=torch.float64) * 3
    err = (oracle.round_bf16(z) - z).abs()
    half_ulp = torch.ldexp(torch.ones_like(z), torch.frexp(z)[1] - 9)
    assert bool((err <= half_ulp).all())


def test_pool_normal_within_half_ulp():
    g = torch.Generator().manual_seed(6)
    x = torch.randn(4096, 64, generator=g).to(torch.bfloat16)
    p = oracle.pool(x, 16).double()
    exact = x.double().view(256, 16, 64).mean(dim=1)
    # bf16 spacing at |p|: 2^(floor(log2|p|) - 7); RNE error <= half of it,
    # plus the fp32 summation error (<= 16 * 2^-24 * sum|x| / 16)
    ulp = torch.exp2(torch.floor(torch.log2(exact.abs().clamp_min(1e-30))) - 7)
    slack = x.double().abs().view(256, 16, 64).sum(dim=1) * 2.0 ** -24
    assert bool(((p - exact).abs() <= 0.5 * ulp + slack + 1e-30).all())


# ----------------------------------------------------------------- KAP: exact arithmetic

def _exact_kap(wl, q, k, beta):
    """Integer-exact KAP on grid inputs with Python ints (pooled value * s)."""
    s, bq, bk = wl.stride, wl.bq, wl.bk
    G = wl.Hq // wl.Hkv
    off = wl.Nkv - wl.Nq
    res = {}
    qs = q.long().view(wl.B, wl.Hq, wl.Nq // s, s, wl.d).sum(3)       # = s * pooled
    ks = k.long().view(wl.B, wl.Hkv, wl.Nkv // s, s, wl.d).sum(3)
    for b in range(wl.B):
        for h in range(wl.Hq):
            S = (qs[b, h] @ ks[b, h // G].T).tolist()                  # = s^2 * pooled score
            nr, nc = len(S), len(S[0])
            for I in range(wl.n_qblocks):
                rows = range(I * bq // s, min((I + 1) * bq, wl.Nq) // s)
                last_q = min((I + 1) * bq, wl.Nq) - 1
                n = min((off + last_q) // bk + 1, wl.n_kblocks)
                bs = {}
                for r in rows:
                    for j in range(wl.n_kblocks):
                        vals = [S[r][c] for c in range(j * bk // s, min((j + 1) * bk // s, nc))
                                if s * c <= off + s * r + s - 1]
                        bs[r, j] = max(vals) if vals else None
                score = {j: None for j in range(n)}
                hrm = {j: 0 for j in range(n)}
                for r in rows:
                    rowvals = [(bs[r, j], j) for j in range(wl.n_kblocks) if bs[r, j] is not None]
                    mx = max(v for v, _ in rowvals)
                    jstar = min(j for v, j in rowvals if v == mx)
                    hrm[jstar] = 1
                    for j in range(n):
                        if bs[r, j] is not None:
                            z = bs[r, j] - mx
                            score[j] = z if score[j] is None else max(score[j], z)
                bp = round(beta * 10000)
                kk = max(1, -(-n * bp // 10000))
                ranked = sorted(range(n), key=lambda j: (-hrm[j], -score[j], j))
                res[b, h, I] = (ranked[:kk], score, hrm)
    return res


@pytest.mark.parametrize("shape", [
    dict(Hq=2, Hkv=1, Nq=512, Nkv=512, bq=64, bk=64),
    dict(Hq=4, Hkv=2, Nq=256, Nkv=640, bq=128, bk=64),      # offset (chunk after a cache)
    dict(Hq=2, Hkv=2, Nq=400, Nkv=400, bq=128, bk=128),     # ragged last blocks
])
@pytest.mark.parametrize("beta", [0.3, 1.0])
def test_kap_exact_on_grid(shape, beta):
    wl = tiny(d=16, **shape)
    inp = synth.generate(wl, grid=True)
    res = oracle.kap(inp, beta, want_scores=True)
    ref = _exact_kap(wl, inp.q.float(), inp.k.float(), beta)
    s2 = float(wl.stride ** 2)
    nqb = wl.n_qblocks
    for (b, h, I), (ordr, score, hrm) in ref.items():
        i = (b * wl.Hq + h) * nqb + I
        assert res["count"][i].item() == len(ordr)
        assert res["order"][i, : len(ordr)].tolist() == ordr
        for j, z in score.items():
            assert res["score"][i, j].item() == z / s2
            assert res["hrm"][i, j].item() == hrm[j]
        assert res["hrm_count"][i].item() == sum(hrm.values())


@settings(max_examples=30, deadline=None, derandomize=True)
@given(B=st.sampled_from([1, 2]), hq_g=st.sampled_from([(1, 1), (2, 1), (2, 2), (4, 2), (4, 4)]),
       bq=st.sampled_from([32, 64, 128]), bk=st.sampled_from([32, 64, 128]), stride=st.sampled_from([8, 16]),
       nq_units=st.integers(1, 24), off_units=st.integers(0, 24), beta=st.sampled_from([0.05, 0.3, 0.7, 1.0]),
       structured=st.booleans(), wid=st.integers(0, 500))
def test_kap_exact_on_random_grids(B, hq_g, bq, bk, stride, nq_units, off_units, beta, structured, wid):
    """The same integer-exact brute force over random shapes: ragged Q- and
    KV-blocks, a causal offset (queries after a cache), strides 8 and 16,
    GQA groups of 1-4 heads and budgets from 5% to 100%."""
    Hq, G = hq_g
    Nq = stride * nq_units
    Nkv = Nq + stride * off_units
    wl = tiny(d=16, wid=wid, B=B, Hq=Hq, Hkv=Hq // G, Nq=Nq, Nkv=Nkv, bq=bq, bk=bk, stride=stride,
              structured=structured, n_needle=1 if structured else 0)
    inp = synth.generate(wl, grid=True)
    res = oracle.kap(inp, beta, want_scores=True)
    ref = _exact_kap(wl, inp.q.float(), inp.k.float(), beta)
    s2 = float(stride ** 2)
    for (b, h, I), (ordr, score, hrm) in ref.items():
        i = (b * wl.Hq + h) * wl.n_qblocks + I
        assert res["count"][i].item() == len(ordr)
        assert res["order"][i, : len(ordr)].tolist() == ordr
        for j, z in score.items():
            assert res["score"][i, j].item() == z / s2
            assert res["hrm"][i, j].item() == hrm[j]


# ----------------------------------------------------------------- KAP: invariants on real-valued data

def test_kap_invariants_structured():
    wl = synth.WORKLOADS["gqa_32k"].replace(Nq=4096, Nkv=4096, Hq=4, Hkv=1, d=128, n_needle=4)
    inp = synth.generate(wl)
    beta = 0.2
    res = oracle.kap(inp, beta, want_scores=True)
    G = wl.Hq // wl.Hkv
    s = wl.stride
    # pooled scores through torch (a library matmul), same pooled vectors
    qp = torch.stack([torch.stack([oracle.pool(inp.q[0, h], s) for h in range(wl.Hq)])])
    kp = torch.stack([torch.stack([oracle.pool(inp.k[0, g], s) for g in range(wl.Hkv)])])
    nqb, nkb = wl.n_qblocks, wl.n_kblocks
    for h in range(wl.Hq):
        S = (qp[0, h].double() @ kp[0, h // G].double().T)
        r = torch.arange(S.shape[0])[:, None]
        c = torch.arange(S.shape[1])[None, :]
        S[c > r] = -math.inf
        Bs = S.view(S.shape[0], nkb, wl.bk // s).amax(-1)
        argmax = Bs.argmax(-1)          # first index among equal maxima
        for I in range(nqb):
            i = h * nqb + I
            rows = range(I * wl.bq // s, (I + 1) * wl.bq // s)
            flagged = {j for j in range(nkb) if res["hrm"][i, j]}
            assert flagged == {int(argmax[r]) for r in rows}       # HRM holds each row's max
            for j in flagged:
                assert res["score"][i, j].item() == 0.0
            n = oracle.causal_blocks(wl, I)
            k = res["count"][i].item()
            assert k == max(1, -(-n * round(beta * 1e4) // 10000))
            ordr = res["order"][i, :k].tolist()
            assert len(set(ordr)) == k and all(0 <= j < n for j in ordr)
            keys = [(res["hrm"][i, j].item(), res["score"][i, j].item()) for j in ordr]
            assert keys == sorted(keys, reverse=True)               # HRM first, then score desc
            rest = [(res["hrm"][i, j].item(), res["score"][i, j].item())
                    for j in range(n) if j not in ordr]
            if rest:
                assert min(keys) >= max(rest)                         # selected = top-k


def test_budget_arithmetic():
    assert oracle.budget_blocks(30, 0.1) == 3           # float ceil(0.1*30) would give 4
    assert oracle.budget_blocks(1, 0.01) == 1
    assert oracle.budget_blocks(528, 1.0) == 528
    wl = synth.WORKLOADS["single_head_2k"]
    total = sum(oracle.budget_blocks(oracle.causal_blocks(wl, I), 0.25) for I in range(wl.n_qblocks))
    assert total == sum(-(-n // 4) for n in range(1, 33)) == 144


# ----------------------------------------------------------------- dense reference

@pytest.mark.parametrize("shape", [
    dict(Hq=2, Hkv=1, Nq=256, Nkv=256, bq=64, bk=64),
    dict(Hq=4, Hkv=2, Nq=128, Nkv=384, bq=128, bk=64),
    dict(Hq=2, Hkv=2, Nq=208, Nkv=208, bq=64, bk=128),
])
def test_dense_matches_sdpa(shape):
    wl = tiny(**shape)
    inp = synth.generate(wl)
    got = full_rows(oracle.dense(inp), wl)
    assert torch.allclose(got, sdpa_reference(inp), atol=1e-12, rtol=0)


def test_paged_equals_contiguous():
    wl = tiny(Hq=4, Hkv=2, Nq=128, Nkv=512, bq=128, bk=64, structured=True, n_needle=1)
    flat = synth.generate(wl)
    paged = synth._to_paged(wl.replace(paged=True), flat.q, flat.k, flat.v, wid=77)
    a, b = oracle.kap(flat, 0.5), oracle.kap(paged, 0.5)
    assert torch.equal(a["order"], b["order"])
    oa = oracle.osk(flat, a["order"], a["count"], 1e-4)
    ob = oracle.osk(paged, b["order"], b["count"], 1e-4)
    assert torch.equal(oa["out"], ob["out"]) and torch.equal(oa["skipped"], ob["skipped"])


# ----------------------------------------------------------------- OSK closed forms

def _random_orders(wl, frac, seed):
    rng = random.Random(seed)
    n_all = wl.B * wl.Hq * wl.n_qblocks
    km = wl.n_kblocks
    order = torch.full((n_all, km), -1, dtype=torch.int32)
    count = torch.zeros(n_all, dtype=torch.int32)
    allowed = {}
    i = 0
    for b in range(wl.B):
        for h in range(wl.Hq):
            for I in range(wl.n_qblocks):
                n = oracle.causal_blocks(wl, I)
                js = rng.sample(range(n), max(1, int(n * frac)))
                order[i, : len(js)] = torch.tensor(js, dtype=torch.int32)
                count[i] = len(js)
                allowed[b, h, I] = js
                i += 1
    return order, count, allowed


@pytest.mark.parametrize("shape", [
    dict(Hq=2, Hkv=1, Nq=512, Nkv=512, bq=64, bk=64),
    dict(Hq=4, Hkv=2, Nq=256, Nkv=640, bq=128, bk=64),
])
def test_osk_eps0_equals_block_masked_sdpa(shape):
    wl = tiny(**shape)
    inp = synth.generate(wl)
    order, count, allowed = _random_orders(wl, 0.5, 1)
    res = oracle.osk(inp, order, count, 0.0)
    assert res["skipped"].sum().item() == 0
    ref = sdpa_reference(inp, allowed)
    assert torch.allclose(full_rows(res, wl), ref, atol=1e-12, rtol=0)


@settings(max_examples=20, deadline=None, derandomize=True)
@given(B=st.sampled_from([1, 2]), hq_g=st.sampled_from([(1, 1), (2, 1), (4, 2), (4, 4)]),
       bq=st.sampled_from([32, 64, 128]), bk=st.sampled_from([32, 64, 128]), nq_units=st.integers(1, 20),
       off_units=st.integers(0, 20), frac=st.sampled_from([0.2, 0.5, 1.0]), paged=st.booleans(),
       wid=st.integers(0, 500))
def test_osk_eps0_equals_block_masked_sdpa_random(B, hq_g, bq, bk, nq_units, off_units, frac, paged, wid):
    """The same identity over random shapes: ragged blocks, queries after a
    cache, GQA groups, batches, a paged cache, random block subsets."""
    Hq, G = hq_g
    Nq = 16 * nq_units
    Nkv = Nq + 16 * off_units
    wl = tiny(d=32, wid=wid, B=B, Hq=Hq, Hkv=Hq // G, Nq=Nq, Nkv=Nkv, bq=bq, bk=bk, paged=paged)
    inp = synth.generate(wl)
    order, count, allowed = _random_orders(wl, frac, wid)
    res = oracle.osk(inp, order, count, 0.0)
    assert res["skipped"].sum().item() == 0
    ref = sdpa_reference(inp, allowed)
    assert torch.allclose(full_rows(res, wl), ref, atol=1e-12, rtol=0)


def test_full_budget_eps0_equals_dense():
    wl = tiny(Hq=4, Hkv=2, Nq=384, Nkv=384, bq=128, bk=128, structured=True, n_needle=1)
    inp = synth.generate(wl)
    plan = oracle.kap(inp, 1.0)
    res = oracle.osk(inp, plan["order"], plan["count"], 0.0)
    assert torch.allclose(full_rows(res, wl), sdpa_reference(inp), atol=1e-12, rtol=0)


def test_order_invariance():
    wl = tiny(Hq=2, Hkv=1, Nq=512, Nkv=512, bq=64, bk=64)
    inp = synth.generate(wl)
    order, count, _ = _random_orders(wl, 0.6, 2)
    perm = order.clone()
    g = torch.Generator().manual_seed(3)
    for i in range(order.shape[0]):
        c = count[i].item()
        perm[i, :c] = order[i, :c][torch.randperm(c, generator=g)]
    a = oracle.osk(inp, order, count, 0.0)
    b = oracle.osk(inp, perm, count, 0.0)
    assert (a["out"] - b["out"]).abs().max().item() < 1e-12
    assert (a["lse"] - b["lse"]).abs().max().item() < 1e-12


def test_skip_error_bound_and_monotone():
    """A skipped block's every weight is < eps relative to the running max
    weight, which is itself <= the final max; so per row the error against the
    block-masked dense result is <= 2 * max|v| * (skipped keys) * eps."""
    wl = synth.WORKLOADS["gqa_32k"].replace(Nq=2048, Nkv=2048, Hq=4, Hkv=1, n_needle=4)
    inp = synth.generate(wl)
    plan = oracle.kap(inp, 1.0)
    prev = None
    for eps in (1e-6, 1e-4, 1e-2):
        res = oracle.osk(inp, plan["order"], plan["count"], eps)
        sk = res["skipped"].bool()
        assert sk.any()
        ref = oracle.dense(inp, order=plan["order"], count=plan["count"])["out"]
        err = (res["out"] - ref).abs().amax(dim=(1, 2))
        vmax = inp.v.double().abs().max().item()
        bound = 2.0 * vmax * sk.sum(1).double() * wl.bk * eps
        assert bool((err <= bound + 1e-12).all())
        if prev is not None:
            assert bool((prev <= sk).all())          # a larger eps only adds skips
        prev = sk


def test_skip_decisions_bruteforce_grid():
    """On integer grids every logit is an exact integer: recompute each skip
    decision from the definition with numpy integers."""
    wl = tiny(Hq=2, Hkv=1, Nq=512, Nkv=512, bq=64, bk=64, d=32, structured=True, n_needle=2)
    inp = synth.generate(wl, grid=True)
    plan = oracle.kap(inp, 1.0)
    eps = 1e-3
    T = math.log(eps) * math.sqrt(wl.d)
    T32 = np.float32(T)
    res = oracle.osk(inp, plan["order"], plan["count"], eps)
    q = inp.q.long().numpy()
    k = inp.k.long().numpy()
    nqb = wl.n_qblocks
    for h in range(wl.Hq):
        for I in range(nqb):
            i = h * nqb + I
            L = q[0, h, I * 64:(I + 1) * 64] @ k[0, 0].T
            pos = np.arange(I * 64, (I + 1) * 64)[:, None]
            valid = np.arange(wl.Nkv)[None, :] <= pos
            m_run = np.full(64, -np.inf)
            for t in range(plan["count"][i].item()):
                j = plan["order"][i, t].item()
                blk = np.where(valid[:, j * 64:(j + 1) * 64], L[:, j * 64:(j + 1) * 64], -np.inf)
                m_loc = blk.max(1)
                vote = (m_loc == -np.inf) | (np.isfinite(m_run) & (m_loc - m_run < T))
                skip = bool(vote.all())
                assert res["skipped"][i, t].item() == int(skip)
                assert res["margin"][i, t].item() == _margin_by_definition(m_loc, m_run, T32)
                if not skip:
                    m_run = np.maximum(m_run, m_loc)
    assert res["skipped"].sum().item() > 0          # decisions of both kinds were checked


def _margin_by_definition(m_loc, m_run, T32):
    """The skip margin of one visit from its definition: over the rows whose
    m_loc is finite, the largest fp32(m_loc - m_run) - T (fp32 subtraction,
    then the difference to T in fp64); +inf if such a row has no running max
    yet or T = -inf (eps = 0); -inf if no row sees a key of the block.  The
    block is skipped iff this is negative (every row then votes skip)."""
    seen = np.isfinite(m_loc)
    if not seen.any():
        return -math.inf
    if not np.isfinite(T32) or not np.isfinite(m_run[seen]).all():
        return math.inf
    diff = np.float32(m_loc[seen]).astype(np.float32) - np.float32(m_run[seen]).astype(np.float32)
    return float(diff.astype(np.float32).max()) - float(T32)


@settings(max_examples=25, deadline=None, derandomize=True)
@given(hq_g=st.sampled_from([(1, 1), (2, 1), (4, 2)]), bq=st.sampled_from([32, 64]), bk=st.sampled_from([32, 64]),
       nq_units=st.integers(1, 12), off_units=st.integers(0, 12), frac=st.sampled_from([0.3, 0.7, 1.0]),
       eps=st.sampled_from([1e-4, 1e-3, 0.05, 0.5]), wid=st.integers(0, 500))
def test_skip_decisions_bruteforce_random(hq_g, bq, bk, nq_units, off_units, frac, eps, wid):
    """The same definition over random shapes and visit orders: ragged last
    Q-block (rows past Nq take no part in the vote), queries after a cache,
    GQA groups, random subsets of the causal blocks in random order."""
    Hq, G = hq_g
    Nq = 16 * nq_units
    Nkv = Nq + 16 * off_units
    wl = tiny(d=32, wid=wid, Hq=Hq, Hkv=Hq // G, Nq=Nq, Nkv=Nkv, bq=bq, bk=bk, structured=True, n_needle=1)
    inp = synth.generate(wl, grid=True)
    order, count, _ = _random_orders(wl, frac, wid)
    T = math.log(eps) * math.sqrt(wl.d)
    T32 = np.float32(T)
    res = oracle.osk(inp, order, count, eps)
    q = inp.q.long().numpy()
    k = inp.k.long().numpy()
    off = Nkv - Nq
    for h in range(Hq):
        for I in range(wl.n_qblocks):
            i = h * wl.n_qblocks + I
            r0, r1 = I * bq, min((I + 1) * bq, Nq)
            L = q[0, h, r0:r1] @ k[0, h // G].T
            pos = off + np.arange(r0, r1)[:, None]
            valid = np.arange(Nkv)[None, :] <= pos
            m_run = np.full(r1 - r0, -np.inf)
            for t in range(count[i].item()):
                j = order[i, t].item()
                c0, c1 = j * bk, min((j + 1) * bk, Nkv)
                blk = np.where(valid[:, c0:c1], L[:, c0:c1], -np.inf)
                m_loc = blk.max(1)
                with np.errstate(invalid="ignore"):          # -inf - -inf on rows the mask leaves out
                    vote = (m_loc == -np.inf) | (np.isfinite(m_run) & (m_loc - m_run < T))
                skip = bool(vote.all())
                assert res["skipped"][i, t].item() == int(skip), (h, I, t)
                assert res["margin"][i, t].item() == _margin_by_definition(m_loc, m_run, T32), (h, I, t)
                if not skip:
                    m_run = np.maximum(m_run, m_loc)


def test_skip_margin_rounds_the_difference_to_fp32():
    """The margin takes m_loc - m_run in fp32, as the skip test does (worked
    by hand): one head, d = 1, blocks of one token, query 1 = 1024 visits key
    0 = 1024 (logit 2^20, computed first) and then key 1 = (1 + 2^-7) / 1024
    (logit 1 + 2^-7).  The exact difference -1048574.9921875 lies between the
    fp32 neighbours -1048575 and -1048574.9375 (spacing 2^-4 below 2^20) and
    rounds to -1048575, so the margin is -1048575 - T, not the exact
    difference minus T."""
    wl = tiny(Hq=1, Nq=2, Nkv=2, d=1, bq=1, bk=1, stride=1)
    t = lambda x: torch.tensor(x, dtype=torch.float64).view(1, 1, 2, 1)
    inp = inputs_from(wl, t([1.0, 1024.0]), t([1024.0, (1.0 + 2.0 ** -7) / 1024.0]), t([1.0, -1.0]))
    assert inp.k[0, 0, 1, 0].double().item() == (1.0 + 2.0 ** -7) / 1024.0      # exact in bf16
    order = torch.tensor([[0, -1], [0, 1]], dtype=torch.int32)
    count = torch.tensor([1, 2], dtype=torch.int32)
    eps = 1e-4
    T32 = np.float32(math.log(eps))
    res = oracle.osk(inp, order, count, eps)
    assert res["margin"][1, 0].item() == math.inf
    assert res["margin"][1, 1].item() == -1048575.0 - float(T32)
    assert res["margin"][1, 1].item() != -1048574.9921875 - float(T32)
    assert res["skipped"][1].tolist() == [0, 1]
    assert res["out"][1, 0, 0].item() == 1.0          # the skipped key adds nothing


@settings(max_examples=20, deadline=None, derandomize=True)
@given(hq_g=st.sampled_from([(1, 1), (2, 1), (4, 2)]), bq=st.sampled_from([32, 64]), bk=st.sampled_from([32, 64]),
       nq_units=st.integers(1, 12), off_units=st.integers(0, 12), frac=st.sampled_from([0.3, 0.7, 1.0]),
       eps=st.sampled_from([0.0, 1e-4, 1e-2, 0.3]), wid=st.integers(0, 500))
def test_skip_margin_bruteforce_normal(hq_g, bq, bk, nq_units, off_units, frac, eps, wid):
    """The skip margin on real-valued (N(0,1) plus structure) inputs, which
    the GPU parity tests use to tell fragile skip decisions from robust ones:
    recomputed from its definition with numpy fp64 logits rounded to fp32
    (the products are summed in another order than the oracle's, so the
    comparison allows 1e-3 raw-logit units), decisions exact wherever the
    margin is farther than that from 0, and, from the oracle alone, a
    negative margin exactly on the skipped visits (+inf everywhere at eps 0)."""
    Hq, G = hq_g
    Nq = 16 * nq_units
    Nkv = Nq + 16 * off_units
    wl = tiny(d=32, wid=wid, Hq=Hq, Hkv=Hq // G, Nq=Nq, Nkv=Nkv, bq=bq, bk=bk, structured=True, n_needle=1)
    inp = synth.generate(wl)
    order, count, _ = _random_orders(wl, frac, wid)
    T = oracle.skip_threshold(eps, wl.d)
    T32 = np.float32(T)
    res = oracle.osk(inp, order, count, eps)
    q = inp.q.double().numpy()
    k = inp.k.double().numpy()
    off = Nkv - Nq
    for h in range(Hq):
        for I in range(wl.n_qblocks):
            i = h * wl.n_qblocks + I
            n = count[i].item()
            mg = res["margin"][i, :n]
            sk = res["skipped"][i, :n].bool()
            if eps == 0.0:
                assert bool(torch.isinf(mg).all() & (mg > 0).all()) and not sk.any()
            else:
                assert torch.equal(sk, mg < 0)
            r0, r1 = I * bq, min((I + 1) * bq, Nq)
            L = (q[0, h, r0:r1] @ k[0, h // G].T).astype(np.float32)
            pos = off + np.arange(r0, r1)[:, None]
            valid = np.arange(Nkv)[None, :] <= pos
            m_run = np.full(r1 - r0, -np.inf, dtype=np.float32)
            for t in range(n):
                j = order[i, t].item()
                c0, c1 = j * bk, min((j + 1) * bk, Nkv)
                m_loc = np.where(valid[:, c0:c1], L[:, c0:c1], -np.inf).max(1).astype(np.float32)
                want = _margin_by_definition(m_loc, m_run, T32)
                got = mg[t].item()
                if math.isinf(want):
                    assert got == want, (h, I, t)
                else:
                    assert abs(got - want) <= 1e-3, (h, I, t, got, want)
                if abs(want) > 1e-3:
                    assert bool(sk[t]) == (want < 0)
                if not sk[t]:
                    m_run = np.maximum(m_run, m_loc)


# ----------------------------------------------------------------- attention-mass recall of M_KAP

def test_mass_recall_identity():
    """The fraction of a row's dense softmax mass inside the selected blocks
    (the block attention mass m_b = sum over the block's keys of
    exp(q.k / sqrt(d)), normalised by the row total) equals
    exp(lse_selected - lse_dense).  Block masses come from a direct fp64
    matmul here; the lse values from the oracle's dense routine."""
    wl = tiny(Hq=2, Hkv=1, Nq=256, Nkv=384, bq=64, bk=64, structured=True, n_needle=1)
    inp = synth.generate(wl)
    plan = oracle.kap(inp, 0.3)
    dense = oracle.dense(inp)
    sel = oracle.dense(inp, order=plan["order"], count=plan["count"])
    recall = torch.exp(sel["lse"] - dense["lse"])                      # [n, bq]
    q = inp.q.double()
    k = inp.k.double()
    off = wl.Nkv - wl.Nq
    i = 0
    for h in range(wl.Hq):
        s = (q[0, h] @ k[0, 0].T) / math.sqrt(wl.d)                     # [Nq, Nkv]
        pos = torch.arange(wl.Nq)[:, None] + off
        s[torch.arange(wl.Nkv)[None, :] > pos] = -math.inf
        w = torch.softmax(s, dim=-1)
        for I in range(wl.n_qblocks):
            chosen = plan["order"][i, : plan["count"][i]].tolist()
            cols = torch.zeros(wl.Nkv, dtype=torch.bool)
            for j in chosen:
                cols[j * wl.bk:(j + 1) * wl.bk] = True
            mass = w[I * wl.bq:(I + 1) * wl.bq][:, cols].sum(-1)
            assert torch.allclose(recall[i], mass, atol=1e-12, rtol=1e-9)
            i += 1
    assert bool((recall <= 1 + 1e-12).all()) and bool((recall > 0).all())


# ----------------------------------------------------------------- block union (CompactAttention)

def test_block_union_hand_example():
    """CompactAttention, method, selection stage: per (batch, kv-head) the
    union over the chunk's Q-blocks and the group's heads.  Worked by hand:
    Hq=4, Hkv=2 (heads 0,1 -> group 0; 2,3 -> group 1), two Q-blocks of 128
    after 512 cached keys, blocks of 128 (nKB = 6; Q-block 0 sees blocks
    0..4, Q-block 1 sees 0..5).  Entries past count, negative entries and
    indices >= nKB are not selections; count is clamped to kmax."""
    wl = tiny(Hq=4, Hkv=2, Nq=256, Nkv=768, bq=128, bk=128)
    order = torch.tensor([[3, 1, -1], [0, 5, 2],      # h0: I0 {3,1}, I1 {0,5,2}
                          [4, 9, 9], [1, 7, 2],       # h1: I0 {4} (9 past count), I1 {1} (7 out of range)
                          [6, -1, -1], [2, 3, 12],    # h2: I0 {} (6 out of range), I1 {2,3}
                          [0, 0, 0], [8, 0, 0]],      # h3: I0 count 0, I1 count 5 -> 3: {0}
                         dtype=torch.int32)
    count = torch.tensor([2, 3, 1, 2, 1, 3, 0, 5], dtype=torch.int32)
    tables, rows = oracle.block_union(wl, order, count)
    assert tables == [[0, 1, 2, 3, 4, 5], [0, 2, 3]]
    assert rows == [[0, 1, 2, 3, 4], [0, 1, 2, 3, 4, 5]] * 2 + [[0, 2, 3], [0, 2, 3]] * 2


def test_block_union_properties_random():
    """Coverage (every selected block of the group is in its table),
    minimality (every table entry was selected by some Q-block or head of the
    group), ascending order, and each row's prefix = the table entries the
    Q-block can see -- checked against a boolean selection matrix built
    independently of the oracle's sets."""
    rng = torch.Generator().manual_seed(11)
    wl = tiny(B=2, Hq=8, Hkv=2, Nq=384, Nkv=2048, bq=128, bk=64)
    n, nkb, km = wl.B * wl.Hq * wl.n_qblocks, wl.n_kblocks, 9
    order = torch.randint(-3, nkb + 3, (n, km), generator=rng, dtype=torch.int32)
    count = torch.randint(-1, km + 3, (n,), generator=rng, dtype=torch.int32)
    tables, rows = oracle.block_union(wl, order, count)
    G = wl.Hq // wl.Hkv
    sel = torch.zeros(wl.B, wl.Hkv, nkb, dtype=torch.bool)
    o4 = order.view(wl.B, wl.Hq, wl.n_qblocks, km)
    c3 = count.view(wl.B, wl.Hq, wl.n_qblocks).clamp(0, km)
    t = torch.arange(km)
    valid = (t < c3[..., None]) & (o4 >= 0) & (o4 < nkb)
    for b in range(wl.B):
        for h in range(wl.Hq):
            sel[b, h // G, o4[b, h][valid[b, h]].long()] = True
    off = wl.Nkv - wl.Nq
    for b in range(wl.B):
        for g in range(wl.Hkv):
            tab = tables[b * wl.Hkv + g]
            assert tab == torch.nonzero(sel[b, g]).view(-1).tolist()
            for h in range(g * G, (g + 1) * G):
                for I in range(wl.n_qblocks):
                    last_key = off + min((I + 1) * wl.bq, wl.Nq) - 1
                    assert rows[(b * wl.Hq + h) * wl.n_qblocks + I] == [j for j in tab if j * wl.bk <= last_key]


# ----------------------------------------------------------------- decode step

@pytest.mark.parametrize("bk", [64, 128])
def test_decode_kap_equals_prefill_kap_of_a_repeated_query(bk):
    """A decode query at position Nkv-1 is the prefill proxy's single pooled
    row when its Q-block holds 16 copies of that query: the mean of 16 equal
    bf16 values is the value itself, the pooled causality 16c <= off + 15
    admits every pooled key, and the budget counts every block.  So the
    Python decode proxy must agree exactly with the C prefill proxy there."""
    g = torch.Generator().manual_seed(5)
    B, Hq, Hkv, Nkv, d = 2, 4, 2, 1024 + 3 * bk, 32
    q = (torch.randn(B, Hq, d, generator=g) * 2).to(torch.bfloat16)
    k = torch.randn(B, Hkv, Nkv, d, generator=g).to(torch.bfloat16)
    k[:, :, 5 * bk + 7] += 6                                        # a clear maximum somewhere
    for budget in (0.1, 0.37, 1.0):
        dec = oracle.decode_kap(q, k, bk, 16, budget)
        wl = tiny(B=B, Hq=Hq, Hkv=Hkv, Nq=16, Nkv=Nkv, d=d, bq=16, bk=bk)
        qq = q[:, :, None, :].expand(B, Hq, 16, d).contiguous()
        inp = synth.Inputs(wl, qq, k.contiguous(), k.contiguous())
        ref = oracle.kap(inp, budget, want_scores=True)
        assert torch.equal(dec["order"], ref["order"][:, : dec["order"].shape[1]])
        assert torch.equal(dec["count"], ref["count"])
        assert torch.equal(dec["hrm_count"], ref["hrm_count"])
        assert torch.equal(dec["score"], ref["score"])
        assert torch.equal(dec["hrm"], ref["hrm"])


@settings(max_examples=20, deadline=None, derandomize=True)
@given(B=st.sampled_from([1, 2]), hq_g=st.sampled_from([(1, 1), (2, 1), (4, 2), (4, 4)]),
       bk=st.sampled_from([32, 64, 128]), kv_units=st.integers(1, 60), budget=st.sampled_from([0.05, 0.2, 0.5, 1.0]),
       seed=st.integers(0, 10_000))
def test_decode_kap_equals_prefill_kap_random(B, hq_g, bk, kv_units, budget, seed):
    """The same equivalence over random cache lengths (a ragged last block),
    block sizes, GQA groups, batches and budgets."""
    Hq, G = hq_g
    Hkv, Nkv, d = Hq // G, 16 * kv_units, 32
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(B, Hq, d, generator=g) * 2).to(torch.bfloat16)
    k = torch.randn(B, Hkv, Nkv, d, generator=g).to(torch.bfloat16)
    dec = oracle.decode_kap(q, k, bk, 16, budget)
    wl = tiny(B=B, Hq=Hq, Hkv=Hkv, Nq=16, Nkv=Nkv, d=d, bq=16, bk=bk)
    qq = q[:, :, None, :].expand(B, Hq, 16, d).contiguous()
    ref = oracle.kap(synth.Inputs(wl, qq, k.contiguous(), k.contiguous()), budget, want_scores=True)
    assert torch.equal(dec["order"], ref["order"][:, : dec["order"].shape[1]])
    assert torch.equal(dec["count"], ref["count"])
    assert torch.equal(dec["hrm_count"], ref["hrm_count"])
    assert torch.equal(dec["score"], ref["score"])
    assert torch.equal(dec["hrm"], ref["hrm"])


def test_decode_osk_eps0_is_dense_attention_of_the_row():
    """With eps = 0 nothing is skipped, and visiting every block in any order
    is softmax attention of the one query row over the whole cache
    (Sec. 2.1, order invariance), checked against torch's SDPA in fp64."""
    g = torch.Generator().manual_seed(6)
    B, Hq, Hkv, Nkv, d, bk = 1, 4, 2, 1000, 128, 128
    q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, Hkv, Nkv, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, Nkv, d, generator=g).to(torch.bfloat16)
    nkb = -(-Nkv // bk)
    order = torch.stack([torch.randperm(nkb, generator=g) for _ in range(B * Hq)]).to(torch.int32)
    count = torch.full((B * Hq,), nkb, dtype=torch.int32)
    res = oracle.decode_osk(q, k, v, order, count, bk, 0.0)
    kk = k.double().repeat_interleave(Hq // Hkv, dim=1)
    vv = v.double().repeat_interleave(Hq // Hkv, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(q.double()[:, :, None, :], kk, vv)
    assert torch.allclose(res["out"].view(B, Hq, 1, d), ref, atol=1e-12, rtol=1e-10)
    assert int(res["skipped"].sum()) == 0


def test_decode_osk_skip_is_the_rows_own_test():
    """With one row the tile-wide vote is the row's own test: on integer
    logits, a visited block is skipped exactly when its max minus the running
    max (over the computed blocks before it) is below T, computed here by
    brute force."""
    g = torch.Generator().manual_seed(7)
    B, Hq, Hkv, Nkv, d, bk = 1, 2, 1, 1024, 32, 64
    q = torch.randint(-2, 3, (B, Hq, d), generator=g).to(torch.bfloat16)
    k = torch.randint(-2, 3, (B, Hkv, Nkv, d), generator=g).to(torch.bfloat16)
    k[:, :, 130] += 4 * q[:, 0].sign().to(torch.bfloat16)           # a block with much larger logits
    v = torch.randint(-2, 3, (B, Hkv, Nkv, d), generator=g).to(torch.bfloat16)
    nkb = Nkv // bk
    order = torch.stack([torch.tensor([2] + [j for j in range(nkb) if j != 2])] * Hq).to(torch.int32)
    count = torch.full((Hq,), nkb, dtype=torch.int32)
    eps = 1e-3
    res = oracle.decode_osk(q, k, v, order, count, bk, eps)
    T = oracle.skip_threshold(eps, d)
    for h in range(Hq):
        logits = (q[0, h].double() @ k[0, 0].double().T)
        m_run = float("-inf")
        for t in range(nkb):
            j = int(order[h, t])
            m_loc = float(logits[j * bk:(j + 1) * bk].max())
            skip = m_run != float("-inf") and (torch.tensor(m_loc, dtype=torch.float32) -
                                               torch.tensor(m_run, dtype=torch.float32)).item() < T
            assert int(res["skipped"][h, t]) == int(skip), (h, t)
            if not skip:
                m_run = max(m_run, m_loc)
    assert int(res["skipped"].sum()) > 0
