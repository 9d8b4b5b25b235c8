"""The seeded input generators (no method arithmetic lives here): what the
parity tests rely on them for.

- Integer-grid inputs, plain and structured, hold small integers only, so
  every pooled mean is exact in bf16 and every logit exact in fp32 -- the
  premise of the bit-exact comparisons.
- Generation is deterministic per seed, and replicas (ranks) differ.
- The paged form is a permutation of the logical cache.
- The dense causal FLOP counts (the numerator of the headline metric) are
  the closed form 4 * B * Hq * d * (number of causal query/key pairs).
"""
import torch

import synth


def _small(**kw):
    base = dict(name="t", wid=93, B=2, Hq=4, Hkv=2, Nq=512, Nkv=1024, bq=128, bk=64, stride=16,
                structured=True, n_needle=2)
    base.update(kw)
    return synth.Workload(**base)


def test_grid_values_are_small_integers():
    for structured in (False, True):
        inp = synth.generate(_small(structured=structured), grid=True)
        for t in (inp.q, inp.k, inp.v):
            x = t.double()
            assert torch.equal(x, x.round())
            assert x.abs().max().item() <= 6
        # pooled means of 16 integers are multiples of 1/16 below 8 in magnitude:
        # at most 8 significant bits, exact in bf16
        kp = inp.k.double().view(2, 2, -1, 16, 128).mean(3)
        assert torch.equal(kp.to(torch.bfloat16).double(), kp)
        # logits of such values stay far below 2^24: exact in fp32
        assert (inp.q.double().abs().sum(-1).max() * 6).item() < 2 ** 24


def test_structured_grid_has_dominant_keys():
    """The keys that carry the query direction (sinks and needle blocks) sit
    far above the rest: every row's maximum logit exceeds its median by more
    than 100 raw units, so blocks without them fall below the skip threshold
    of eps = 1e-4 (T = -104 at d = 128) once a dominant block is computed."""
    wl = _small(Nq=256, Nkv=256, B=1, Hq=2, Hkv=1)
    inp = synth.generate(wl, grid=True)
    s = inp.q[0, 0].double() @ inp.k[0, 0].double().T          # [256, 256]
    gap = s.max(1).values - s.median(1).values
    assert gap.min().item() > 100
    plain = synth.generate(wl.replace(structured=False), grid=True)
    s0 = plain.q[0, 0].double() @ plain.k[0, 0].double().T
    assert (s0.max(1).values - s0.median(1).values).max().item() < 100


def test_deterministic_and_rank_dependent():
    wl = _small()
    a, b = synth.generate(wl), synth.generate(wl)
    assert torch.equal(a.q, b.q) and torch.equal(a.k, b.k) and torch.equal(a.v, b.v)
    c = synth.generate(wl, rank=1)
    assert not torch.equal(a.q, c.q)


def test_paged_is_a_permutation_of_the_logical_cache():
    wl = _small(Nkv=1000)                                      # a partial last page
    inp = synth.generate(wl)
    pinp = synth._to_paged(wl.replace(paged=True), inp.q, inp.k, inp.v, wid=3)
    assert pinp.page_table.shape == (wl.B, wl.n_kblocks)
    assert sorted(pinp.page_table.flatten().tolist()) == list(range(wl.B * wl.n_kblocks))
    k, v = synth.logical_kv(pinp)
    assert torch.equal(k, inp.k) and torch.equal(v, inp.v)


def test_dense_causal_flops_closed_form():
    expect = {"single_head_2k": 1.07e9, "gqa_32k": 8.80e12, "gqa_128k": 140.7e12,
              "chunked_128k_paged": 8.66e12, "sweep_64k_b2": 70.4e12}
    for name, wl in synth.WORKLOADS.items():
        pairs = sum(min(wl.Nkv, wl.Nkv - wl.Nq + i + 1) for i in range(wl.Nq))
        assert wl.dense_causal_flops() == 4.0 * wl.B * wl.Hq * wl.d * pairs
        assert abs(wl.dense_causal_flops() / expect[name] - 1) < 5e-3, name


def test_planned_recipe_weakens_the_structure():
    """The "planned" recipe (query direction 2, needles 3 * ubar) draws the
    same noise as the default one and differs only by the structure terms:
    queries move by (16 - 2) * u_h, needle keys by 3 * (sqrt(d) - 1) * ubar_g."""
    wl = _small(Nq=1024, Nkv=1024, bk=128)
    a = synth.generate(wl)
    b = synth.generate(wl.replace(recipe="planned"))
    assert torch.equal(a.v, b.v)
    dq = (a.q.float() - b.q.float()).norm(dim=-1)
    assert abs(dq.mean().item() - 14.0) < 0.3          # |(16 - 2) u_h| = 14, up to bf16 rounding
    dk = (a.k.float() - b.k.float()).norm(dim=-1)
    assert dk[:, :, :4].abs().max().item() < 0.2       # sinks unchanged
    assert abs(dk.max().item() - 3.0 * (128 ** 0.5 - 1.0)) < 0.5
