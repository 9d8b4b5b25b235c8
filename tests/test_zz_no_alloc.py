"""cosa_plan_static: the planning call for callers that cannot allocate.

Some callers cannot give the library a workspace: a serving engine that
reserves all device memory at start-up and passes kernels only the tensors
it owns, or a plug-in whose host framework keeps the allocator to itself.
cosa_plan_static serves them with scratch taken from a fixed array inside
the library.  These tests call it through the C ABI twice in a row, on two
different problems, and require exactly what cosa_plan returns with a
caller-provided workspace (same kernels on the same inputs: the integer
outputs and the scores must match bit for bit); a problem too large for the
fixed array must be refused before anything runs.

The file name sorts last so that a run stopping at the first failure has
already run every other test.
"""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cosa():
    import block_sparse_attention_kap_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def _plan_both_ways(cosa, inp, budget):
    wl = inp.wl
    shape = cosa.shape_of_workload(wl)
    m = cosa.CoSA(shape)
    q, k = inp.q.cuda(), inp.k.cuda()
    pt = inp.page_table.cuda() if inp.page_table is not None else None
    ref = m.plan(q, k, budget, page_table=pt, scores=True)
    order, count, hrm = m.alloc_plan(budget)
    order.fill_(-7)
    count.fill_(-7)
    score = torch.full_like(ref["block_score"], float("nan"))
    flags = torch.full_like(ref["hrm"], 7)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    cosa.cosa_plan_static(shape, q, k, pt, budget, order.shape[-1], order, count, hrm, score, flags, status)
    torch.cuda.synchronize()
    assert status.item() == 0 and m.device_status() == 0
    assert torch.equal(order, ref["order"])
    assert torch.equal(count, ref["count"])
    assert torch.equal(hrm, ref["hrm_count"])
    assert torch.equal(score, ref["block_score"])
    assert torch.equal(flags, ref["hrm"])


def test_static_scratch_plan_matches_workspace_plan_on_two_calls(cosa):
    # call 1: GQA layer, 8K tokens, structured inputs
    wl1 = synth.WORKLOADS["gqa_32k"].replace(name="gqa_8k", Hq=8, Hkv=2, Nq=8192, Nkv=8192, n_needle=4)
    assert cosa.cosa_plan_workspace_bytes(cosa.shape_of_workload(wl1)) <= cosa.STATIC_SCRATCH_BYTES
    _plan_both_ways(cosa, synth.generate(wl1), 0.1)
    # call 2: a different problem (a query chunk over a paged cache) reusing the same scratch
    wl2 = synth.WORKLOADS["chunked_128k_paged"].replace(name="chunk_16k", Nq=1024, Nkv=16384, n_needle=4)
    _plan_both_ways(cosa, synth.generate(wl2), 0.2)


def test_static_scratch_refuses_problems_larger_than_the_array(cosa):
    wl = synth.WORKLOADS["gqa_128k"]
    shape = cosa.shape_of_workload(wl)
    assert cosa.cosa_plan_workspace_bytes(shape) > cosa.STATIC_SCRATCH_BYTES
    km = cosa.cosa_kmax(shape, 0.1)
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(cosa.CosaError) as e:
        cosa.cosa_plan_static(shape, dummy.view(torch.bfloat16), dummy.view(torch.bfloat16), None, 0.1, km,
                              dummy, dummy)
    assert e.value.status == 4     # COSA_EWORKSPACE, before any launch
