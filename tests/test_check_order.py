"""cosa_check_order: the host-side check of a visit order before cosa_attend
(CoSA technical summary Sec. 2.1: the computation-order mask lists each
block a Q-block visits once; a duplicate would enter the softmax twice).
CPU only: the check runs on host memory, and the orders come from the oracle."""
import ctypes

import pytest
import torch

import block_sparse_attention_kap_b200 as cosa
import oracle
import synth

SHAPE = dict(B=1, Hq=2, Hkv=1, Nq=384, Nkv=640, bq=128, bk=64)


@pytest.fixture(scope="module")
def plan():
    wl = synth.Workload("check", 5, structured=True, **SHAPE)
    inp = synth.generate(wl, grid=True)
    ref = oracle.kap(inp, 0.5)
    shape = cosa.shape_of_workload(wl)
    nqb = cosa.cosa_num_qblocks(shape)
    km = ref["order"].shape[1]
    order = ref["order"].to(torch.int32).reshape(SHAPE["B"], SHAPE["Hq"], nqb, km).contiguous()
    count = ref["count"].to(torch.int32).reshape(SHAPE["B"], SHAPE["Hq"], nqb).contiguous()
    return shape, order, count


def _raw(shape, order, count, kmax):
    bad = ctypes.c_int64(123)
    st = cosa._lib.cosa_check_order(ctypes.byref(shape), ctypes.c_void_p(order.data_ptr()),
                                    ctypes.c_void_p(count.data_ptr()), kmax, ctypes.byref(bad))
    return st, bad.value


def test_oracle_plan_passes(plan):
    shape, order, count = plan
    assert cosa.cosa_check_order(shape, order, count) == 0
    assert _raw(shape, order, count, order.shape[-1]) == (0, 0)


def test_dense_order_passes(plan):
    shape, _, _ = plan
    nqb, nkb = cosa.cosa_num_qblocks(shape), cosa.cosa_num_kblocks(shape)
    off = SHAPE["Nkv"] - SHAPE["Nq"]
    n = [min(nkb, (off + min((i + 1) * SHAPE["bq"], SHAPE["Nq"]) - 1) // SHAPE["bk"] + 1) for i in range(nqb)]
    order = torch.full((1, SHAPE["Hq"], nqb, nkb), -1, dtype=torch.int32)
    for i in range(nqb):
        order[:, :, i, :n[i]] = torch.arange(n[i], dtype=torch.int32)
    count = torch.tensor(n, dtype=torch.int32).repeat(1, SHAPE["Hq"], 1)
    assert cosa.cosa_check_order(shape, order, count) == 0
    # one block beyond the causal limit of Q-block 0 is refused
    count2 = count.clone()
    order2 = order.clone()
    order2[0, 0, 0, n[0]] = n[0]
    count2[0, 0, 0] = n[0] + 1
    st, bad = _raw(shape, order2, count2, nkb)
    assert st == 1 and bad == n[0]


@pytest.mark.parametrize("kind", ["duplicate", "negative", "beyond_nkb", "non_causal"])
def test_bad_entry_is_located(plan, kind):
    shape, order, count = plan
    km = order.shape[-1]
    o = order.clone()
    flat_c = count.view(-1)
    row = next(r for r in range(flat_c.numel()) if flat_c[r] >= 2)
    I = row % cosa.cosa_num_qblocks(shape)
    off = SHAPE["Nkv"] - SHAPE["Nq"]
    n_vis = min(cosa.cosa_num_kblocks(shape), (off + min((I + 1) * SHAPE["bq"], SHAPE["Nq"]) - 1) // SHAPE["bk"] + 1)
    t = 1
    o.view(-1, km)[row, t] = {"duplicate": int(o.view(-1, km)[row, 0]), "negative": -1,
                              "beyond_nkb": cosa.cosa_num_kblocks(shape), "non_causal": n_vis}[kind]
    st, bad = _raw(shape, o, count, km)
    assert st == 1 and bad == row * km + t
    with pytest.raises(cosa.CosaError, match=f"row {row}, visit {t}"):
        cosa.cosa_check_order(shape, o, count)


@pytest.mark.parametrize("value", [-1, "kmax+1"])
def test_bad_count_is_located(plan, value):
    shape, order, count = plan
    km = order.shape[-1]
    c = count.clone()
    c.view(-1)[3] = km + 1 if value == "kmax+1" else value
    st, bad = _raw(shape, order, c, km)
    assert st == 1 and bad == -1 - 3
    with pytest.raises(cosa.CosaError, match="of row 3"):
        cosa.cosa_check_order(shape, order, c)


def test_entries_past_count_are_not_read(plan):
    shape, order, count = plan
    o = order.clone()
    km = o.shape[-1]
    flat_c = count.view(-1)
    row = next(r for r in range(flat_c.numel()) if flat_c[r] < km)
    o.view(-1, km)[row, int(flat_c[row]):] = 10 ** 6
    assert cosa.cosa_check_order(shape, o, count) == 0


def test_invalid_shape_and_kmax(plan):
    shape, order, count = plan
    assert _raw(shape, order, count, 0)[0] == 3
    bad_shape = cosa.make_shape(1, 3, 2, 384, 640, bq=128, bk=64)       # Hq % Hkv != 0
    assert _raw(bad_shape, order, count, order.shape[-1])[0] == 3
    with pytest.raises(cosa.CosaError):
        cosa.cosa_check_order(bad_shape, order, count)
