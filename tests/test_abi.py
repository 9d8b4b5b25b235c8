"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/cosa.h declares, and its host logic (budget
arithmetic, threshold, argument validation) agrees with the oracle.  No
call here reaches a kernel launch."""
import ctypes
import math
import os
import re

import pytest

import oracle
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def cosa():
    import block_sparse_attention_kap_b200 as m
    return m


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "cosa.h")).read()
    return set(re.findall(r"COSA_API\s+[\w\s\*]+?\b(cosa_\w+)\s*\(", text))


def test_exports_every_declared_symbol(cosa):
    names = declared_symbols()
    assert len(names) >= 10
    for n in names:
        assert hasattr(cosa._lib, n), n
        assert n in cosa.EXPORTS


def test_version(cosa):
    assert cosa.cosa_version() == 101


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_kmax_and_blocks_match_oracle(cosa, name):
    wl = synth.WORKLOADS[name]
    s = cosa.shape_of_workload(wl)
    assert cosa.cosa_num_qblocks(s) == wl.n_qblocks
    assert cosa.cosa_num_kblocks(s) == wl.n_kblocks
    for beta in wl.budgets + (0.01, 0.333):
        assert cosa.cosa_kmax(s, beta) == oracle.kmax(wl, beta)
    assert cosa.cosa_plan_workspace_bytes(s) > 0


def test_skip_threshold_matches_oracle(cosa):
    for eps in (0.0, 1e-6, 1e-4, 0.05, 0.5):
        for d in (1, 64, 128):
            a, b = cosa.cosa_skip_threshold(eps, d), oracle.skip_threshold(eps, d)
            assert (a == b) or (math.isinf(a) and math.isinf(b))


def test_shape_validation(cosa):
    good = dict(B=1, Hq=4, Hkv=2, Nq=256, Nkv=512, d=128, bq=128, bk=64, stride=16)
    assert cosa.cosa_kmax(cosa.make_shape(**good), 0.1) > 0
    bad = [dict(d=64), dict(Hkv=3), dict(Nkv=128), dict(bq=32), dict(stride=3), dict(stride=64),
           dict(Nq=250)]
    for b in bad:
        kw = dict(good)
        kw.update(b)
        assert cosa.cosa_kmax(cosa.make_shape(**kw), 0.1) == -1, b
    s = cosa.make_shape(**good)
    for beta in (0.0, -0.1, 1.5, float("nan")):
        assert cosa.cosa_kmax(s, beta) == -1


def _raw_plan(cosa, shape, q=1 << 20, k=1 << 20, budget=0.1, kmax=64, order=1 << 20, count=1 << 20,
              ws=1 << 20, ws_bytes=None, pt=None):
    lib = cosa._lib
    ws_bytes = cosa.cosa_plan_workspace_bytes(shape) if ws_bytes is None else ws_bytes
    return lib.cosa_plan(ctypes.byref(shape), q, k, pt, budget, kmax, order, count, None, None, None, ws,
                         ws_bytes, None, None)


def test_plan_argument_errors_return_before_launch(cosa):
    s = cosa.make_shape(1, 4, 2, 256, 512, 128, 128, 64, 16)
    km = cosa.cosa_kmax(s, 0.1)
    assert _raw_plan(cosa, s, q=None, kmax=km) == 1            # EINVAL
    assert _raw_plan(cosa, s, kmax=km - 1) == 1                # kmax too small
    assert _raw_plan(cosa, s, budget=0.0, kmax=km) == 1
    assert _raw_plan(cosa, s, q=(1 << 20) + 2, kmax=km) == 2   # EALIGN
    assert _raw_plan(cosa, s, kmax=km, ws_bytes=16) == 4        # EWORKSPACE
    assert _raw_plan(cosa, s, kmax=km, ws=None) == 4
    bad = cosa.make_shape(1, 4, 2, 256, 512, 96, 128, 64, 16)
    assert _raw_plan(cosa, bad, kmax=km) == 6                   # EUNSUPPORTED (d)
    paged = cosa.make_shape(1, 4, 2, 256, 512, 128, 128, 64, 16, True, 8)
    assert _raw_plan(cosa, paged, kmax=km) == 1                 # paged without a page table
    empty = cosa.make_shape(1, 4, 2, 0, 512, 128, 128, 64, 16)
    assert _raw_plan(cosa, empty, q=None, k=None, order=None, count=None, ws=None, kmax=0) == 0


def test_plan_chunk_argument_errors_return_before_launch(cosa):
    lib = cosa._lib
    s = cosa.make_shape(1, 4, 2, 256, 1024, 128, 128, 64, 16)     # 64 pooled keys per head
    km = cosa.cosa_kmax(s, 0.1)
    P = 1 << 20
    ws_bytes = cosa.cosa_plan_workspace_bytes(s)

    def call(cache=P, cap=64, valid=48, q=P, kmax=km, ws_bytes=ws_bytes, shape=s):
        return lib.cosa_plan_chunk(ctypes.byref(shape), q, P, None, cache, cap, valid, 0.1, kmax, P, P, None,
                                   None, None, P, ws_bytes, None, None)
    assert call(cache=None) == 1                  # EINVAL: no cache
    assert call(cap=63) == 1                      # capacity below Nkv / stride
    assert call(valid=-1) == 1
    assert call(valid=65) == 1                    # more valid rows than keys
    assert call(cache=P + 8) == 2                 # EALIGN
    assert call(q=None) == 1
    assert call(kmax=km - 1) == 1
    assert call(ws_bytes=256) == 4                # EWORKSPACE
    assert call(shape=cosa.make_shape(1, 4, 2, 256, 1000, 128, 128, 64, 16)) == 3
    assert call(shape=cosa.make_shape(1, 4, 2, 0, 1024, 128, 128, 64, 16), q=None, cache=None) == 0


def test_block_union_argument_errors_return_before_launch(cosa):
    lib = cosa._lib
    s = cosa.make_shape(1, 4, 2, 256, 768, 128, 128, 128, 16)      # nKB = 6; the last Q-block sees 6
    P = 1 << 20

    def call(order=P, count=P, kmax=4, table=P, tlen=P, uo=P, uc=P, ukmax=6, shape=s):
        return lib.cosa_block_union(ctypes.byref(shape), order, count, kmax, table, tlen, uo, uc, ukmax, None)
    assert call(table=None) == 1
    assert call(tlen=None) == 1
    assert call(order=None) == 1
    assert call(kmax=-1) == 1
    assert call(ukmax=5) == 1                     # too short for the last Q-block's visible blocks
    assert call(uc=None) == 1                     # union_order without union_count
    assert call(shape=cosa.make_shape(1, 4, 3, 256, 768, 128, 128, 128, 16)) == 3
    assert call(shape=cosa.make_shape(0, 4, 2, 256, 768, 128, 128, 128, 16), table=None) == 0


def test_decode_plan_argument_errors_return_before_launch(cosa):
    lib = cosa._lib
    s = cosa.make_shape(1, 4, 2, 1, 1024, 128, 128, 128, 16)        # one query after 1023 keys; nKB = 8
    P = 1 << 20

    def call(q=P, k=P, cache=P, cap=64, valid=0, budget=0.25, kmax=2, order=P, count=P, shape=s):
        return lib.cosa_decode_plan(ctypes.byref(shape), q, k, None, cache, cap, valid, budget, kmax, order,
                                    count, None, None, None, None)
    assert call(shape=cosa.make_shape(1, 4, 2, 2, 1024, 128, 128, 128, 16)) == 3     # Nq != 1
    assert call(shape=cosa.make_shape(1, 4, 2, 1, 1000, 128, 128, 128, 16)) == 6     # Nkv not a stride multiple
    assert call(cache=None) == 1
    assert call(q=None) == 1
    assert call(budget=0.0) == 1
    assert call(kmax=1) == 1                      # ceil(8 * 0.25) = 2 blocks kept
    assert call(cap=63) == 1
    assert call(valid=65) == 1
    assert call(q=P + 4) == 2
    assert call(shape=cosa.make_shape(0, 4, 2, 1, 1024, 128, 128, 128, 16), q=None) == 0


def test_attend_argument_errors_return_before_launch(cosa):
    lib = cosa._lib
    s = cosa.make_shape(1, 4, 2, 256, 512, 128, 128, 64, 16)
    P = 1 << 20

    def call(q=P, k=P, v=P, out=P, order=P, count=P, kmax=8, eps=1e-4, shape=s):
        return lib.cosa_attend(ctypes.byref(shape), q, k, v, None, order, count, kmax, eps, out, None, None,
                               None, None)
    assert call(v=None) == 1
    assert call(out=None) == 1
    assert call(kmax=0) == 1
    assert call(eps=1.0) == 1
    assert call(eps=-0.5) == 1
    assert call(out=P + 8) == 2
    assert call(shape=cosa.make_shape(1, 4, 3, 256, 512, 128, 128, 64, 16)) == 3
    assert call(shape=cosa.make_shape(1, 4, 2, 0, 512, 128, 128, 64, 16), q=None) == 0


def test_wait_timeout_hook_argument_errors_return_before_launch(cosa):
    lib = cosa._lib
    s = cosa.make_shape(1, 4, 2, 256, 512, 128, 128, 64, 16)
    P = 1 << 20

    def call(status=P, limit=10 ** 6):
        return lib.cosa_test_attend_wait_timeout(ctypes.byref(s), P, P, P, None, P, P, 8, P, status, limit, None)
    assert call(status=None) == 1
    assert call(limit=10) == 1
    assert call(limit=2 * 10 ** 9) == 1
    # the same validation as cosa_attend before any launch: a misaligned output
    assert lib.cosa_test_attend_wait_timeout(ctypes.byref(s), P, P, P, None, P, P, 8, P + 8, P, 10 ** 6,
                                             None) == 2


def test_status_strings(cosa):
    for code in range(7):
        assert cosa.cosa_status_string(code).startswith("COSA_")
