"""Python binding of the CoSA B200 library (libcosa.so, C ABI in include/cosa.h).

Argument marshalling only: torch tensors supply device memory and the
current CUDA stream; every step of KAP (pooling, scoring, sorting) and OSK
runs in the library's CUDA kernels.  There is no CPU fallback: importing
this package without the built library raises ImportError, and every call
checks the returned cosa_status.

CoSA: "Accelerating Long-Context Inference via Proxy-Kernel Co-Designed
Sparse Attention" (gist.science/paper/2607.25291), technical summary
Sec. 2.2 (Kernel-Aware Proxy) and Sec. 2.3 (Ordered-Skipping Kernel).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcosa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m block_sparse_attention_kap_b200.build` "
                      "(the CoSA path has no CPU fallback)")

_lib = ctypes.CDLL(LIB_PATH)


class cosa_shape(ctypes.Structure):
    """Mirror of the C struct cosa_shape."""
    _fields_ = [(n, ctypes.c_int) for n in
                ("B", "Hq", "Hkv", "Nq", "Nkv", "d", "bq", "bk", "stride", "paged", "num_pages")]


STATUS = {0: "COSA_OK", 1: "COSA_EINVAL", 2: "COSA_EALIGN", 3: "COSA_ESHAPE", 4: "COSA_EWORKSPACE",
          5: "COSA_ECUDA", 6: "COSA_EUNSUPPORTED"}


class CosaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.cosa_status_string(status).decode()
        super().__init__(f"{where}: {msg}")


_P = ctypes.c_void_p
_S = ctypes.POINTER(cosa_shape)
_lib.cosa_num_qblocks.argtypes = [_S]
_lib.cosa_num_kblocks.argtypes = [_S]
_lib.cosa_kmax.argtypes = [_S, ctypes.c_double]
_lib.cosa_plan_workspace_bytes.argtypes = [_S]
_lib.cosa_plan_workspace_bytes.restype = ctypes.c_size_t
_lib.cosa_plan.argtypes = [_S, _P, _P, _P, ctypes.c_double, ctypes.c_int, _P, _P, _P, _P, _P, _P,
                           ctypes.c_size_t, _P, _P]
_lib.cosa_plan_chunk.argtypes = [_S, _P, _P, _P, _P, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int,
                                 _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P, _P]
_lib.cosa_dense_order.argtypes = [_S, ctypes.c_int, _P, _P, _P]
_lib.cosa_block_union.argtypes = [_S, _P, _P, ctypes.c_int, _P, _P, _P, _P, ctypes.c_int, _P]
_lib.cosa_decode_plan.argtypes = [_S, _P, _P, _P, _P, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int,
                                  _P, _P, _P, _P, _P, _P]
_lib.cosa_plan_static.argtypes = [_S, _P, _P, _P, ctypes.c_double, ctypes.c_int, _P, _P, _P, _P, _P, _P, _P]
_lib.cosa_attend.argtypes = [_S, _P, _P, _P, _P, _P, _P, ctypes.c_int, ctypes.c_double, _P, _P, _P, _P, _P]
_lib.cosa_decode_attend_workspace_bytes.argtypes = [_S, ctypes.c_int]
_lib.cosa_decode_attend_workspace_bytes.restype = ctypes.c_size_t
_lib.cosa_decode_attend.argtypes = [_S, _P, _P, _P, _P, _P, _P, ctypes.c_int, ctypes.c_double, _P, _P, _P, _P,
                                    ctypes.c_size_t, _P]
_lib.cosa_attend_group.argtypes = [_S, _P, _P, _P, _P, _P, _P, ctypes.c_int, ctypes.c_double, _P, _P, _P, _P, _P]
_lib.cosa_test_attend_wait_timeout.argtypes = [_S, _P, _P, _P, _P, _P, _P, ctypes.c_int, _P, _P, ctypes.c_uint64, _P]
_lib.cosa_check_order.argtypes = [_S, _P, _P, ctypes.c_int, ctypes.POINTER(ctypes.c_int64)]
_lib.cosa_skip_threshold.argtypes = [ctypes.c_double, ctypes.c_int]
_lib.cosa_skip_threshold.restype = ctypes.c_float
_lib.cosa_status_string.argtypes = [ctypes.c_int]
_lib.cosa_status_string.restype = ctypes.c_char_p

EXPORTS = ("cosa_num_qblocks", "cosa_num_kblocks", "cosa_kmax", "cosa_plan_workspace_bytes", "cosa_plan",
           "cosa_dense_order", "cosa_attend", "cosa_skip_threshold", "cosa_status_string", "cosa_version",
           "cosa_plan_static", "cosa_plan_chunk", "cosa_block_union", "cosa_decode_plan",
           "cosa_test_attend_wait_timeout", "cosa_attend_group", "cosa_decode_attend",
           "cosa_decode_attend_workspace_bytes", "cosa_check_order")
DEV_TIMEOUT_TMA, DEV_TIMEOUT_MMA, DEV_TIMEOUT_PIPE = 0x100, 0x200, 0x300
STATIC_SCRATCH_BYTES = 64 << 20


def make_shape(B, Hq, Hkv, Nq, Nkv, d=128, bq=128, bk=128, stride=16, paged=False, num_pages=0) -> cosa_shape:
    return cosa_shape(B, Hq, Hkv, Nq, Nkv, d, bq, bk, stride, 1 if paged else 0, num_pages)


def _ptr(t: Optional[torch.Tensor], name: str, dtype=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status: int, where: str):
    if status != 0:
        raise CosaError(status, where)


# ----------------------------------------------------------------- same names as the C ABI

def cosa_num_qblocks(shape: cosa_shape) -> int:
    return _lib.cosa_num_qblocks(ctypes.byref(shape))


def cosa_num_kblocks(shape: cosa_shape) -> int:
    return _lib.cosa_num_kblocks(ctypes.byref(shape))


def cosa_kmax(shape: cosa_shape, budget: float) -> int:
    return _lib.cosa_kmax(ctypes.byref(shape), budget)


def cosa_plan_workspace_bytes(shape: cosa_shape) -> int:
    return _lib.cosa_plan_workspace_bytes(ctypes.byref(shape))


def cosa_skip_threshold(eps: float, d: int = 128) -> float:
    return _lib.cosa_skip_threshold(eps, d)


def cosa_status_string(status: int) -> str:
    return _lib.cosa_status_string(status).decode()


def cosa_version() -> int:
    return _lib.cosa_version()


def cosa_check_order(shape: cosa_shape, order, count, kmax: Optional[int] = None) -> int:
    """Check a visit order on the host before cosa_attend: order [B, Hq, nQB,
    kmax] and count [B, Hq, nQB] int32 (copied to host memory if they are on
    the GPU).  Returns 0 when every count is in [0, kmax] and every visited
    block is causally visible to its Q-block and appears once in its row;
    otherwise raises CosaError naming the first bad row and entry."""
    if order.dtype != torch.int32 or count.dtype != torch.int32:
        raise ValueError("order and count must be int32")
    km = order.shape[-1] if kmax is None else kmax
    o = order.detach().to("cpu").contiguous()
    c = count.detach().to("cpu").contiguous()
    if o.numel() != c.numel() * km:
        raise ValueError(f"order has {o.numel()} entries, count {c.numel()} rows of kmax {km}")
    bad = ctypes.c_int64(0)
    st = _lib.cosa_check_order(ctypes.byref(shape), ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(c.data_ptr()),
                               km, ctypes.byref(bad))
    if st == 1 and bad.value < 0:
        raise CosaError(st, f"cosa_check_order: count {int(c.view(-1)[-1 - bad.value])} of row {-1 - bad.value}")
    if st == 1:
        raise CosaError(st, f"cosa_check_order: row {bad.value // km}, visit {bad.value % km} "
                            f"(block {int(o.view(-1)[bad.value])})")
    _check(st, "cosa_check_order")
    return 0


def cosa_plan(shape: cosa_shape, q, k, page_table, budget: float, kmax: int, order, count,
              hrm_count=None, block_score=None, hrm_flags=None, workspace=None, dev_status=None,
              stream=None) -> None:
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.cosa_plan(ctypes.byref(shape), _ptr(q, "q", torch.bfloat16), _ptr(k, "k", torch.bfloat16),
                          _ptr(page_table, "page_table", torch.int32), budget, kmax,
                          _ptr(order, "order", torch.int32), _ptr(count, "count", torch.int32),
                          _ptr(hrm_count, "hrm_count", torch.int32), _ptr(block_score, "block_score", torch.float32),
                          _ptr(hrm_flags, "hrm_flags", torch.uint8), _ptr(workspace, "workspace"), ws_bytes,
                          _ptr(dev_status, "dev_status", torch.int32), _stream(stream)), "cosa_plan")


def cosa_plan_chunk(shape: cosa_shape, q, k, page_table, kp_cache, kp_valid: int, budget: float, kmax: int,
                    order, count, hrm_count=None, block_score=None, hrm_flags=None, workspace=None,
                    dev_status=None, stream=None) -> None:
    """cosa_plan for one prefill chunk: kp_cache [B, Hkv, capacity, d] bf16
    keeps the pooled keys across chunks; its rows below kp_valid are reused,
    the rest are pooled from k and written back."""
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    if kp_cache is not None and kp_cache.dim() != 4:
        raise ValueError("kp_cache must be [B, Hkv, capacity, d]")
    cap = kp_cache.shape[2] if kp_cache is not None else 0
    _check(_lib.cosa_plan_chunk(ctypes.byref(shape), _ptr(q, "q", torch.bfloat16), _ptr(k, "k", torch.bfloat16),
                                _ptr(page_table, "page_table", torch.int32),
                                _ptr(kp_cache, "kp_cache", torch.bfloat16), cap, kp_valid, budget, kmax,
                                _ptr(order, "order", torch.int32), _ptr(count, "count", torch.int32),
                                _ptr(hrm_count, "hrm_count", torch.int32),
                                _ptr(block_score, "block_score", torch.float32),
                                _ptr(hrm_flags, "hrm_flags", torch.uint8), _ptr(workspace, "workspace"), ws_bytes,
                                _ptr(dev_status, "dev_status", torch.int32), _stream(stream)), "cosa_plan_chunk")


def cosa_plan_static(shape: cosa_shape, q, k, page_table, budget: float, kmax: int, order, count,
                     hrm_count=None, block_score=None, hrm_flags=None, dev_status=None, stream=None) -> None:
    """cosa_plan for callers that cannot supply a workspace: the scratch is a
    fixed STATIC_SCRATCH_BYTES array inside the library (shared by all calls;
    calls that may overlap on the GPU race on it)."""
    _check(_lib.cosa_plan_static(ctypes.byref(shape), _ptr(q, "q", torch.bfloat16), _ptr(k, "k", torch.bfloat16),
                                 _ptr(page_table, "page_table", torch.int32), budget, kmax,
                                 _ptr(order, "order", torch.int32), _ptr(count, "count", torch.int32),
                                 _ptr(hrm_count, "hrm_count", torch.int32),
                                 _ptr(block_score, "block_score", torch.float32),
                                 _ptr(hrm_flags, "hrm_flags", torch.uint8),
                                 _ptr(dev_status, "dev_status", torch.int32), _stream(stream)), "cosa_plan_static")


def cosa_dense_order(shape: cosa_shape, kmax: int, order, count, stream=None) -> None:
    _check(_lib.cosa_dense_order(ctypes.byref(shape), kmax, _ptr(order, "order", torch.int32),
                                 _ptr(count, "count", torch.int32), _stream(stream)), "cosa_dense_order")


def cosa_decode_plan(shape: cosa_shape, q, k, page_table, kp_cache, kp_valid: int, budget: float, kmax: int,
                     order, count, hrm_count=None, block_score=None, hrm_flags=None, stream=None) -> None:
    """The proxy for one decode step (shape.Nq == 1): q [B, Hq, 1, d]; the
    pooled keys come from kp_cache [B, Hkv, capacity, d] (rows below
    kp_valid reused, the rest pooled from k first)."""
    if kp_cache is not None and kp_cache.dim() != 4:
        raise ValueError("kp_cache must be [B, Hkv, capacity, d]")
    cap = kp_cache.shape[2] if kp_cache is not None else 0
    _check(_lib.cosa_decode_plan(ctypes.byref(shape), _ptr(q, "q", torch.bfloat16), _ptr(k, "k", torch.bfloat16),
                                 _ptr(page_table, "page_table", torch.int32),
                                 _ptr(kp_cache, "kp_cache", torch.bfloat16), cap, kp_valid, budget, kmax,
                                 _ptr(order, "order", torch.int32), _ptr(count, "count", torch.int32),
                                 _ptr(hrm_count, "hrm_count", torch.int32),
                                 _ptr(block_score, "block_score", torch.float32),
                                 _ptr(hrm_flags, "hrm_flags", torch.uint8), _stream(stream)), "cosa_decode_plan")


def cosa_block_union(shape: cosa_shape, order, count, kmax: int, table, table_len, union_order=None,
                     union_count=None, stream=None) -> None:
    union_kmax = union_order.shape[-1] if union_order is not None else 0
    _check(_lib.cosa_block_union(ctypes.byref(shape), _ptr(order, "order", torch.int32),
                                 _ptr(count, "count", torch.int32), kmax, _ptr(table, "table", torch.int32),
                                 _ptr(table_len, "table_len", torch.int32),
                                 _ptr(union_order, "union_order", torch.int32),
                                 _ptr(union_count, "union_count", torch.int32), union_kmax, _stream(stream)),
           "cosa_block_union")


def cosa_attend(shape: cosa_shape, q, k, v, page_table, order, count, kmax: int, skip_eps: float, out,
                lse=None, skip_bits=None, dev_status=None, stream=None) -> None:
    _check(_lib.cosa_attend(ctypes.byref(shape), _ptr(q, "q", torch.bfloat16), _ptr(k, "k", torch.bfloat16),
                            _ptr(v, "v", torch.bfloat16), _ptr(page_table, "page_table", torch.int32),
                            _ptr(order, "order", torch.int32), _ptr(count, "count", torch.int32), kmax, skip_eps,
                            _ptr(out, "out", torch.bfloat16), _ptr(lse, "lse", torch.float32),
                            _ptr(skip_bits, "skip_bits", torch.int32), _ptr(dev_status, "dev_status", torch.int32),
                            _stream(stream)), "cosa_attend")


def cosa_decode_attend_workspace_bytes(shape: cosa_shape, kmax: int) -> int:
    return _lib.cosa_decode_attend_workspace_bytes(ctypes.byref(shape), kmax)


def cosa_decode_attend(shape: cosa_shape, q, k, v, page_table, order, count, kmax: int, skip_eps: float, out,
                       lse=None, skip_bits=None, workspace=None, stream=None) -> None:
    """The attention of one decode step (shape.Nq == 1): OSK on the single
    query row of each head, with memory-bound kernels (parallel logits, a
    prefix-max scan for the skip decisions, parallel P.V)."""
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.cosa_decode_attend(ctypes.byref(shape), _ptr(q, "q", torch.bfloat16), _ptr(k, "k", torch.bfloat16),
                                   _ptr(v, "v", torch.bfloat16), _ptr(page_table, "page_table", torch.int32),
                                   _ptr(order, "order", torch.int32), _ptr(count, "count", torch.int32), kmax,
                                   skip_eps, _ptr(out, "out", torch.bfloat16), _ptr(lse, "lse", torch.float32),
                                   _ptr(skip_bits, "skip_bits", torch.int32), _ptr(workspace, "workspace"), ws_bytes,
                                   _stream(stream)), "cosa_decode_attend")


def cosa_attend_group(shape: cosa_shape, q, k, v, page_table, order, count, kmax: int, skip_eps: float, out,
                      lse=None, skip_bits=None, dev_status=None, stream=None) -> None:
    """OSK with one visit order per (batch, kv-head, Q-block) shared by the
    group's query heads: order [B, Hkv, nQB, kmax], count [B, Hkv, nQB]."""
    _check(_lib.cosa_attend_group(ctypes.byref(shape), _ptr(q, "q", torch.bfloat16), _ptr(k, "k", torch.bfloat16),
                                  _ptr(v, "v", torch.bfloat16), _ptr(page_table, "page_table", torch.int32),
                                  _ptr(order, "order", torch.int32), _ptr(count, "count", torch.int32), kmax,
                                  skip_eps, _ptr(out, "out", torch.bfloat16), _ptr(lse, "lse", torch.float32),
                                  _ptr(skip_bits, "skip_bits", torch.int32),
                                  _ptr(dev_status, "dev_status", torch.int32), _stream(stream)),
           "cosa_attend_group")


def cosa_test_attend_wait_timeout(shape: cosa_shape, q, k, v, page_table, order, count, kmax: int, out,
                                  dev_status, wait_limit_ns: int, stream=None) -> None:
    """Failure-detection test hook: cosa_attend's kernel with one wait per
    CTA that nothing completes, so every bounded wait gives up after
    wait_limit_ns and the kernel reports DEV_TIMEOUT_PIPE in dev_status."""
    _check(_lib.cosa_test_attend_wait_timeout(ctypes.byref(shape), _ptr(q, "q", torch.bfloat16),
                                              _ptr(k, "k", torch.bfloat16), _ptr(v, "v", torch.bfloat16),
                                              _ptr(page_table, "page_table", torch.int32),
                                              _ptr(order, "order", torch.int32), _ptr(count, "count", torch.int32),
                                              kmax, _ptr(out, "out", torch.bfloat16),
                                              _ptr(dev_status, "dev_status", torch.int32), wait_limit_ns,
                                              _stream(stream)), "cosa_test_attend_wait_timeout")


# ----------------------------------------------------------------- convenience (allocation via torch)

class CoSA:
    """Holds a shape and the KAP workspace; allocates outputs with torch.

    plan(q, k, budget)           -> order [B,Hq,nQB,kmax], count, hrm_count
    attend(q, k, v, order, count, eps) -> out [B,Hq,Nq,d] (+ lse, skip bits)
    dense(q, k, v)               -> out of the dense causal path
    """

    def __init__(self, shape: cosa_shape, device="cuda"):
        self.shape = shape
        self.device = torch.device(device)
        self.nqb = cosa_num_qblocks(shape)
        self.nkb = cosa_num_kblocks(shape)
        if self.nqb < 0:
            raise CosaError(3, "shape")
        self._ws = None
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)

    def workspace(self) -> torch.Tensor:
        if self._ws is None:
            nbytes = cosa_plan_workspace_bytes(self.shape)
            if nbytes == 0:
                raise CosaError(6, "cosa_plan_workspace_bytes")
            self._ws = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        return self._ws

    def alloc_plan(self, budget: float):
        s = self.shape
        km = max(cosa_kmax(s, budget), 1)
        order = torch.empty(s.B, s.Hq, self.nqb, km, dtype=torch.int32, device=self.device)
        count = torch.empty(s.B, s.Hq, self.nqb, dtype=torch.int32, device=self.device)
        hrm = torch.empty(s.B, s.Hq, self.nqb, dtype=torch.int32, device=self.device)
        return order, count, hrm

    def plan(self, q, k, budget: float, page_table=None, out=None, scores: bool = False, stream=None):
        order, count, hrm = out if out is not None else self.alloc_plan(budget)
        bs = hf = None
        if scores:
            s = self.shape
            bs = torch.empty(s.B, s.Hq, self.nqb, self.nkb, dtype=torch.float32, device=self.device)
            hf = torch.empty(s.B, s.Hq, self.nqb, self.nkb, dtype=torch.uint8, device=self.device)
        cosa_plan(self.shape, q, k, page_table, budget, order.shape[-1], order, count, hrm, bs, hf,
                  self.workspace(), self.status, stream)
        res = dict(order=order, count=count, hrm_count=hrm)
        if scores:
            res.update(block_score=bs, hrm=hf)
        return res

    def plan_chunk(self, q, k, budget: float, kp_cache, kp_valid: int, page_table=None, out=None,
                   scores: bool = False, stream=None):
        """plan() for one chunk of a chunked prefill, reusing the pooled keys
        kept in kp_cache (rows below kp_valid) and pooling only the rest."""
        order, count, hrm = out if out is not None else self.alloc_plan(budget)
        bs = hf = None
        if scores:
            s = self.shape
            bs = torch.empty(s.B, s.Hq, self.nqb, self.nkb, dtype=torch.float32, device=self.device)
            hf = torch.empty(s.B, s.Hq, self.nqb, self.nkb, dtype=torch.uint8, device=self.device)
        cosa_plan_chunk(self.shape, q, k, page_table, kp_cache, kp_valid, budget, order.shape[-1], order, count,
                        hrm, bs, hf, self.workspace(), self.status, stream)
        res = dict(order=order, count=count, hrm_count=hrm)
        if scores:
            res.update(block_score=bs, hrm=hf)
        return res

    def decode_plan(self, q, k, budget: float, kp_cache, kp_valid: int, page_table=None, scores: bool = False,
                    stream=None):
        """The proxy for one decode step (shape.Nq == 1)."""
        s = self.shape
        km = self.nkb                      # row stride of order: room for every block; count says how many
        order = torch.empty(s.B, s.Hq, 1, km, dtype=torch.int32, device=self.device)
        count = torch.empty(s.B, s.Hq, 1, dtype=torch.int32, device=self.device)
        hrm = torch.empty(s.B, s.Hq, 1, dtype=torch.int32, device=self.device)
        bs = hf = None
        if scores:
            bs = torch.empty(s.B, s.Hq, 1, self.nkb, dtype=torch.float32, device=self.device)
            hf = torch.empty(s.B, s.Hq, 1, self.nkb, dtype=torch.uint8, device=self.device)
        cosa_decode_plan(s, q, k, page_table, kp_cache, kp_valid, budget, km, order, count, hrm, bs, hf, stream)
        res = dict(order=order, count=count, hrm_count=hrm)
        if scores:
            res.update(block_score=bs, hrm=hf)
        return res

    def decode_attend(self, q, k, v, order, count, eps: float, page_table=None, out=None, lse: bool = False,
                      skip_bits: bool = False, stream=None):
        """The attention of one decode step (shape.Nq == 1) with the decode
        kernels: order [B, Hq, 1, kmax], count [B, Hq, 1]."""
        s = self.shape
        km = order.shape[-1]
        if out is None:
            out = torch.empty(s.B, s.Hq, 1, s.d, dtype=torch.bfloat16, device=self.device)
        lse_t = torch.empty(s.B, s.Hq, 1, dtype=torch.float32, device=self.device) if lse else None
        sb = torch.empty(s.B, s.Hq, 1, (km + 31) // 32, dtype=torch.int32, device=self.device) if skip_bits else None
        nbytes = cosa_decode_attend_workspace_bytes(s, km)
        if getattr(self, "_dws", None) is None or self._dws.numel() < nbytes:
            self._dws = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        cosa_decode_attend(s, q, k, v, page_table, order, count, km, eps, out, lse_t, sb, self._dws, stream)
        return dict(out=out, lse=lse_t, skip_bits=sb)

    def block_union(self, order, count, expand: bool = True, stream=None):
        """Per-(batch, kv-head) union of a selection over the Q-blocks and the
        heads of each group; with expand, also the causally visible prefix
        of the table per Q-block as an order for attend()."""
        s = self.shape
        table = torch.empty(s.B, s.Hkv, self.nkb, dtype=torch.int32, device=self.device)
        table_len = torch.empty(s.B, s.Hkv, dtype=torch.int32, device=self.device)
        uo = uc = None
        if expand:
            uo = torch.empty(s.B, s.Hq, self.nqb, self.nkb, dtype=torch.int32, device=self.device)
            uc = torch.empty(s.B, s.Hq, self.nqb, dtype=torch.int32, device=self.device)
        cosa_block_union(s, order, count, order.shape[-1], table, table_len, uo, uc, stream)
        return dict(table=table, table_len=table_len, order=uo, count=uc)

    def dense_order(self, stream=None):
        s = self.shape
        order = torch.empty(s.B, s.Hq, self.nqb, self.nkb, dtype=torch.int32, device=self.device)
        count = torch.empty(s.B, s.Hq, self.nqb, dtype=torch.int32, device=self.device)
        cosa_dense_order(s, self.nkb, order, count, stream)
        return order, count

    def attend(self, q, k, v, order, count, eps: float, page_table=None, out=None, lse: bool = False,
               skip_bits: bool = False, stream=None):
        s = self.shape
        km = order.shape[-1]
        if out is None:
            out = torch.empty(s.B, s.Hq, s.Nq, s.d, dtype=torch.bfloat16, device=self.device)
        lse_t = torch.empty(s.B, s.Hq, s.Nq, dtype=torch.float32, device=self.device) if lse else None
        sb = torch.empty(s.B, s.Hq, self.nqb, (km + 31) // 32, dtype=torch.int32, device=self.device) \
            if skip_bits else None
        cosa_attend(s, q, k, v, page_table, order, count, km, eps, out, lse_t, sb, self.status, stream)
        return dict(out=out, lse=lse_t, skip_bits=sb)

    def dense(self, q, k, v, page_table=None, stream=None, group: bool = False, **kw):
        """The dense path: every causal block, eps 0.  group=True runs it
        through attend_group (one shared order per GQA group)."""
        if group:
            order, count = self.dense_order_group(stream)
            return self.attend_group(q, k, v, order, count, 0.0, page_table=page_table, stream=stream, **kw)
        order, count = self.dense_order(stream)
        return self.attend(q, k, v, order, count, 0.0, page_table=page_table, stream=stream, **kw)

    def dense_order_group(self, stream=None):
        """The dense path's order with one row per (b, kv-head, Q-block)."""
        s = self.shape
        gs = make_shape(s.B, s.Hkv, s.Hkv, s.Nq, s.Nkv, s.d, s.bq, s.bk, s.stride, bool(s.paged), s.num_pages)
        order = torch.empty(s.B, s.Hkv, self.nqb, self.nkb, dtype=torch.int32, device=self.device)
        count = torch.empty(s.B, s.Hkv, self.nqb, dtype=torch.int32, device=self.device)
        cosa_dense_order(gs, self.nkb, order, count, stream)
        return order, count

    def attend_group(self, q, k, v, order, count, eps: float, page_table=None, out=None, lse: bool = False,
                     skip_bits: bool = False, stream=None):
        """attend() with one order per (b, kv-head, Q-block): order
        [B, Hkv, nQB, kmax], count [B, Hkv, nQB]."""
        s = self.shape
        km = order.shape[-1]
        if out is None:
            out = torch.empty(s.B, s.Hq, s.Nq, s.d, dtype=torch.bfloat16, device=self.device)
        lse_t = torch.empty(s.B, s.Hq, s.Nq, dtype=torch.float32, device=self.device) if lse else None
        sb = torch.empty(s.B, s.Hq, self.nqb, (km + 31) // 32, dtype=torch.int32, device=self.device) \
            if skip_bits else None
        cosa_attend_group(s, q, k, v, page_table, order, count, km, eps, out, lse_t, sb, self.status, stream)
        return dict(out=out, lse=lse_t, skip_bits=sb)

    def device_status(self) -> int:
        return int(self.status.item())

    def check_plan(self, order, count) -> None:
        """cosa_check_order on this shape: raises CosaError at the first visit
        a caller-edited order must not make (a block visited twice, one its
        Q-block cannot see, a count outside [0, kmax])."""
        cosa_check_order(self.shape, order, count)


def shape_of_workload(wl) -> cosa_shape:
    return make_shape(wl.B, wl.Hq, wl.Hkv, wl.Nq, wl.Nkv, wl.d, wl.bq, wl.bk, wl.stride, wl.paged,
                      wl.num_pages if wl.paged else 0)


def unpack_skip_bits(bits: torch.Tensor, kmax: int) -> torch.Tensor:
    """[..., words] int32 -> [..., kmax] uint8 (1 = skipped in-kernel)."""
    w = bits.to(torch.int64) & 0xFFFFFFFF
    shifts = torch.arange(32, device=bits.device, dtype=torch.int64)
    b = (w.unsqueeze(-1) >> shifts) & 1
    return b.reshape(*bits.shape[:-1], -1)[..., :kmax].to(torch.uint8)
