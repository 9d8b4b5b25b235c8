"""Benchmark of the CoSA hot path (KAP plan + OSK attend) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--budget B] [--eps E] [--impl cosa|reference]
                    [--sweep | --chunked | --decode]

One step = one pass of the whole hot path over one batch of synthetic
input: cosa_plan (kap_pool, kap_score, kap_sort) then cosa_attend
(osk_attention).  The default workload is the 128K-token GQA layer
(B=1, 32 query heads, 8 kv heads, d=128, N=131072, blocks of 128, budget
10%).  Metric: effective TFLOP/s = dense causal attention FLOPs / step time
(higher is better); ms_per_step is the latency.  Inputs are resident in HBM
when the timed region starts and exceed L2, so no L2 flush is needed.

N > 1 (torchrun, one rank per GPU): every rank runs its own replica of the
workload (different seeds) with no data-path collective ("weak" scaling);
the barrier and max-over-ranks reduction use NCCL.

--impl reference times the CPU oracle (oracle/, plain C + OpenMP, as it
stands) on a bounded sample of the same workload; rank 0 alone runs it.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "128K-token prefill attention latency & effective TFLOP/s (frac of peak) vs dense"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="gqa_128k", choices=list(synth.WORKLOADS))
    ap.add_argument("--heads", default=None, metavar="HQ:HKV",
                    help="override the workload's query/kv head counts (a smaller case of the same layer, "
                         "e.g. for profiling); the workload is then reported as NAME[hqHQ:hkvHKV]")
    ap.add_argument("--recipe", default="default", choices=["default", "planned"],
                    help="input recipe: the default one, or a weaker structure (query direction 2, needles without sqrt(d))")
    ap.add_argument("--budget", type=float, default=None)
    ap.add_argument("--eps", type=float, default=None)
    ap.add_argument("--impl", default="cosa", choices=["cosa", "reference"])
    ap.add_argument("--no-dense", action="store_true", help="skip timing the dense path")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="CPU-baseline sample budget")
    ap.add_argument("--chunked", action="store_true",
                    help="chunked prefill: KAP with the pooled keys kept across chunks (cosa_plan_chunk) "
                         "against KAP that re-pools the whole cache (cosa_plan), one line (no headline line)")
    ap.add_argument("--decode", action="store_true",
                    help="one decode step per head after the workload's cache: cosa_decode_plan + cosa_attend "
                         "(Nq = 1) against the dense decode step, one line (no headline line)")
    ap.add_argument("--sweep", action="store_true",
                    help="one line per budget of the workload: latency, in-kernel skip fraction and error "
                         "against the dense path (no headline line)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), d.get("bf16_tflops_sustained", 1400.0), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def recorded_traffic(kernel: str):
    """DRAM bytes per launch (read + write) of `kernel` on the 128K workload,
    from the committed ncu record, or None if the record is missing or any
    source the kernel was built from changed since the capture."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic_gqa_128k.json")
    try:
        rec = json.load(open(path))["kernels"][kernel]
    except (OSError, KeyError, ValueError):
        return None
    csrc = os.path.join(ROOT, "block_sparse_attention_kap_b200", "csrc")
    for fname, digest in rec["sources_sha256_16"].items():
        try:
            cur = hashlib.sha256(open(os.path.join(csrc, fname), "rb").read()).hexdigest()[:16]
        except OSError:
            return None
        if cur != digest:
            return None
    return rec["dram_read_bytes"] + rec["dram_write_bytes"]


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.file = None

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.file is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.file.flush()
        rows = []
        with open(self.file.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.file.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        pw = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "sm_min_mhz": min(sm) if sm else None, "power_w_max": max(pw) if pw else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------- CPU oracle timing

def oracle_sample(inp, budget, eps, seconds, seed=0):
    """Run the oracle (KAP + OSK) on (b, h, Q-block) rows drawn from the
    workload until about `seconds` of wall time.  Returns (dense-equivalent
    FLOPs of the rows done, seconds, rows, threads)."""
    import random
    import oracle
    wl = inp.wl
    rng = random.Random(seed)
    off = wl.Nkv - wl.Nq
    flops, done, t_all = 0.0, 0, 0.0
    km = oracle.kmax(wl, budget)
    while t_all < seconds and done < 4096:
        sel = [(rng.randrange(wl.B), rng.randrange(wl.Hq), rng.randrange(wl.n_qblocks)) for _ in range(8)]
        t0 = time.perf_counter()
        plan = oracle.kap(inp, budget, sel=sel, kmax_=km)
        oracle.osk(inp, plan["order"], plan["count"], eps, sel=sel)
        t_all += time.perf_counter() - t0
        for (_, _, I) in sel:
            lo, hi = I * wl.bq, min((I + 1) * wl.bq, wl.Nq)
            pairs = sum(off + i + 1 for i in range(lo, hi))
            flops += 4.0 * wl.d * pairs
        done += len(sel)
    return flops, t_all, done, oracle.num_threads()


def config_of(wl, budget, eps, world, resident_bytes):
    """The workload's config block, the same for both arms of the benchmark."""
    return {"workload": wl.name, "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "Nq": wl.Nq, "Nkv": wl.Nkv,
            "d": wl.d, "bq": wl.bq, "bk": wl.bk, "stride": wl.stride, "paged": wl.paged,
            "budget": budget, "eps": eps, "parallelism": f"replicas x{world}",
            "l2": (f"inputs larger than L2 ({resident_bytes / 1e9:.2f} GB resident), no flush"
                   if resident_bytes > 126e6 else
                   f"inputs fit in L2 ({resident_bytes / 1e9:.3f} GB), no flush: steps run L2-warm")}


def run_reference(args, wl, budget, eps):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    inp = synth.generate(wl)
    per_step = max(2.0, min(12.0, 150.0 / max(1, args.steps + args.warmup)))
    for w in range(args.warmup):
        oracle_sample(inp, budget, eps, per_step / 4, seed=100 + w)
    tot_f, tot_t, rows, thr = 0.0, 0.0, 0, 1
    for s in range(args.steps):
        f, t, r, thr = oracle_sample(inp, budget, eps, per_step, seed=s)
        tot_f, tot_t, rows = tot_f + f, tot_t + t, rows + r
    value = tot_f / tot_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": config_of(wl, budget, eps, args.gpus, sum(t.numel() * 2 for t in (inp.q, inp.k, inp.v))),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                         "sample": f"{rows} random (b, head, Q-block) rows of {wl.name}, KAP + OSK each, "
                                   f"~{per_step:.0f} s per step"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- rank aggregation

def max_over_ranks(values, dist=None, device=None):
    """Element-wise max of a list of floats over all ranks (the slowest rank
    sets every time); identity when running on one rank."""
    if dist is None:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_tflops(flops_per_rank: float, world: int, ms: float) -> float:
    """Aggregate throughput: the work of all ranks over the slowest rank's time."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


# ----------------------------------------------------------------- budget sweep

def run_sweep(args, wl, eps):
    """For every budget of the workload: step latency (plan + attend), the
    fraction of selected blocks skipped in-kernel, and the error of the
    sparse output against the dense path on the same inputs."""
    import block_sparse_attention_kap_b200 as cosa
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    inp = synth.generate(wl)
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    pt = inp.page_table.to(dev) if inp.page_table is not None else None
    shape = cosa.shape_of_workload(wl)
    m = cosa.CoSA(shape, device=dev)
    dense = m.dense(q, k, v, page_table=pt, lse=True)
    dense_out, dense_lse = dense["out"].float(), dense["lse"]
    stream = torch.cuda.current_stream()
    dense_flops = wl.dense_causal_flops()
    for budget in wl.budgets:
        e = 0.0 if budget >= 1.0 else eps
        order, count, hrm = m.alloc_plan(budget)
        km = order.shape[-1]
        out = torch.empty(wl.B, wl.Hq, wl.Nq, wl.d, dtype=torch.bfloat16, device=dev)

        def step():
            cosa.cosa_plan(shape, q, k, pt, budget, km, order, count, hrm, None, None, m.workspace(), m.status,
                           stream)
            cosa.cosa_attend(shape, q, k, v, pt, order, count, km, e, out, None, None, m.status, stream)

        for _ in range(max(3, args.warmup)):
            step()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            step()
        b.record(stream)
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / args.steps
        res = m.attend(q, k, v, order, count, e, page_table=pt, skip_bits=True)
        # attention-mass recall of the plan: share of each row's dense softmax
        # mass inside the selected blocks, exp(lse over them - dense lse)
        sel_lse = m.attend(q, k, v, order, count, 0.0, page_table=pt, lse=True)["lse"]
        recall = torch.exp(sel_lse.double() - dense_lse.double())
        torch.cuda.synchronize()
        sel = int(count.sum().item())
        skipped = int(cosa.unpack_skip_bits(res["skip_bits"], km).sum().item())
        err = (res["out"].float() - dense_out).abs()
        assert m.device_status() == 0
        print(json.dumps({
            "kind": "sweep", "workload": wl.name, "budget": budget, "eps": e, "ms_per_step": ms,
            "effective_tflops": dense_flops / (ms * 1e-3) / 1e12, "selected_blocks": sel,
            "skipped_in_kernel_frac": skipped / max(1, sel),
            "err_vs_dense": {"max_abs": err.max().item(), "mean_abs": err.mean().item()},
            "mass_recall": {"mean": recall.mean().item(), "p01": torch.quantile(recall.flatten()[::97].float(), 0.01).item(),
                            "min": recall.min().item()}}), flush=True)


# ----------------------------------------------------------------- chunked prefill

def run_chunked(args, wl, budget, eps):
    """One prefill chunk (Nq new queries after Nkv - Nq cached keys): plan
    latency when every key is pooled again (cosa_plan) and when the pooled
    keys of earlier chunks come from a cache (cosa_plan_chunk), the attend
    latency on that plan, and the block union of the plan over the chunk's
    Q-blocks and each group's heads (CompactAttention's selection stage)
    executed with eps 0 and with in-kernel skipping; errors against the
    dense path."""
    import block_sparse_attention_kap_b200 as cosa
    if wl.Nkv == wl.Nq:
        raise SystemExit("--chunked needs a workload with cached keys (Nkv > Nq)")
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    inp = synth.generate(wl)
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    pt = inp.page_table.to(dev) if inp.page_table is not None else None
    shape = cosa.shape_of_workload(wl)
    m = cosa.CoSA(shape, device=dev)
    order, count, hrm = m.alloc_plan(budget)
    km = order.shape[-1]
    nkp, valid = wl.Nkv // wl.stride, (wl.Nkv - wl.Nq) // wl.stride
    cache = torch.empty(wl.B, wl.Hkv, nkp, wl.d, dtype=torch.bfloat16, device=dev)
    out = torch.empty(wl.B, wl.Hq, wl.Nq, wl.d, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    ws = m.workspace()
    cosa.cosa_plan_chunk(shape, q, k, pt, cache, 0, budget, km, order, count, hrm, None, None, ws, m.status,
                         stream)

    def timed(fn):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / args.steps

    full_ms = timed(lambda: cosa.cosa_plan(shape, q, k, pt, budget, km, order, count, hrm, None, None, ws,
                                           m.status, stream))
    full_order = order.clone()
    chunk_ms = timed(lambda: cosa.cosa_plan_chunk(shape, q, k, pt, cache, valid, budget, km, order, count, hrm,
                                                  None, None, ws, m.status, stream))
    attend_ms = timed(lambda: cosa.cosa_attend(shape, q, k, v, pt, order, count, km, eps, out, None, None,
                                               m.status, stream))
    # block union of the plan (per kv-head group, over the chunk's Q-blocks and
    # the group's heads), executed densely (eps 0) and with in-kernel skipping
    ures = m.block_union(order, count)
    u_order, u_count = ures["order"], ures["count"]
    u_km = u_order.shape[-1]
    union_ms = timed(lambda: cosa.cosa_block_union(shape, order, count, km, ures["table"], ures["table_len"],
                                                   u_order, u_count, stream))
    out_u = torch.empty_like(out)
    attend_union_dense_ms = timed(lambda: cosa.cosa_attend(shape, q, k, v, pt, u_order, u_count, u_km, 0.0, out_u,
                                                           None, None, m.status, stream))
    attend_union_eps_ms = timed(lambda: cosa.cosa_attend(shape, q, k, v, pt, u_order, u_count, u_km, eps, out_u,
                                                         None, None, m.status, stream))
    # the same union executed by the group kernel (one order per kv-head
    # group, K/V tiles shared by two heads); its rows are the union's rows of
    # the group's first head
    G = wl.Hq // wl.Hkv
    g_order = u_order.view(wl.B, wl.Hkv, G, m.nqb, u_km)[:, :, 0].contiguous()
    g_count = u_count.view(wl.B, wl.Hkv, G, m.nqb)[:, :, 0].contiguous()
    out_g = torch.empty_like(out)
    group_dense_ms = timed(lambda: cosa.cosa_attend_group(shape, q, k, v, pt, g_order, g_count, u_km, 0.0, out_g,
                                                           None, None, m.status, stream))
    group_eps_ms = timed(lambda: cosa.cosa_attend_group(shape, q, k, v, pt, g_order, g_count, u_km, eps, out_g,
                                                         None, None, m.status, stream))
    torch.cuda.synchronize()
    assert m.device_status() == 0
    assert torch.equal(order, full_order), "cached pooled keys changed the plan"
    # errors against the dense path on the same inputs
    dense_out = m.dense(q, k, v, page_table=pt)["out"].float()
    kap_out = m.attend(q, k, v, order, count, eps, page_table=pt)["out"].float()
    union_dense_out = m.attend(q, k, v, u_order, u_count, 0.0, page_table=pt)["out"].float()
    torch.cuda.synchronize()
    err = lambda o: {"max_abs": (o - dense_out).abs().max().item(), "mean_abs": (o - dense_out).abs().mean().item()}
    union_blocks = int(u_count.sum().item())
    kap_blocks = int(count.sum().item())
    row = 2.0 * wl.d
    q_bytes = row * wl.B * wl.Hq * wl.Nq * (1 + 1 / wl.stride)
    full_bytes = q_bytes + row * wl.B * wl.Hkv * wl.Nkv * (1 + 1 / wl.stride)
    chunk_bytes = q_bytes + row * wl.B * wl.Hkv * (wl.Nq * (1 + 1 / wl.stride) + wl.Nkv / wl.stride)
    print(json.dumps({
        "kind": "chunked", "workload": wl.name, "budget": budget, "eps": eps, "Nq": wl.Nq, "Nkv": wl.Nkv,
        "plan_full_ms": full_ms, "plan_chunk_ms": chunk_ms, "plan_speedup": full_ms / chunk_ms,
        "attend_ms": attend_ms, "step_full_ms": full_ms + attend_ms, "step_chunk_ms": chunk_ms + attend_ms,
        "kap_blocks": kap_blocks, "err_kap_vs_dense": err(kap_out),
        "union": {"union_ms": union_ms, "blocks": union_blocks, "attend_eps0_ms": attend_union_dense_ms,
                  "attend_eps_ms": attend_union_eps_ms,
                  "group_attend_eps0_ms": group_dense_ms, "group_attend_eps_ms": group_eps_ms,
                  "step_eps0_ms": chunk_ms + union_ms + min(attend_union_dense_ms, group_dense_ms),
                  "err_eps0_vs_dense": err(union_dense_out)},
        "pool_bytes": {"full": full_bytes, "chunk": chunk_bytes},
        "dense_causal_tflop": wl.dense_causal_flops() / 1e12,
        "effective_tflops_chunk": wl.dense_causal_flops() / ((chunk_ms + attend_ms) * 1e-3) / 1e12}), flush=True)


# ----------------------------------------------------------------- decode step

def run_decode(args, wl, budget, eps):
    """One decode step: the last query row of every head of the workload is
    the new token (position Nkv-1); the pooled keys are already cached, as
    after a prefill with cosa_plan_chunk.  Times the proxy (cosa_decode_plan)
    and the attention (cosa_decode_attend), against the dense decode step
    (every block, eps 0) on the same kernels; reports the K/V bytes the
    sparse step reads, the rate at which it reads them against the measured
    HBM bandwidth, and its error against the dense step.  cosa_attend on the
    same one-row shape is timed as context."""
    import block_sparse_attention_kap_b200 as cosa
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    inp = synth.generate(wl)
    q = inp.q[:, :, -1:, :].contiguous().to(dev)                 # [B, Hq, 1, d]
    k, v = inp.k.to(dev), inp.v.to(dev)
    pt = inp.page_table.to(dev) if inp.page_table is not None else None
    shape = cosa.make_shape(wl.B, wl.Hq, wl.Hkv, 1, wl.Nkv, wl.d, 128, wl.bk, wl.stride, wl.paged,
                            wl.num_pages if wl.paged else 0)
    m = cosa.CoSA(shape, device=dev)
    nkp = wl.Nkv // wl.stride
    cache = torch.empty(wl.B, wl.Hkv, nkp, wl.d, dtype=torch.bfloat16, device=dev)
    plan = m.decode_plan(q, k, budget, cache, 0, page_table=pt)   # fills the pooled-key cache
    order, count = plan["order"], plan["count"]
    km = order.shape[-1]
    out = torch.empty(wl.B, wl.Hq, 1, wl.d, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def timed(fn):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / args.steps

    plan_ms = timed(lambda: cosa.cosa_decode_plan(shape, q, k, pt, cache, nkp, budget, km, order, count,
                                                  plan["hrm_count"], None, None, stream))
    tile_attend_ms = timed(lambda: cosa.cosa_attend(shape, q, k, v, pt, order, count, km, eps, out, None, None,
                                                    m.status, stream))
    d_order, d_count = m.dense_order()
    d_km = d_order.shape[-1]
    ws = torch.empty(max(cosa.cosa_decode_attend_workspace_bytes(shape, km),
                         cosa.cosa_decode_attend_workspace_bytes(shape, d_km)), dtype=torch.uint8, device=dev)
    attend_ms = timed(lambda: cosa.cosa_decode_attend(shape, q, k, v, pt, order, count, km, eps, out, None, None,
                                                      ws, stream))
    dense_ms = timed(lambda: cosa.cosa_decode_attend(shape, q, k, v, pt, d_order, d_count, d_km, 0.0, out, None,
                                                     None, ws, stream))
    tile_dense_ms = timed(lambda: cosa.cosa_attend(shape, q, k, v, pt, d_order, d_count, d_km, 0.0, out, None, None,
                                                   m.status, stream))
    res = m.decode_attend(q, k, v, order, count, eps, page_table=pt, skip_bits=True)
    dense_out = m.decode_attend(q, k, v, d_order, d_count, 0.0, page_table=pt)["out"].float()
    torch.cuda.synchronize()
    assert m.device_status() == 0
    sel = int(count.sum().item())
    skipped = int(cosa.unpack_skip_bits(res["skip_bits"], km).sum().item())
    tile = wl.bk * wl.d * 2
    sparse_bytes = tile * (sel + (sel - skipped))                  # K of every visit, V of computed ones
    dense_bytes = 2 * tile * int(d_count.sum().item())
    err = (res["out"].float() - dense_out).abs()
    rows = wl.B * wl.Hq
    hbm_peak = load_peaks()[0]
    print(json.dumps({
        "kind": "decode", "workload": wl.name, "rows": rows, "Nkv": wl.Nkv, "budget": budget, "eps": eps,
        "plan_ms": plan_ms, "attend_ms": attend_ms, "step_ms": plan_ms + attend_ms, "dense_step_ms": dense_ms,
        "speedup_vs_dense": dense_ms / (plan_ms + attend_ms),
        "selected_blocks": sel, "skipped_in_kernel_frac": skipped / max(1, sel),
        "kv_bytes": {"sparse": sparse_bytes, "dense": dense_bytes},
        "attend_gbs": sparse_bytes / (attend_ms * 1e-3) / 1e9,
        "attend_frac_of_hbm": sparse_bytes / (attend_ms * 1e-3) / 1e9 / hbm_peak,
        "dense_gbs": dense_bytes / (dense_ms * 1e-3) / 1e9,
        "dense_frac_of_hbm": dense_bytes / (dense_ms * 1e-3) / 1e9 / hbm_peak,
        "tile_kernel_context": {"attend_ms": tile_attend_ms, "dense_ms": tile_dense_ms,
                                "note": "cosa_attend (128-row tensor-core tiles, one valid row) on the same step"},
        "err_vs_dense": {"max_abs": err.max().item(), "mean_abs": err.mean().item()}}), flush=True)


# ----------------------------------------------------------------- GPU arm

def main():
    args = parse()
    wl = synth.WORKLOADS[args.workload]
    if args.heads:
        hq, hkv = (int(x) for x in args.heads.split(":"))
        wl = wl.replace(Hq=hq, Hkv=hkv, name=f"{wl.name}[hq{hq}:hkv{hkv}]")
    if args.recipe != "default":
        wl = wl.replace(recipe=args.recipe, name=f"{wl.name}[{args.recipe}]")
    budget = args.budget if args.budget is not None else (0.1 if 0.1 in wl.budgets else wl.budgets[0])
    eps = args.eps if args.eps is not None else wl.eps
    if args.impl == "reference":
        run_reference(args, wl, budget, eps)
        return
    if args.sweep:
        run_sweep(args, wl, eps)
        return
    if args.chunked:
        run_chunked(args, wl, budget, eps)
        return
    if args.decode:
        run_decode(args, wl, budget, eps)
        return
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    import block_sparse_attention_kap_b200 as cosa

    # inputs: generated on the host, pinned, copied once to HBM
    inp = synth.generate(wl, rank=rank)
    host = [inp.q.pin_memory(), inp.k.pin_memory(), inp.v.pin_memory()]
    pt_h = inp.page_table.pin_memory() if inp.page_table is not None else None
    q, k, v = (t.to(dev) for t in host)
    pt = pt_h.to(dev) if pt_h is not None else None
    shape = cosa.shape_of_workload(wl)
    m = cosa.CoSA(shape, device=dev)
    order, count, hrm = m.alloc_plan(budget)
    km = order.shape[-1]
    out = torch.empty(wl.B, wl.Hq, wl.Nq, wl.d, dtype=torch.bfloat16, device=dev)
    ws = m.workspace()
    stream = torch.cuda.current_stream()

    ev = lambda: torch.cuda.Event(enable_timing=True)

    def step(timers=None):
        if timers is not None:
            timers[0].record(stream)
        cosa.cosa_plan(shape, q, k, pt, budget, km, order, count, hrm, None, None, ws, m.status, stream)
        if timers is not None:
            timers[1].record(stream)
        cosa.cosa_attend(shape, q, k, v, pt, order, count, km, eps, out, None, None, m.status, stream)
        if timers is not None:
            timers[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert m.device_status() == 0, "device status reported a failure"

    # ---------------------------------------------------------- timed region
    timers = [[ev(), ev(), ev()] for _ in range(args.steps)]
    t_start, t_end = ev(), ev()
    with ClockSampler(local) as clk:
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        t_start.record(stream)
        for i in range(args.steps):
            step(timers[i])
        t_end.record(stream)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
    ms_total = t_start.elapsed_time(t_end)
    kap_ms = statistics.mean(t[0].elapsed_time(t[1]) for t in timers)
    osk_ms = statistics.mean(t[1].elapsed_time(t[2]) for t in timers)
    ms_step = ms_total / args.steps
    ms_step, kap_ms, osk_ms = max_over_ranks([ms_step, kap_ms, osk_ms], dist, dev)
    clocks = clk.summary()

    # ---------------------------------------------------------- work accounting (outside the timed region)
    res = m.attend(q, k, v, order, count, eps, page_table=pt, skip_bits=True)
    torch.cuda.synchronize()
    sel_blocks = int(count.sum().item())
    skipped = int(cosa.unpack_skip_bits(res["skip_bits"], km).sum().item())
    computed = sel_blocks - skipped
    blk_flops = 2.0 * wl.bq * wl.bk * wl.d
    osk_flops = blk_flops * (sel_blocks + computed)          # QK for every visited block, PV for computed
    dense_flops = wl.dense_causal_flops()
    n_causal = sum(min(wl.n_kblocks, ((wl.Nkv - wl.Nq) + min((I + 1) * wl.bq, wl.Nq) - 1) // wl.bk + 1)
                   for I in range(wl.n_qblocks)) * wl.B * wl.Hq
    kap_bytes = 2.0 * wl.d * (wl.B * wl.Hq * wl.Nq + wl.B * wl.Hkv * wl.Nkv) * (1 + 1 / wl.stride) + \
        4.0 * order.numel() + 8.0 * count.numel()

    hbm_peak, tc_peak, tc_sust, peak_kind = load_peaks()
    value = whole_job_tflops(dense_flops, world, ms_step)
    osk_tflops = osk_flops / (osk_ms * 1e-3) / 1e12

    # ---------------------------------------------------------- dense path (same kernel, natural order, eps 0)
    dense = None
    if not args.no_dense:
        d_order, d_count = m.dense_order()
        dsteps = max(1, min(args.steps, 5))
        m.attend(q, k, v, d_order, d_count, 0.0, page_table=pt, out=out)
        torch.cuda.synchronize()
        a, b = ev(), ev()
        # the dense path keeps the tensor pipe far busier than the sparse step:
        # its clocks are sampled on their own (the power cap lowers them)
        with ClockSampler(local) as dclk:
            a.record(stream)
            for _ in range(dsteps):
                cosa.cosa_attend(shape, q, k, v, pt, d_order, d_count, d_order.shape[-1], 0.0, out, None, None,
                                 m.status, stream)
            b.record(stream)
            torch.cuda.synchronize()
        dense_ms = max_over_ranks([a.elapsed_time(b) / dsteps], dist, dev)[0]
        dense = {"kernel": "osk_attention", "ms": dense_ms, "tflops": dense_flops / (dense_ms * 1e-3) / 1e12,
                 "frac_of_peak": dense_flops / (dense_ms * 1e-3) / 1e12 / tc_peak,
                 "speedup_of_sparse_step": dense_ms / ms_step, "clocks": dclk.summary()}
        del d_order, d_count
        if (wl.Hq // wl.Hkv) % 2 == 0:
            # the same dense path through the group kernel (one order per
            # kv-head group, each K/V tile loaded once for two query heads);
            # the dense path reported is the faster of the two
            g_order, g_count = m.dense_order_group()
            m.attend_group(q, k, v, g_order, g_count, 0.0, page_table=pt, out=out)
            torch.cuda.synchronize()
            a, b = ev(), ev()
            with ClockSampler(local) as gclk:
                a.record(stream)
                for _ in range(dsteps):
                    cosa.cosa_attend_group(shape, q, k, v, pt, g_order, g_count, g_order.shape[-1], 0.0, out, None,
                                           None, m.status, stream)
                b.record(stream)
                torch.cuda.synchronize()
            g_ms = max_over_ranks([a.elapsed_time(b) / dsteps], dist, dev)[0]
            group = {"kernel": "osk_group", "ms": g_ms, "tflops": dense_flops / (g_ms * 1e-3) / 1e12,
                     "frac_of_peak": dense_flops / (g_ms * 1e-3) / 1e12 / tc_peak,
                     "speedup_of_sparse_step": g_ms / ms_step, "clocks": gclk.summary()}
            per_head = dict(dense)
            dense = dict(group if g_ms < dense_ms else per_head)
            dense["per_head_kernel"] = {k_: per_head[k_] for k_ in ("ms", "tflops", "frac_of_peak")}
            dense["group_kernel"] = {k_: group[k_] for k_ in ("ms", "tflops", "frac_of_peak")}
            del g_order, g_count
        # context only, not this library: torch's fused causal attention on the
        # same inputs (whatever backend torch picks), when its top-left causal
        # alignment matches (Nq == Nkv) and K/V are contiguous
        if wl.Nq == wl.Nkv and not wl.paged:
            try:
                sdpa = torch.nn.functional.scaled_dot_product_attention
                o_ref = sdpa(q, k, v, is_causal=True, enable_gqa=True)
                torch.cuda.synchronize()
                a, b = ev(), ev()
                a.record(stream)
                for _ in range(dsteps):
                    o_ref = sdpa(q, k, v, is_causal=True, enable_gqa=True)
                b.record(stream)
                torch.cuda.synchronize()
                sdpa_ms = max_over_ranks([a.elapsed_time(b) / dsteps], dist, dev)[0]
                dense["torch_sdpa_context"] = {
                    "ms": sdpa_ms, "tflops": dense_flops / (sdpa_ms * 1e-3) / 1e12,
                    "speedup_of_sparse_step": sdpa_ms / ms_step,
                    "note": "torch.nn.functional.scaled_dot_product_attention, library kernel, context only"}
                del o_ref
            except (RuntimeError, TypeError) as exc:
                dense["torch_sdpa_context"] = {"unavailable": str(exc).splitlines()[0][:200]}

    # ---------------------------------------------------------- end to end through the public API (host buffers)
    # Every step copies its inputs from pinned host memory and its output
    # back.  The copies run on their own streams with two device buffer sets,
    # so step i's host-to-device copy and step i-1's device-to-host copy
    # overlap step i-1's and i's compute (the two copy directions use
    # separate copy engines); the timed region spans the first copy in to
    # the last copy out.
    h2d = sum(t.numel() * t.element_size() for t in host) + (pt_h.numel() * 4 if pt_h is not None else 0)
    d2h = out.numel() * out.element_size()
    s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    dev_in = [(q, k, v, pt),
              tuple(torch.empty_like(t) if t is not None else None for t in (q, k, v, pt))]
    outs = [out, torch.empty_like(out)]
    outs_h = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
    sync_ev = lambda: [torch.cuda.Event(), torch.cuda.Event()]
    in_ready, in_free, out_ready, out_free = sync_ev(), sync_ev(), sync_ev(), sync_ev()

    def e2e_run(nsteps):
        for i in range(nsteps):
            bi = i % 2
            qd, kd, vd, ptd = dev_in[bi]
            s_h2d.wait_event(in_free[bi])             # step i-2's compute is done with this set
            with torch.cuda.stream(s_h2d):
                qd.copy_(host[0], non_blocking=True)
                kd.copy_(host[1], non_blocking=True)
                vd.copy_(host[2], non_blocking=True)
                if ptd is not None:
                    ptd.copy_(pt_h, non_blocking=True)
            in_ready[bi].record(s_h2d)
            stream.wait_event(in_ready[bi])
            stream.wait_event(out_free[bi])           # step i-2's output has left the device
            cosa.cosa_plan(shape, qd, kd, ptd, budget, km, order, count, hrm, None, None, ws, m.status, stream)
            cosa.cosa_attend(shape, qd, kd, vd, ptd, order, count, km, eps, outs[bi], None, None, m.status,
                             stream)
            in_free[bi].record(stream)
            out_ready[bi].record(stream)
            s_d2h.wait_event(out_ready[bi])
            with torch.cuda.stream(s_d2h):
                outs_h[bi].copy_(outs[bi], non_blocking=True)
            out_free[bi].record(s_d2h)

    e2e_run(2)
    torch.cuda.synchronize()
    esteps = max(3, min(args.steps, 10))
    a, b = ev(), ev()
    if dist is not None:
        dist.barrier()
    a.record(stream)
    s_h2d.wait_stream(stream)
    e2e_run(esteps)
    stream.wait_stream(s_d2h)
    stream.wait_stream(s_h2d)
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks([a.elapsed_time(b) / esteps], dist, dev)[0]
    assert m.device_status() == 0
    assert torch.equal(outs_h[(esteps - 1) % 2], outs[(esteps - 1) % 2].cpu())

    # the same copies in the same pattern with no compute between them: the
    # host link's floor for this step's bytes
    def copies_only(nsteps):
        for i in range(nsteps):
            bi = i % 2
            qd, kd, vd, ptd = dev_in[bi]
            with torch.cuda.stream(s_h2d):
                qd.copy_(host[0], non_blocking=True)
                kd.copy_(host[1], non_blocking=True)
                vd.copy_(host[2], non_blocking=True)
                if ptd is not None:
                    ptd.copy_(pt_h, non_blocking=True)
            with torch.cuda.stream(s_d2h):
                outs_h[bi].copy_(outs[bi], non_blocking=True)

    torch.cuda.synchronize()
    a, b = ev(), ev()
    a.record(stream)
    s_h2d.wait_stream(stream)
    s_d2h.wait_stream(stream)
    copies_only(esteps)
    stream.wait_stream(s_d2h)
    stream.wait_stream(s_h2d)
    b.record(stream)
    torch.cuda.synchronize()
    copy_floor_ms = max_over_ranks([a.elapsed_time(b) / esteps], dist, dev)[0]

    # ---------------------------------------------------------- CPU baseline (rank 0, N = 1)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        f, t, rows, thr = oracle_sample(inp, budget, eps, args.cpu_seconds)
        cpu = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
               "sample": f"{rows} random (b, head, Q-block) rows of {wl.name} (KAP + OSK each), {t:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_of(wl, budget, eps, world, sum(t.numel() * 2 for t in host)),
            "roofline": {"bound": "tensor", "kernel": "osk_attention", "achieved": osk_tflops, "peak": tc_peak,
                         "unit": "TFLOP/s", "frac": osk_tflops / tc_peak,
                         "traffic": recorded_traffic("osk_attention_kernel<128>") if wl.name == "gqa_128k" and
                         abs(budget - 0.1) < 1e-9 and abs(eps - 1e-4) < 1e-12 and world == 1 else None,
                         "peak_kind": f"{peak_kind} bf16 dense (burst)",
                         "algorithmic_flops_per_launch": osk_flops},
            "kap_roofline": {"bound": "hbm", "kernels": "kap_pool+kap_score+kap_sort", "ms": kap_ms,
                             "achieved": kap_bytes / (kap_ms * 1e-3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                             "frac": kap_bytes / (kap_ms * 1e-3) / 1e9 / hbm_peak,
                             "algorithmic_bytes_per_launch": kap_bytes},
            "cpu_baseline": cpu,
            "e2e": {"value": whole_job_tflops(dense_flops, world, e2e_ms), "unit": "TFLOP/s",
                    "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": esteps, "pipelined": "copies in/out overlap the neighbouring steps' compute",
                    "copy_floor_ms": copy_floor_ms,
                    "copy_floor": "the same host-to-device and device-to-host copies per step with no compute"},
            "gpu_launches": 4 * args.steps,
            "clocks": clocks,
            "kap_ms": kap_ms, "osk_ms": osk_ms,
            "selected_blocks": sel_blocks, "causal_blocks": n_causal,
            "selected_frac": sel_blocks / n_causal, "skipped_in_kernel_frac": skipped / max(1, sel_blocks),
            "dense": dense,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
