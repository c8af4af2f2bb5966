"""Benchmark: effective TFLOP/s of block-sparse varlen attention, forward +
backward, on one of the five workloads (default C3: BNSD B=2, N1=N2=32,
S=8192, D=128, bf16, block (128,512), fully dense index -- the tensor-core
roofline workload).

A step is one forward (bsa_fwd: index compaction, work list, attention)
followed by one backward (bsa_bwd: inverse index, work list, preprocess,
KV-major dK/dV with dQ reduction, dQ conversion) on inputs resident in HBM,
the backward consuming the forward's out and lse.  Effective FLOPs count
kept (q head, valid q token, valid kv token) pairs only: 4*D per pair
forward, 10*D backward.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config C3] [--causal] [--impl ours|reference]

Under torchrun each rank runs an independent replica of the workload on its
own GPU (the path shards by batch / kv-head group with no exchange), so the
job value is N x the per-replica work over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "effective TFLOP/s (selected blocks only) fwd and bwd; % of B200 bf16 tensor peak"
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
DESCR = {
    1: "C1: BNSD B=1 N1=N2=2 S=512 D=64 bf16, block (128,128), random index [1,2,4,4]",
    2: "C2: TND B=4 lens U[256,3072] N1=16 N2=4 D=128 bf16, block (128,128), 25% + diagonal",
    3: "C3: BNSD B=2 N1=N2=32 S=8192 D=128 bf16, block (128,512), dense index [2,32,64,16]",
    4: "C4: BNSD B=1 N1=N2=24 S=32768 D=128 bf16, block (128,128), sink+diag+14 random of 256",
    5: "C5: TND q B=8 lens U[512,4096] + paged KV [P,128,8,128] fp16, N1=32 N2=8, top-8 blocks",
}
# kernels this library launches per call: forward geometry, compaction, sort
# (+ the rank merge when the list spans more than one 4096-key chunk), main;
# backward geometry, compaction, inverse count, scan, inverse fill, keys,
# sort (+ rank), preprocessing, main, dQ conversion, kv tail; the
# deterministic backward adds the forward list's sort (+ rank) and the dQ
# pass and drops the dQ conversion
SORT_CHUNK = 4096


def _sort_launches(slots: int) -> int:
    return 0 if slots == 0 else (1 if slots <= SORT_CHUNK else 2)


def launches_per_step(fwd_slots: int, bwd_slots: int, deterministic: bool) -> int:
    fwd = 3 + _sort_launches(fwd_slots)
    bwd = 10 + _sort_launches(bwd_slots)
    if deterministic:
        bwd += _sort_launches(fwd_slots)
    return fwd + bwd


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return FALLBACK_PEAKS, "fallback"


def _pairs(p):
    # kept pairs = sum over (head, query block row) of valid q rows x valid
    # kv tokens of the accepted blocks (causal: only the tokens each row
    # sees); the index of every workload here is valid (ascending, in
    # range), so accepted = present entries
    idx = p.index.view(torch.int16).numpy().view(np.uint16).astype(np.int64)
    g = p.N1 // p.N2
    heads = 1 if p.Hidx == p.N1 else g
    causal = bool(getattr(p, "causal", False))

    def row_pairs(b, i, e):
        e = e[e != 0xFFFF]
        rows = min(p.BQ, p.lens_q[b] - i * p.BQ)
        lo = e * p.BKV
        hi = np.minimum(lo + p.BKV, p.lens_kv[b])
        if not causal:
            return rows * int((hi - lo).sum())
        t = i * p.BQ + np.arange(rows, dtype=np.int64)
        last = t[None, :] + (p.lens_kv[b] - p.lens_q[b]) + 1   # one past the last token row t sees
        return int(np.maximum(0, np.minimum(hi[:, None], last) - lo[:, None]).sum())

    total = 0
    if p.layout_q == "BNSD":
        for b in range(p.B):
            for hi in range(p.Hidx):
                for i in range(idx.shape[2]):
                    total += heads * row_pairs(b, i, idx[b, hi, i])
    else:
        off = 0
        for b in range(p.B):
            nq = -(-p.lens_q[b] // p.BQ)
            for hi in range(p.Hidx):
                for i in range(nq):
                    total += heads * row_pairs(b, i, idx[hi, off + i])
            off += nq
    return total


def _alg_bytes(p):
    """Algorithmic bytes of one forward and one backward call: every tensor
    the pass must touch, once.  Forward: Q, out, lse, the index and the K, V
    rows of the kv blocks some row of the kv head's group selects.  Backward:
    Q, out, dOut, lse read and dQ written; those K, V rows read; dK, dV
    written for every used kv row (zeros where nothing selects it)."""
    es = 1 if p.dtype == torch.float8_e4m3fn else 2
    D, N1, N2 = p.D, p.N1, p.N2
    g = N1 // N2
    tq = sum(p.lens_q) if p.layout_q == "TND" else p.B * p.q.shape[2]
    qb = tq * N1 * D
    idx = p.index.view(torch.int16).numpy().view(np.uint16).astype(np.int64)
    kv_sel = 0   # selected kv rows, summed over kv heads
    off = 0
    for b in range(p.B):
        nq = -(-p.lens_q[b] // p.BQ)
        for h2 in range(N2):
            his = range(h2 * g, (h2 + 1) * g) if p.Hidx == N1 else [h2]
            rows = [idx[b, hi, :nq] if p.layout_q == "BNSD" else idx[hi, off:off + nq] for hi in his]
            blocks = set(int(x) for r in rows for x in r.ravel()) - {0xFFFF}
            kv_sel += sum(max(0, min(p.BKV, p.lens_kv[b] - j * p.BKV)) for j in blocks)
        off += nq if p.layout_q == "TND" else 0
    kv_used = sum(p.lens_kv) * N2
    small = p.index.numel() * 2 + sum(0 if t is None else t.numel() * t.element_size()
                                      for t in (p.cu_q, p.cu_kv, p.seqused_kv, p.block_table))
    fwd = qb * es + qb * 2 + tq * N1 * 4 + 2 * kv_sel * D * es + small
    bwd = qb * 2 * 4 + tq * N1 * 4 + 2 * kv_sel * D * 2 + 2 * kv_used * D * 2 + small
    return fwd, bwd


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "100"], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.25)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- oracle leg
def _oracle_subproblem(cfg: int, q_rows: int, causal: bool = False, fp8: bool = False,
                       shared_rows: bool = False):
    """A bounded slice of the workload for the CPU oracle: batch 0, head 0,
    the first q_rows query rows against the full key range (causal: the
    last q_rows rows, which keeps every row's place relative to the end of
    the kv sequence); a BNSD slice of more rows than one head holds takes
    whole heads 0..h-1 of batch 0.  TND workloads: batch 0's first q_rows query rows of
    head 0 against batch 0's kv rows of kv head 0 (gathered out of the pages
    for a paged cache: the same rows, stored contiguously)."""
    import workloads
    from workloads.gen import make_problem, pat_dense
    p = workloads.make_config(cfg, causal=causal, fp8=fp8, shared_rows=shared_rows)
    if p.layout_q != "BNSD":
        L0, kv0 = p.lens_q[0], p.lens_kv[0]
        q_rows = max(min(L0, p.BQ), min(L0, (q_rows // p.BQ) * p.BQ))
        sub = make_problem(layout_q="TND", layout_kv="TND", B=1, N1=1, N2=1, D=p.D,
                           lens_q=[q_rows], lens_kv=[kv0], BQ=p.BQ, BKV=p.BKV, W=p.W,
                           pattern=pat_dense, dtype=p.dtype, scale=p.scale)
        sub.q = p.q[:q_rows, :1].contiguous()
        sub.dout = p.dout[:q_rows, :1].contiguous()
        if p.layout_kv == "TND":
            sub.k, sub.v = (t[:kv0, :1].contiguous() for t in (p.k, p.v))
        else:
            pages = p.block_table[0, :-(-kv0 // p.page_size)].long()
            sub.k, sub.v = (t[pages].reshape(-1, p.N2, p.D)[:kv0, :1].contiguous()
                            for t in (p.k, p.v))
        sub.index = p.index[:1, :-(-q_rows // p.BQ)].contiguous()
        return sub
    S = p.q.shape[2]
    # past one head's rows the slice takes whole heads of batch 0 (BNSD
    # workloads here have one kv head per query head and one index row each)
    h = 1
    if q_rows > S and p.N1 == p.N2 == p.Hidx:
        h = min(p.N1, (q_rows + S // 2) // S)  # the nearest whole number of heads
    q_rows = max(p.BQ, min(S, (q_rows // p.BQ) * p.BQ))
    sub = make_problem(B=1, N1=h, N2=h, D=p.D, Sq=q_rows, Skv=p.k.shape[2], lens_kv=[p.lens_kv[0]],
                       BQ=p.BQ, BKV=p.BKV, W=p.W, pattern=pat_dense, dtype=p.dtype, scale=p.scale,
                       causal=causal, out_dtype=p.out_dtype)
    rows = slice(S - q_rows, S) if causal else slice(0, q_rows)
    blocks = slice(rows.start // p.BQ, rows.stop // p.BQ)
    sub.q = p.q[:1, :h, rows].contiguous()
    sub.k = p.k[:1, :h].contiguous()
    sub.v = p.v[:1, :h].contiguous()
    sub.dout = p.dout[:1, :h, rows].contiguous()
    sub.index = p.index[:1, :h, blocks].contiguous()
    sub.lens_q = [q_rows]
    return sub


def _oracle_step(sub):
    import oracle
    o = oracle.Oracle(sub)
    t = time.perf_counter()
    out, lse, _ = o.fwd()
    o.bwd(out, sub.dout, lse)
    return time.perf_counter() - t


def _oracle_rate(cfg: int, target_s: float, causal: bool = False, shared_rows: bool = False):
    """Calibrate the slice to ~target_s per step; returns (sub, pairs)."""
    sub = _oracle_subproblem(cfg, 128, causal, shared_rows=shared_rows)
    t = _oracle_step(sub)
    rows = int(128 * max(1.0, target_s / max(t, 1e-3)))
    sub = _oracle_subproblem(cfg, rows, causal, shared_rows=shared_rows)
    return sub, _pairs(sub)


def _descr(cfg: int, causal: bool, deterministic: bool = False, shared_rows: bool = False,
           per_head_rows: bool = False) -> str:
    return (DESCR[cfg] + (", causal mask + lower-triangular index" if causal else "")
            + (", deterministic backward" if deterministic else "")
            + (", one index row per GQA group (Hidx = N2; packed forward tiles)"
               if shared_rows and not per_head_rows else "")
            + (", the per-group index rows copied to every query head (Hidx = N1)"
               if per_head_rows else ""))


def cpu_baseline(cfg: int, target_s: float = 16.0, causal: bool = False, shared_rows: bool = False):
    sub, pairs = _oracle_rate(cfg, target_s, causal, shared_rows)
    t = _oracle_step(sub)
    flops = 14 * sub.D * pairs
    return {"value": flops / t / 1e12, "unit": "TFLOP/s", "cores": _omp_threads(), "kind": "oracle",
            "sample": f"fp64 oracle fwd+bwd on batch 0, {_heads_of(sub)}, "
                      f"{'last' if causal else 'first'} {_rows_of(sub)} query rows "
                      f"x {sub.lens_kv[0]} keys of {DESCR[cfg].split(':')[0]} ({pairs} kept pairs, "
                      f"{t:.1f} s)"}


def _rows_of(sub):
    return sub.q.shape[2] if sub.layout_q == "BNSD" else sub.q.shape[0]


def _heads_of(sub):
    return "head 0" if sub.N1 == 1 else f"heads 0..{sub.N1 - 1}"


def _omp_threads():
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n and n.isdigit() else (os.cpu_count() or 1)


def run_reference(args):
    """The oracle on the host cores, on the same workload, metric and unit as
    the GPU arm (--causal, --deterministic and --fp8 select the same variant;
    the deterministic mode changes nothing the oracle computes; --fp8 times
    the forward alone, as the GPU arm does)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    fp8 = getattr(args, "fp8", False)
    if fp8:
        sub = _oracle_subproblem(3, 1024, fp8=True)
        pairs = _pairs(sub)

        def one():
            import oracle
            t = time.perf_counter()
            oracle.Oracle(sub).fwd()
            return time.perf_counter() - t
        metric, per_pair = "effective TFLOP/s (selected blocks only), FP8 forward", 4
        workload = DESCR[3] + ", q/k/v e4m3 (bf16 out), forward only"
    else:
        sub, pairs = _oracle_rate(args.config, 2.0, args.causal, args.shared_rows)

        def one():
            return _oracle_step(sub)
        metric, per_pair = METRIC, 14
        workload = _descr(args.config, args.causal, getattr(args, "deterministic", False),
                          args.shared_rows, args.per_head_rows)
    for _ in range(args.warmup):
        one()
    ts = [one() for _ in range(args.steps)]
    total = sum(ts)
    flops = per_pair * sub.D * pairs
    val = flops * args.steps / total / 1e12
    line = {"impl": "reference", "metric": metric, "value": val, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload, "sample": "see cpu_baseline"},
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": _omp_threads(),
                             "kind": "oracle",
                             "sample": f"batch 0, {_heads_of(sub)}, {'last' if args.causal else 'first'} "
                                       f"{_rows_of(sub)} query rows "
                                       f"({pairs} kept pairs) per step"},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ rank plumbing
def max_over_ranks(dist, values, device):
    """Element-wise maximum of per-rank timings (the slowest rank sets the
    time); identity without a process group."""
    if dist is None:
        return [float(x) for x in values]
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_tflops(world, flops_per_replica_step, ms_per_step):
    """Whole-job throughput: every rank runs one replica of the step, so the
    job does world x the work in the slowest rank's time."""
    return world * flops_per_replica_step / (ms_per_step * 1e-3) / 1e12


# -------------------------------------------------------------------- GPU leg
def run_ours(args):
    import block_sparse_variable_b200 as bsa
    import workloads

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    p = workloads.make_config(args.config, args.batch, args.causal, shared_rows=args.shared_rows,
                              per_head_rows=args.per_head_rows, heads=args.heads)
    p.deterministic = args.deterministic
    pairs = _pairs(p)
    P = bsa.params_of_problem(p)
    to = lambda t: None if t is None else t.to(dev)  # noqa: E731
    q, k, v, dout, index = (to(getattr(p, n)) for n in ("q", "k", "v", "dout", "index"))
    opt = dict(cu_seqlens_q=to(p.cu_q), cu_seqlens_kv=to(p.cu_kv), seqused_kv=to(p.seqused_kv),
               block_table=to(p.block_table))
    out = torch.empty_like(q)
    lse = torch.empty((q.shape[0], q.shape[1], q.shape[2]) if p.layout_q == "BNSD"
                      else (q.shape[0], q.shape[1]), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    wsf = torch.empty(bsa.bsa_fwd_get_workspace(q, k, v, index, P, out=out, lse=lse, **opt),
                      dtype=torch.uint8, device=dev)
    wsb = torch.empty(bsa.bsa_bwd_get_workspace(q, k, v, out, dout, lse, index, P, dq=dq, dk=dk,
                                                dv=dv, **opt), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    # the work lists' slot counts (their regions hold one int32 per slot)
    fwd_slots = bsa.bsa_fwd_workspace_layout(q, k, v, index, P, out=out, lse=lse, **opt).fwd_items.bytes // 4
    bwd_slots = bsa.bsa_bwd_workspace_layout(q, k, v, out, dout, lse, index, P, **opt).bwd_items.bytes // 4

    def step():
        bsa.bsa_fwd(q, k, v, index, P, out=out, lse=lse, workspace=wsf, stream=stream, **opt)
        bsa.bsa_bwd(q, k, v, out, dout, lse, index, P, dq=dq, dk=dk, dv=dv, workspace=wsb,
                    stream=stream, **opt)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    flags = bsa.bsa_read_status(wsf) | bsa.bsa_read_status(wsb)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    # events the library records around each call's main attention kernel;
    # they must exist on the device before their handles are passed on
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for e in (e for row in kev for e in row):
        e.record(stream)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index if world == 1 else local) as clk:
        start.record(stream)
        for s in range(args.steps):
            ev[s][0].record(stream)
            bsa.bsa_set_main_kernel_events(kev[s][0], kev[s][1])
            bsa.bsa_fwd(q, k, v, index, P, out=out, lse=lse, workspace=wsf, stream=stream, **opt)
            ev[s][1].record(stream)
            bsa.bsa_set_main_kernel_events(kev[s][2], kev[s][3])
            bsa.bsa_bwd(q, k, v, out, dout, lse, index, P, dq=dq, dk=dk, dv=dv, workspace=wsb,
                        stream=stream, **opt)
            ev[s][2].record(stream)
        stop.record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    ms = start.elapsed_time(stop)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    bwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    fwd_kms = statistics.mean(e[0].elapsed_time(e[1]) for e in kev)
    bwd_kms = statistics.mean(e[2].elapsed_time(e[3]) for e in kev)
    ms, fwd_ms, bwd_ms, fwd_kms, bwd_kms = max_over_ranks(dist, [ms, fwd_ms, bwd_ms, fwd_kms, bwd_kms], dev)

    # ---- end to end through the C ABI from pinned host buffers
    hq, hk, hv, hdo = (t.cpu().pin_memory() for t in (q, k, v, dout))
    hidx = index.cpu().pin_memory()
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h_lse = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    h_dq = torch.empty(dq.shape, dtype=dq.dtype).pin_memory()
    h_dk = torch.empty(dk.shape, dtype=dk.dtype).pin_memory()
    h_dv = torch.empty(dv.shape, dtype=dv.dtype).pin_memory()
    e2e_steps = max(2, min(args.steps, 5))
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdo, hidx))
    d2h = sum(t.numel() * t.element_size() for t in (h_out, h_lse, h_dq, h_dk, h_dv))

    def e2e_step():
        for d_, h_ in ((q, hq), (k, hk), (v, hv), (dout, hdo), (index, hidx)):
            d_.copy_(h_, non_blocking=True)
        step()
        for h_, d_ in ((h_out, out), (h_lse, lse), (h_dq, dq), (h_dk, dk), (h_dv, dv)):
            h_.copy_(d_, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms, = max_over_ranks(dist, [e0.elapsed_time(e1) / e2e_steps], dev)

    if rank == 0:
        peaks, which = _peaks()
        D = p.D
        step_flops = 14 * D * pairs
        ms_step = ms / args.steps
        value = job_tflops(world, step_flops, ms_step)
        fwd_tf = 4 * D * pairs / (fwd_ms * 1e-3) / 1e12
        bwd_tf = 10 * D * pairs / (bwd_ms * 1e-3) / 1e12
        fwd_ktf = 4 * D * pairs / (fwd_kms * 1e-3) / 1e12
        bwd_ktf = 10 * D * pairs / (bwd_kms * 1e-3) / 1e12
        peak = peaks["bf16_tflops"]
        dominant = "bwd" if bwd_kms >= fwd_kms else "fwd"
        fwd_b, bwd_b = _alg_bytes(p)
        dom_flops = (10 if dominant == "bwd" else 4) * D * pairs
        dom_bytes = bwd_b if dominant == "bwd" else fwd_b
        dom_ms = bwd_kms if dominant == "bwd" else fwd_kms
        # below the ridge (FLOPs per algorithmic byte under peak FLOP/s over
        # peak bytes/s) the kernel is held to the HBM roofline instead
        hbm = dom_flops / dom_bytes < peak * 1e12 / (peaks["hbm_gbs"] * 1e9)
        achieved = (dom_bytes / (dom_ms * 1e-3) / 1e9 if hbm else
                    (bwd_ktf if dominant == "bwd" else fwd_ktf))
        rpeak = peaks["hbm_gbs"] if hbm else peak
        variant = (args.causal or args.deterministic or args.shared_rows or args.batch is not None
                   or args.heads is not None)
        traffic = None if variant else _traffic_from_profiles(args.config, dominant)
        bwd_name = "k_bwd_tc+k_dq_tc" if args.deterministic else "k_bwd_tc"
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if p.dtype == torch.bfloat16 else "f16", "data": "synthetic",
            "config": {"workload": _descr(args.config, args.causal, args.deterministic,
                                          args.shared_rows, args.per_head_rows)
                       + ("" if args.batch is None else f" (batch overridden to {args.batch})")
                       + ("" if args.heads is None else f" (heads overridden to {args.heads})"),
                       "kept_pairs_per_replica": pairs,
                       "parallelism": f"replicas x{world} (no exchange)",
                       "l2": "inputs larger than L2 (q/k/v/dout %d MiB each)"
                             % (q.numel() * q.element_size() >> 20)},
            "fwd_ms": round(fwd_ms, 4), "bwd_ms": round(bwd_ms, 4),
            "fwd_tflops": round(fwd_tf, 2), "bwd_tflops": round(bwd_tf, 2),
            "kernel_ms": {"k_fwd_tc": round(fwd_kms, 4), bwd_name: round(bwd_kms, 4)},
            "kernel_tflops": {"k_fwd_tc": round(fwd_ktf, 2), bwd_name: round(bwd_ktf, 2)},
            "alg_bytes": {"fwd": fwd_b, "bwd": bwd_b},
            "kernel_gbs": {"k_fwd_tc": round(fwd_b / (fwd_kms * 1e-3) / 1e9, 1),
                           bwd_name: round(bwd_b / (bwd_kms * 1e-3) / 1e9, 1)},
            "pct_of_peak": round(100 * value / world / peak, 2),
            "roofline": {"bound": "hbm" if hbm else "tensor",
                         "kernel": bwd_name if dominant == "bwd" else "k_fwd_tc",
                         "units": (f"{'backward' if dominant == 'bwd' else 'forward'} algorithmic bytes "
                                   "per launch" if hbm else
                                   f"{10 if dominant == 'bwd' else 4}*D*kept_pairs FLOPs per launch"),
                         "achieved": round(achieved, 2), "peak": rpeak,
                         "unit": "GB/s" if hbm else "TFLOP/s",
                         "frac": round(achieved / rpeak, 4),
                         "peak_source": f"{which} {'HBM copy' if hbm else 'bf16 burst'}",
                         "traffic": traffic},
            "e2e": {"value": round(job_tflops(world, step_flops, e2e_ms), 3), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": round(e2e_ms, 3)},
            "gpu_launches": launches_per_step(fwd_slots, bwd_slots, args.deterministic) * args.steps,
            "status_flags": flags,
            "clocks": clk.summary(),
        }
        if not hbm:
            line["roofline"]["frac_of_sustained"] = round(
                achieved / peaks.get("bf16_tflops_sustained", peak), 4)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(args.config, causal=args.causal,
                                                shared_rows=args.shared_rows)
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def run_fp8(args):
    """C3 with e4m3 q, k, v (bf16 out): the forward alone (the backward takes
    16-bit inputs), timed like run_ours; the roofline peak is the measured
    bf16 burst x 2 (the nominal fp8 / bf16 tensor ratio, 4.5 / 2.25 PFLOP/s)."""
    import block_sparse_variable_b200 as bsa
    import workloads

    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("--fp8 is a one-GPU line; run it without torchrun")
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    p = workloads.make_config(3, fp8=True)
    pairs = _pairs(p)
    P = bsa.params_of_problem(p)
    q, k, v, index = (getattr(p, n).to(dev) for n in ("q", "k", "v", "index"))
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    wsf = torch.empty(bsa.bsa_fwd_get_workspace(q, k, v, index, P, out=out, lse=lse),
                      dtype=torch.uint8, device=dev)
    fwd_slots = bsa.bsa_fwd_workspace_layout(q, k, v, index, P, out=out, lse=lse).fwd_items.bytes // 4
    stream = torch.cuda.current_stream()

    def step():
        bsa.bsa_fwd(q, k, v, index, P, out=out, lse=lse, workspace=wsf, stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    flags = bsa.bsa_read_status(wsf)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for e in (e for row in kev for e in row):
        e.record(stream)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with ClockSampler(0) as clk:
        start.record(stream)
        for s_ in range(args.steps):
            ev[s_][0].record(stream)
            bsa.bsa_set_main_kernel_events(kev[s_][0], kev[s_][1])
            step()
            ev[s_][1].record(stream)
        stop.record(stream)
        torch.cuda.synchronize()
    ms = start.elapsed_time(stop) / args.steps
    kms = statistics.mean(e[0].elapsed_time(e[1]) for e in kev)
    # end to end: q, k, v, index in from pinned host memory, out and lse back
    hq, hk, hv, hidx = (t.cpu().pin_memory() for t in (q, k, v, index))
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h_lse = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hidx))
    d2h = sum(t.numel() * t.element_size() for t in (h_out, h_lse))

    def e2e_step():
        for d_, h_ in ((q, hq), (k, hk), (v, hv), (index, hidx)):
            d_.copy_(h_, non_blocking=True)
        step()
        for h_, d_ in ((h_out, out), (h_lse, lse)):
            h_.copy_(d_, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(2, min(args.steps, 5))
    e0.record(stream)
    for _ in range(n_e2e):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / n_e2e
    peaks, which = _peaks()
    flops = 4 * p.D * pairs
    peak = 2 * peaks["bf16_tflops"]
    ktf = flops / (kms * 1e-3) / 1e12
    line = {
        "metric": "effective TFLOP/s (selected blocks only), FP8 forward", "value": round(flops / (ms * 1e-3) / 1e12, 3),
        "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3", "data": "synthetic",
        "config": {"workload": DESCR[3] + ", q/k/v e4m3 (bf16 out), forward only",
                   "kept_pairs_per_replica": pairs, "parallelism": "replicas x1 (no exchange)",
                   "l2": "inputs larger than L2 (q/k/v %d MiB each)" % (q.numel() >> 20)},
        "kernel_ms": {"k_fwd_tc": round(kms, 4)}, "kernel_tflops": {"k_fwd_tc": round(ktf, 2)},
        "roofline": {"bound": "tensor", "kernel": "k_fwd_tc", "units": "4*D*kept_pairs FLOPs per launch",
                     "achieved": round(ktf, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(ktf / peak, 4),
                     "peak_source": f"{which} bf16 burst x 2 (nominal fp8/bf16 ratio)", "traffic": None},
        "e2e": {"value": round(flops / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 3)},
        "gpu_launches": (3 + _sort_launches(fwd_slots)) * args.steps, "status_flags": flags,
        "clocks": clk.summary(),
    }
    if not args.no_cpu_baseline:
        import oracle

        def fwd_time(sub):
            t = time.perf_counter()
            oracle.Oracle(sub).fwd()
            return time.perf_counter() - t
        t = fwd_time(_oracle_subproblem(3, 1024, fp8=True))
        sub = _oracle_subproblem(3, int(1024 * max(1.0, 12.0 / max(t, 1e-3))), fp8=True)
        t = fwd_time(sub)
        line["cpu_baseline"] = {"value": 4 * sub.D * _pairs(sub) / t / 1e12, "unit": "TFLOP/s",
                                "cores": _omp_threads(), "kind": "oracle",
                                "sample": f"fp64 oracle forward on batch 0, {_heads_of(sub)}, first "
                                          f"{sub.q.shape[2]} query rows x {sub.k.shape[2]} keys ({t:.1f} s)"}
    print(json.dumps(line), flush=True)


def _traffic_from_profiles(cfg, which):
    """DRAM bytes per launch of the dominant kernel from a committed ncu summary."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d.get(f"C{cfg}", {}).get(which)
    except (OSError, ValueError):
        return None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=lambda s: int(s.lstrip("Cc")), default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=None,
                    help="smaller batch for C3/C4 (profiler captures only; not a bench line)")
    ap.add_argument("--heads", type=int, default=None,
                    help="fewer heads for C3/C4 (profiler captures only; not a bench line)")
    ap.add_argument("--causal", action="store_true",
                    help="C3 with the causal mask and its lower-triangular block index")
    ap.add_argument("--deterministic", action="store_true",
                    help="the deterministic backward (bitwise reproducible dq)")
    ap.add_argument("--fp8", action="store_true",
                    help="C3 with e4m3 q/k/v: the FP8 forward alone (one GPU)")
    ap.add_argument("--shared-rows", action="store_true",
                    help="C2/C5 with one index row per GQA group (packed forward tiles)")
    ap.add_argument("--per-head-rows", action="store_true",
                    help="with --shared-rows: the same rows copied to every query head")
    args = ap.parse_args()
    if args.causal and args.config != 3:
        ap.error("--causal applies to C3")
    if args.shared_rows and args.config not in (2, 5):
        ap.error("--shared-rows applies to C2 and C5")
    if args.per_head_rows and not args.shared_rows:
        ap.error("--per-head-rows needs --shared-rows")
    if args.impl == "reference":
        run_reference(args)
    elif args.fp8:
        run_fp8(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
