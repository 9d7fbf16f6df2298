"""Benchmark of one decode step of load-balanced split-KV attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload extreme] [--impl ours|reference]

A step is the whole hot path over one batch: the per-step device planner, the persistent
attention kernel and the log-sum-exp merge, plus the fused prologue for the FP8
workload. The default workload is the mixed-length batch the dynamic scheduler targets:
1 x 131072 + 31 x 4096 tokens, 64 q / 8 kv heads, head dim 128, page 64, bf16 KV. The
KV cache (1.06 GB) is larger than L2, so there is no flush between steps.

Rank 0 prints one JSON line. ``value`` is the effective GB/s over the algorithmic bytes
(valid KV + q + out), summed over ranks. The timed region is K eager steps on one stream,
bracketed by a barrier and synchronize, timed with CUDA events. Under torchrun, each rank
runs an independent replica: the workload has no cross-GPU exchange.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from load_balanced_split_step_b200 import workloads as W  # noqa: E402

WORKLOAD_TEXT = {
    "tiny": "tiny: 4 requests {17,64,200,513}, 8 q / 2 kv heads, D 64, page 16, bf16 KV",
    "uniform": "uniform: 32 x 4096 tokens, 64 q / 8 kv heads, D 128, page 64, bf16 KV",
    "extreme": "extreme mixed: 1 x 131072 + 31 x 4096 tokens, 64 q / 8 kv heads, D 128, page 64, bf16 KV",
    "heavy": "heavy-tailed: 64 requests, L log-uniform [512, 65536), +1 per step over 8 steps, 64/8 heads, D 128, "
             "page 64, bf16 KV",
    "fp8": "large batch FP8: 256 requests, L ~ U[1024, 16384], 64/8 heads, D 128, page 64, E4M3 KV + fused "
           "RoPE/QK-RMSNorm/KV-write prologue",
}
METRIC = "decode-attention KV-read GB/s (effective, algorithmic KV+Q+O bytes / step time) on mixed-length batches"
CLOCK_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="extreme", choices=list(WORKLOAD_TEXT))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--tile-len", type=int, default=0)
    ap.add_argument("--ctas-per-sm", type=int, default=1)
    ap.add_argument("--layout", default="HND", choices=["HND", "NHD"], help="KV cache page layout")
    ap.add_argument("--path", default="fused", choices=["fused", "folded", "split"],
                    help="fused: one launch per step (in-kernel plan + ticket merge), after the prologue kernel on "
                         "the FP8 workload; folded: the same with the prologue folded into that launch; split: "
                         "plan, attention and merge kernels")
    ap.add_argument("--requests", type=int, default=0,
                    help="run only the first N requests of the workload (a bounded sample, e.g. for a profiler)")
    ap.add_argument("--q-len", type=int, default=1,
                    help="new tokens per request, attending causally (1 to 4; single-launch path)")
    ap.add_argument("--shard", action="store_true",
                    help="request-sharded placement of ONE batch over the ranks (strong scaling): each rank runs its "
                         "parts, (out, lse) are all-gathered and split requests merged; default: independent replicas")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the graph, distribution, static split-k, CPU baseline and other-workload legs")
    ap.add_argument("--item-cost", type=int, default=None,
                    help="single-launch split: cost of an item start in 1/16 tile (default: the library's)")
    ap.add_argument("--e4m3-kernel", default="mma", choices=["mma", "tcgen05"], help="kernel for E4M3 caches")
    ap.add_argument("--multi-kernel", default="default", choices=["default", "mma", "tcgen05"],
                    help="kernel for several new tokens per request (--q-len > 1)")
    ap.add_argument("--record-traffic", default=None, metavar="CSV",
                    help="write profiles/traffic.json's entry for --workload from an ncu CSV of one attention launch "
                         "(dram__bytes_read.sum, dram__bytes_write.sum); with --requests N the capture covered the "
                         "first N requests and is scaled to the full workload by algorithmic bytes")
    ap.add_argument("--trace", action="store_true",
                    help="run the HPC_TRACE build of the library and print a per-CTA load summary of the single "
                         "launch (idle tail, plan and first-data latency) instead of the benchmark line")
    return ap.parse_args(argv)


# ------------------------------------------------------------------------- distributed

def dist_init(args):
    """Returns (rank, world, local_rank). One process per GPU under torchrun."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        local = int(os.environ.get("LOCAL_RANK", "0"))
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
        return dist.get_rank(), world, local
    return 0, 1, 0


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank float over all ranks (identity for one rank)."""
    if world == 1:
        return float(x)
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_done(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampling every 200 ms while the timed region runs."""

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={CLOCK_QUERY}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "200"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
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
            self.f.close()

    def summary(self):
        if self.proc is None or not self.path:
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------------------- our arm

class Step:
    """One decode step through the binding, with buffers allocated once."""

    def __init__(self, B, spec, dc, num_ctas, tile_len, static_splits=None, fused=False, layout="HND",
                 folded=False, item_cost=None, e4m3_kernel="mma", multi_kernel="default"):
        self.B, self.spec, self.dc = B, spec, dc
        self.item_cost, self.e4m3_kernel, self.multi_kernel = item_cost, e4m3_kernel, multi_kernel
        self.trace = None  # HPC_TRACE builds only: per-CTA stamps of the single-launch step
        self.layout = layout
        self.tl = tile_len
        self.fused = (fused or folded) and not static_splits
        self.folded = folded and self.fused and spec.prologue
        dev = dc["seq_lens"].device
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.max_seq = dc["block_table"].shape[1] * spec.page_size
        if static_splits:
            self.plan = B.plan_static(dc["seq_lens"], spec.num_heads, spec.kv_heads, tile_len, static_splits,
                                      self.max_seq, self.status)
            self.static_splits = static_splits
        else:
            self.plan = B.plan(dc["seq_lens"], spec.num_heads, spec.kv_heads, tile_len, num_ctas, self.max_seq,
                               self.status)
            self.static_splits = None
        self.num_ctas = num_ctas
        self.po, self.pml = B.partial_buffers(self.plan, spec.num_heads, spec.head_dim, dev)
        if self.fused:
            self.ws = B.multi_workspace(spec.batch, spec.q_len, spec.num_heads, spec.kv_heads, spec.head_dim,
                                        num_ctas, dev)
        qshape = (spec.batch, spec.num_heads, spec.head_dim) if spec.q_len == 1 else \
            (spec.batch, spec.q_len, spec.num_heads, spec.head_dim)
        self.out = torch.empty(qshape, dtype=torch.float32, device=dev)
        self.q = dc["q"]
        if spec.prologue:
            self.q = torch.empty((spec.batch, spec.num_heads, spec.head_dim), dtype=torch.bfloat16, device=dev)

    def __call__(self, seq_lens=None, ev=None):
        B, s, dc = self.B, self.spec, self.dc
        seq = dc["seq_lens"] if seq_lens is None else seq_lens
        if self.folded:  # one launch: the prologue is folded into the step
            if ev is not None:
                ev[0].record()
            B.decode_step_prologue(dc["qkv"], dc["q_norm_w"], dc["k_norm_w"], dc["k_pages"], dc["v_pages"],
                                   dc["block_table"], seq, s.num_heads, s.kv_heads, self.tl, kv_dtype=s.kv_dtype,
                                   kv_layout=self.layout, k_scale=dc["k_scale"], v_scale=dc["v_scale"],
                                   eps=s.rms_eps, rope_theta=s.rope_theta, num_ctas=self.num_ctas, out=self.out,
                                   status=self.status, workspace=self.ws, item_cost=self.item_cost,
                                   trace=self.trace, seq_lens_ready=True)
            if ev is not None:
                ev[1].record()
            return self.out
        if s.prologue:
            B.prologue(dc["qkv"], dc["q_norm_w"], dc["k_norm_w"], dc["k_pages"], dc["v_pages"], dc["block_table"],
                       seq, s.num_heads, s.kv_heads, kv_dtype=s.kv_dtype, kv_layout=self.layout, k_scale=dc["k_scale"],
                       v_scale=dc["v_scale"], eps=s.rms_eps, rope_theta=s.rope_theta, q_out=self.q,
                       status=self.status)
        if self.fused and s.q_len > 1:
            if ev is not None:
                ev[0].record()
            B.decode_step_multi(self.q, dc["k_pages"], dc["v_pages"], dc["block_table"], seq, s.kv_heads, self.tl,
                                kv_dtype=s.kv_dtype, kv_layout=self.layout, k_scale=dc["k_scale"],
                                v_scale=dc["v_scale"], num_ctas=self.num_ctas, out=self.out, status=self.status,
                                workspace=self.ws, item_cost=self.item_cost, trace=self.trace,
                                multi_kernel=self.multi_kernel, seq_lens_ready=True)
            if ev is not None:
                ev[1].record()
            return self.out
        if self.fused:
            if ev is not None:
                ev[0].record()
            B.decode_step_fused(self.q, dc["k_pages"], dc["v_pages"], dc["block_table"], seq, s.num_heads,
                                s.kv_heads, self.tl, kv_dtype=s.kv_dtype, kv_layout=self.layout, k_scale=dc["k_scale"],
                                v_scale=dc["v_scale"], num_ctas=self.num_ctas, out=self.out, status=self.status,
                                workspace=self.ws, item_cost=self.item_cost, e4m3_kernel=self.e4m3_kernel,
                                trace=self.trace, seq_lens_ready=True)
            if ev is not None:
                ev[1].record()
            return self.out
        if self.static_splits:
            B.plan_static(seq, s.num_heads, s.kv_heads, self.tl, self.static_splits, self.max_seq, self.status,
                          workspace=self.plan.workspace)
        else:
            B.plan(seq, s.num_heads, s.kv_heads, self.tl, self.num_ctas, self.max_seq, self.status,
                   workspace=self.plan.workspace)
        if ev is not None:
            ev[0].record()
        B.attention(self.q, dc["k_pages"], dc["v_pages"], dc["block_table"], seq, self.plan, kv_dtype=s.kv_dtype,
                    kv_layout=self.layout, k_scale=dc["k_scale"], v_scale=dc["v_scale"], out=self.out, partial_o=self.po,
                    partial_ml=self.pml, status=self.status, e4m3_kernel=self.e4m3_kernel)
        if ev is not None:
            ev[1].record()
        B.merge(self.plan, self.po, self.pml, self.out, s.num_heads, self.status)
        return self.out

    @property
    def launches(self):
        pro = 1 if self.spec.prologue and not self.folded else 0
        return (1 if self.fused else 3) + pro


class ShardStep:
    """The step of one batch placed over the ranks by request (load_balanced_split_step_b200.shard):
    the placement follows this step's lengths (kept, or made again past the drift bound), the
    rank's block-table view is rebuilt on the device (hpc_gather_pages), q rows of the local
    parts gathered (hpc_gather_rows), the parts through hpc_decode_step_lse, one all-gather of
    (out, lse), every request formed from its parts (hpc_merge_lse_gather)."""

    def __init__(self, B, spec, dc, num_ctas, tile_len, rank, world, lens_dev):
        from load_balanced_split_step_b200 import shard as SH
        self.spec, self.dc, self.tl = spec, dc, tile_len
        self.status = torch.zeros(1, dtype=torch.int32, device=dc["seq_lens"].device)
        compute = SH.library_compute(spec.num_heads, spec.kv_heads, kv_dtype=spec.kv_dtype, k_scale=dc["k_scale"],
                                     v_scale=dc["v_scale"], num_ctas=num_ctas, status=self.status)
        self.st = SH.ShardedStep(spec.seq_lens, world, rank, spec.page_size, spec.num_heads, spec.head_dim,
                                 compute=compute, merge=SH.library_merge(self.status),
                                 gather=SH.library_gather(self.status), pages=SH.library_pages(self.status))
        # the host knows each step's lengths (a serving loop's scheduler does): decode step i of the
        # workload has seq_lens + i
        self.host_lens = {id(t): [L + i for L in spec.seq_lens] for i, t in enumerate(lens_dev)}
        self.out = None

    def __call__(self, seq_lens=None, ev=None, q=None):
        d = self.dc
        host = self.host_lens.get(id(seq_lens)) if seq_lens is not None else None
        if ev is not None:
            ev[0].record()
        self.out = self.st.step(d["q"] if q is None else q, d["k_pages"], d["v_pages"], d["block_table"], self.tl,
                                seq_lens=host)
        if ev is not None:
            ev[1].record()
        return self.out

    @property
    def launches(self):
        local = 3 if self.st.plan[self.st.rank] else 0  # page view, q gather and the step, when the rank has parts
        return local + 1  # then the indexed merge


def step_lengths(dc, spec):
    """Device length vectors for each decode step (heavy-tailed grows by one per step)."""
    return [dc["seq_lens"] + i for i in range(spec.steps)]


def time_steps(step, lens, K, W_, world, kernel_events=True):
    for i in range(W_):
        step(lens[i % len(lens)])
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)] \
        if kernel_events else [None] * K
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(K):
        step(lens[i % len(lens)], ev[i])
    t1.record()
    torch.cuda.synchronize()
    barrier(world)
    total_ms = t0.elapsed_time(t1)
    kern_ms = float(np.mean([a.elapsed_time(b) for a, b in ev])) if kernel_events else None
    return total_ms, kern_ms


def step_distribution(step, lens, n, world):
    """Distribution of single-step times: CUDA events around each whole step on the launching
    stream, after three untimed steps. The events between steps stop one step's launch from
    overlapping the previous one's tail, so the median sits slightly above the back-to-back mean.
    A workload of several decode steps (lengths growing by one) also gets each step's mean."""
    for i in range(3):
        step(lens[i % len(lens)])
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for i in range(n):
        ev[i][0].record()
        step(lens[i % len(lens)])
        ev[i][1].record()
    torch.cuda.synchronize()
    us = np.array([1000.0 * a.elapsed_time(b) for a, b in ev])
    p10, p50, p90 = (max_over_ranks(float(np.percentile(us, q)), world) for q in (10, 50, 90))
    out = {"reps": n, "median_us": round(p50, 2), "p10_us": round(p10, 2), "p90_us": round(p90, 2),
           "note": "events around every step (max over ranks)"}
    if len(lens) > 1:
        out["per_step_mean_us"] = [round(max_over_ranks(float(us[i::len(lens)].mean()), world), 2)
                                   for i in range(len(lens))]
    return out


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def static_leg(B, spec, dc, tl, steps, sms, layout="HND"):
    S0 = max(1, -(-2 * sms // (spec.batch * spec.kv_heads)))
    res = {}
    lens = step_lengths(dc, spec)
    for S in sorted({S0, 1, 2, 4, 8, 16, 32}):
        st = Step(B, spec, dc, None, tl, static_splits=S, layout=layout)
        ms, _ = time_steps(st, lens, steps, 3, 1, kernel_events=False)
        res[S] = 1000.0 * ms / steps
    best = min(res, key=res.get)
    return {"splits_rule": "S = max(1, ceil(2*SMs/(B*Hkv)))", "S": S0, "us_per_step": round(res[S0], 2),
            "best_S": best, "best_us_per_step": round(res[best], 2),
            "sweep_us": {str(k): round(v, 2) for k, v in res.items()}}


def shard_e2e_leg(step, case, dc, steps, world):
    """The sharded step with q copied in from pinned host memory and the output copied out every
    step, overlapped as in e2e_leg: copy-in, compute (the exchange included) and copy-out
    streams with two buffer sets, ordered by events."""
    dev = dc["seq_lens"].device
    q_host = case.q.pin_memory()
    nbuf = 2
    q_dev = [torch.empty_like(q_host, device=dev) for _ in range(nbuf)]
    hosts = [torch.empty(tuple(q_host.shape), dtype=torch.float32).pin_memory() for _ in range(nbuf)]
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(nbuf)]
    ev_cmp = [torch.cuda.Event() for _ in range(nbuf)]
    ev_out = [torch.cuda.Event() for _ in range(nbuf)]

    def one(i):
        b = i % nbuf
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_cmp[b])  # step i-2 has finished reading this q buffer
            q_dev[b].copy_(q_host, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[b])
            s_cmp.wait_event(ev_out[b])  # step i-2's output has left its host buffer
            out = step(q=q_dev[b])
            ev_cmp[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[b])
            out.record_stream(s_out)  # allocated on the compute stream, read here
            hosts[b].copy_(out, non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(4):
        one(i)
    torch.cuda.synchronize()
    barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    for i in range(steps):
        one(i)
    t1.record(s_out)
    torch.cuda.synchronize()
    barrier(world)
    return t0.elapsed_time(t1), q_host.numel() * q_host.element_size(), hosts[0].numel() * hosts[0].element_size()


def e2e_leg(B, spec, case, dc, tl, num_ctas, steps, world, fused=True, layout="HND", folded=False,
            multi_kernel="default"):
    """Same metric through the public call, with per-step H2D of the step inputs (q or qkv,
    seq_lens, block_table) from pinned host memory and D2H of the output. The KV cache is
    device-resident decode state and is not copied. The step runs as a serving loop would:
    copy-in, compute and copy-out streams with two buffer sets. Step i+1's inputs arrive and
    step i-1's output leaves while step i computes, ordered by events. Every step still
    copies its own inputs in and its own result out."""
    dev = dc["seq_lens"].device
    src = {"seq_lens": case.seq_lens.pin_memory(), "block_table": case.block_table.pin_memory()}
    qname = "qkv" if spec.prologue else "q"
    src[qname] = getattr(case, qname).pin_memory()
    shape = (spec.batch, spec.num_heads, spec.head_dim) if spec.q_len == 1 else \
        (spec.batch, spec.q_len, spec.num_heads, spec.head_dim)
    nbuf = 2
    dsts = [{k: torch.empty_like(v, device=dev) for k, v in src.items()} for _ in range(nbuf)]
    outs = [torch.empty(shape, dtype=torch.float32, device=dev) for _ in range(nbuf)]
    hosts = [torch.empty(shape, dtype=torch.float32).pin_memory() for _ in range(nbuf)]
    qbufs = [torch.empty(shape, dtype=torch.bfloat16, device=dev) for _ in range(nbuf)]
    ws = B.multi_workspace(spec.batch, spec.q_len, spec.num_heads, spec.kv_heads, spec.head_dim, num_ctas, dev) \
        if fused else None
    h2d = sum(v.numel() * v.element_size() for v in src.values())
    d2h = hosts[0].numel() * hosts[0].element_size()
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(nbuf)]
    ev_cmp = [torch.cuda.Event() for _ in range(nbuf)]
    ev_out = [torch.cuda.Event() for _ in range(nbuf)]

    def one(i):
        b = i % nbuf
        d = dict(dc)
        d.update(dsts[b])
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_cmp[b])  # step i-2 has finished reading this input set
            for k in src:
                dsts[b][k].copy_(src[k], non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[b])
            s_cmp.wait_event(ev_out[b])  # step i-2's output has left this buffer
            q = d["q"]
            if folded and spec.prologue:
                B.decode_step_prologue(d["qkv"], d["q_norm_w"], d["k_norm_w"], d["k_pages"], d["v_pages"],
                                       d["block_table"], d["seq_lens"], spec.num_heads, spec.kv_heads, tl,
                                       kv_dtype=spec.kv_dtype, kv_layout=layout, k_scale=d["k_scale"],
                                       v_scale=d["v_scale"], eps=spec.rms_eps, rope_theta=spec.rope_theta,
                                       num_ctas=num_ctas, out=outs[b], workspace=ws, seq_lens_ready=True)
            elif spec.prologue:
                q = B.prologue(d["qkv"], d["q_norm_w"], d["k_norm_w"], d["k_pages"], d["v_pages"], d["block_table"],
                               d["seq_lens"], spec.num_heads, spec.kv_heads, kv_dtype=spec.kv_dtype, kv_layout=layout,
                               k_scale=d["k_scale"], v_scale=d["v_scale"], eps=spec.rms_eps,
                               rope_theta=spec.rope_theta, q_out=qbufs[b])
            if folded and spec.prologue:
                pass  # done above, in one launch
            elif fused and spec.q_len > 1:
                B.decode_step_multi(q, d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"], spec.kv_heads, tl,
                                    kv_dtype=spec.kv_dtype, kv_layout=layout, k_scale=d["k_scale"],
                                    v_scale=d["v_scale"], num_ctas=num_ctas, out=outs[b], workspace=ws,
                                    multi_kernel=multi_kernel, seq_lens_ready=True)
            elif fused:
                B.decode_step_fused(q, d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"], spec.num_heads,
                                    spec.kv_heads, tl, kv_dtype=spec.kv_dtype, kv_layout=layout, k_scale=d["k_scale"],
                                    v_scale=d["v_scale"], num_ctas=num_ctas, out=outs[b], workspace=ws,
                                    seq_lens_ready=True)
            else:
                B.decode_step(q, d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"], spec.num_heads,
                              spec.kv_heads, tl, kv_dtype=spec.kv_dtype, kv_layout=layout, k_scale=d["k_scale"],
                              v_scale=d["v_scale"],
                              num_ctas=num_ctas, out=outs[b])
            ev_cmp[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[b])
            hosts[b].copy_(outs[b], non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(4):
        one(i)
    torch.cuda.synchronize()
    barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    for i in range(steps):
        one(i)
    t1.record(s_out)
    torch.cuda.synchronize()
    barrier(world)
    return t0.elapsed_time(t1), h2d, d2h


# ------------------------------------------------------------------ CPU baseline (the oracle)
#
# The fp64 oracle, as it stands, on a fixed stratified sample of the workload: kv head g of
# request r is in the sample when (g - r) % S == 0, S = min(4, kv_heads), so every request (the
# 128K one of the extreme batch included) contributes the same fraction of its tokens. The
# sample's (request, query head) pairs are the units of work. A pool of single-threaded worker
# processes (started with spawn; BLAS and torch limited to one thread each) takes them from a
# shared queue, longest first; the sample's pages sit in one shared-memory block that the
# workers map without copying. The timed region is one pass over the units.

_CPU = {}


def _cpu_worker_init(shm_name, nbytes):
    import torch
    torch.set_num_threads(1)
    try:
        from threadpoolctl import threadpool_limits
        _CPU["limits"] = threadpool_limits(1)
    except Exception:
        pass
    from multiprocessing import shared_memory
    shm = shared_memory.SharedMemory(name=shm_name)
    _CPU["shm"] = shm
    _CPU["buf"] = np.ndarray((nbytes,), dtype=np.uint8, buffer=shm.buf)
    from oracle import attention  # noqa: F401  (imported before the timed pass)


def _cpu_ready(_):
    return os.getpid()


def _cpu_unit(task):
    """One (request, query head) of the sample through oracle.attention.decode_attention."""
    import torch
    from oracle import attention as OA
    k_off, v_off, n_pages, P, D, L, kv_dtype, q_row, k_s, v_s, scale = task
    buf = _CPU["buf"]
    elt = 1 if kv_dtype == "e4m3" else 2
    n = n_pages * P * D * elt
    if kv_dtype == "e4m3":
        kp = buf[k_off:k_off + n].reshape(n_pages, 1, P, D)
        vp = buf[v_off:v_off + n].reshape(n_pages, 1, P, D)
    else:
        kp = torch.from_numpy(buf[k_off:k_off + n]).view(torch.bfloat16).reshape(n_pages, 1, P, D)
        vp = torch.from_numpy(buf[v_off:v_off + n]).view(torch.bfloat16).reshape(n_pages, 1, P, D)
    q = np.asarray(q_row, dtype=np.float64).reshape(1, 1, D)
    bt = np.arange(n_pages, dtype=np.int64)[None, :]
    t0 = time.perf_counter()
    OA.decode_attention(q, kp, vp, bt, np.array([L]), sm_scale=scale, kv_dtype=kv_dtype, k_scale=[k_s],
                        v_scale=[v_s])
    return time.perf_counter() - t0


class CpuBaseline:
    """The oracle on the host cores over a fixed stratified sample of one workload (see above)."""

    def __init__(self, spec, case, max_workers=32):
        from multiprocessing import shared_memory
        Hkv, grp, D, P = spec.kv_heads, spec.group, spec.head_dim, spec.page_size
        S = min(4, Hkv)
        pairs = [(r, g) for r in range(spec.batch) for g in range(Hkv) if (g - r) % S == 0 and spec.seq_lens[r] > 0]
        kp, vp, q, bt = case.k_pages, case.v_pages, case.q, case.block_table
        self.prologue_note = ""
        if spec.prologue:
            # q and the new token's K/V come from the oracle's own prologue, outside the timed pass
            from oracle import prologue as OR
            kpn, vpn = case.k_pages.numpy().copy(), case.v_pages.numpy().copy()
            qo = OR.decode_prologue(case.qkv, case.q_norm_w, case.k_norm_w, spec.rms_eps, spec.rope_theta,
                                    case.seq_lens.numpy(), case.block_table.numpy(), kpn, vpn, spec.kv_dtype,
                                    case.k_scale, case.v_scale, spec.num_heads, Hkv)[0]
            kp, vp, q = torch.from_numpy(kpn), torch.from_numpy(vpn), qo
            self.prologue_note = "; q and the new token's K/V from the oracle's prologue, untimed (<1% of the work)"
        qf = q.to(torch.float64).numpy() if isinstance(q, torch.Tensor) else np.asarray(q, dtype=np.float64)
        elt = 1 if spec.kv_dtype == "e4m3" else 2
        blocks, tasks, off = [], [], 0
        ks = case.k_scale.double().numpy() if case.k_scale is not None else np.ones(Hkv)
        vs = case.v_scale.double().numpy() if case.v_scale is not None else np.ones(Hkv)
        self.bytes = 0
        self.tokens = 0
        for r, g in pairs:
            L = spec.seq_lens[r]
            npg = -(-L // P)
            rows = bt[r, :npg].long()
            kb = kp[rows, g].contiguous().view(torch.uint8).numpy().reshape(-1)
            vb = vp[rows, g].contiguous().view(torch.uint8).numpy().reshape(-1)
            blocks += [kb, vb]
            for h in range(g * grp, (g + 1) * grp):
                tasks.append((off, off + kb.size, npg, P, D, L, spec.kv_dtype, qf[r, h].tolist(), float(ks[g]),
                              float(vs[g]), spec.sm_scale))
            off += kb.size + vb.size
            self.bytes += L * D * elt * 2 + grp * D * (2 + 4)
            self.tokens += L
        tasks.sort(key=lambda t: -t[5])  # longest first: the queue then balances the workers
        self.tasks = tasks
        self.pairs = len(pairs)
        self.frac = self.bytes / W.algorithmic_bytes(spec)
        self.nbytes = max(off, 1)
        self.shm = shared_memory.SharedMemory(create=True, size=self.nbytes)
        buf = np.ndarray((self.nbytes,), dtype=np.uint8, buffer=self.shm.buf)
        pos = 0
        for b in blocks:
            buf[pos:pos + b.size] = b
            pos += b.size
        del buf
        try:
            avail = len(os.sched_getaffinity(0))
        except AttributeError:
            avail = os.cpu_count() or 1
        self.workers = max(1, min(avail, max_workers, len(tasks)))
        import multiprocessing as mp
        self.pool = mp.get_context("spawn").Pool(self.workers, initializer=_cpu_worker_init,
                                                 initargs=(self.shm.name, self.nbytes))
        self.pool.map(_cpu_ready, range(4 * self.workers), chunksize=1)  # every worker up and imported
        self.S = S

    def run(self):
        """One timed pass over the sample: (GB/s of algorithmic bytes, seconds)."""
        t0 = time.perf_counter()
        self.pool.map(_cpu_unit, self.tasks, chunksize=1)
        el = time.perf_counter() - t0
        return self.bytes / el / 1e9, el

    def describe(self, el):
        return (f"kv heads g of request r with (g - r) % {self.S} == 0: {self.pairs} (request, kv head) pairs, "
                f"{len(self.tasks)} (request, query head) units, {self.frac:.3f} of one step's algorithmic bytes, "
                f"every request in proportion; one pass in {el:.1f} s on {self.workers} single-threaded worker "
                f"processes{self.prologue_note}")

    def close(self):
        self.pool.close()
        self.pool.join()
        self.shm.close()
        self.shm.unlink()


def cpu_baseline(spec, case, passes=3):
    """The oracle on the host cores: the median of `passes` timed passes over the stratified
    sample. Returns the cpu_baseline object of the JSON line."""
    cb = CpuBaseline(spec, case)
    try:
        runs = sorted(cb.run() for _ in range(passes))
        v, el = runs[len(runs) // 2]
        return {"value": round(v, 4), "unit": "GB/s", "cores": cb.workers, "kind": "oracle",
                "sample": cb.describe(el) + f"; median of {passes} passes", "cpu_model": cpu_model(),
                "host_cores": os.cpu_count()}
    finally:
        cb.close()


def qlen_text(args):
    t = "" if args.q_len == 1 else f"; {args.q_len} new tokens per request, causal among themselves"
    return t + (f"; first {args.requests} requests only" if args.requests else "")


def workload_spec(args):
    """The named workload, with q_len new tokens per request when --q-len > 1, and only its
    first --requests requests when that is set."""
    from dataclasses import replace
    spec = W.config_spec(args.workload)
    if args.requests and args.requests < spec.batch:
        spec = replace(spec, seq_lens=tuple(spec.seq_lens[:args.requests]),
                       name=f"{spec.name}, first {args.requests} requests")
    if args.q_len != 1:
        if spec.prologue:
            raise SystemExit("--q-len > 1 is not combined with the prologue workload")
        spec = replace(spec, q_len=args.q_len, name=f"{spec.name}, {args.q_len} new tokens per request")
    return spec


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def uses_tcgen05_multi(spec, multi_kernel):
    """Whether a several-token step runs the tcgen05 kernel: asked for, or the library's default
    for three or four tokens on a bf16 cache with head_dim 128 and q_len x group <= 32."""
    if spec.q_len == 1:
        return False
    fits = spec.kv_dtype == "bf16" and spec.head_dim == 128 and spec.q_len * (spec.num_heads // spec.kv_heads) <= 32
    return fits and (multi_kernel == "tcgen05" or (multi_kernel == "default" and spec.q_len >= 3))


def traffic_key(workload, q_len):
    """profiles/traffic.json key: the workload name, with _q<T> for T new tokens per request."""
    return workload if q_len == 1 else f"{workload}_q{q_len}"


def kernel_source_hash(key="extreme"):
    """Hash of the sources of the kernel that the traffic entry `key` measured: the several-token
    tcgen05 kernel for the four-token entry (its default kernel), the single-launch kernel for
    the others."""
    import hashlib
    h = hashlib.sha256()
    main = "attention_tcm.cu" if key.endswith(("_q3", "_q4")) else "attention.cu"
    for name in (main, "attention_common.cuh", "hpc_common.cuh"):
        with open(os.path.join(ROOT, "load_balanced_split_step_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic(workload):
    """DRAM bytes per attention launch at this workload's full size, from profiles/traffic.json
    (written by --record-traffic from a 1-pass ncu capture of dram bytes), or
    None when the kernel source has changed since those counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        entry = json.load(f).get(workload)
    if not entry or entry.get("source_sha256_16") != kernel_source_hash(workload):
        return None
    return int(entry["traffic_bytes_per_launch"])


def record_traffic(args):
    """profiles/traffic.json entry of --workload from an ncu CSV (see --record-traffic)."""
    import csv
    units = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6, "GB": 1e9}
    got = {}
    with open(args.record_traffic) as f:
        rows = [ln for ln in f if ln.startswith('"')]
    for row in csv.DictReader(rows):
        name = row.get("Metric Name")
        if name in ("dram__bytes_read.sum", "dram__bytes_write.sum") and name not in got:
            got[name] = float(row["Metric Value"].replace(",", "")) * units.get(row["Metric Unit"], 1)
    if len(got) != 2:
        raise SystemExit(f"{args.record_traffic}: no dram__bytes_read.sum / dram__bytes_write.sum rows")
    from dataclasses import replace
    sample = workload_spec(args)
    full = W.config_spec(args.workload)
    if args.q_len > 1:
        full = replace(full, q_len=args.q_len)
    scale = W.algorithmic_bytes(full) / W.algorithmic_bytes(sample)
    traffic = (got["dram__bytes_read.sum"] + got["dram__bytes_write.sum"]) * scale
    p = os.path.join(ROOT, "profiles", "traffic.json")
    data = json.load(open(p)) if os.path.exists(p) else {}
    key = traffic_key(args.workload, args.q_len)
    if args.q_len > 1 and args.multi_kernel != "default":
        raise SystemExit("--record-traffic with --q-len > 1 records the default kernel only")
    data[key] = {"traffic_bytes_per_launch": int(round(traffic)), "source_sha256_16": kernel_source_hash(key),
                           "read_bytes": int(got["dram__bytes_read.sum"]), "write_bytes": int(got["dram__bytes_write.sum"]),
                           "captured_requests": sample.batch, "scale_to_full": round(scale, 6),
                           "algorithmic_bytes_full": int(W.algorithmic_bytes(full))}
    with open(p, "w") as f:
        json.dump(data, f, indent=1, sort_keys=True)
        f.write("\n")
    return {"workload": key, **data[key]}


def device_case(case, dev, layout="HND"):
    dc = {k: (getattr(case, k).to(dev) if getattr(case, k) is not None else None)
          for k in ("q", "qkv", "k_pages", "v_pages", "block_table", "seq_lens", "k_scale", "v_scale", "q_norm_w",
                    "k_norm_w")}
    if layout == "NHD":  # same tokens, vLLM page layout [pages][P][Hkv][D]
        dc["k_pages"] = dc["k_pages"].permute(0, 2, 1, 3).contiguous()
        dc["v_pages"] = dc["v_pages"].permute(0, 2, 1, 3).contiguous()
    return dc


def measure(step, spec, lens, K, W_, world, local, jobs=1, per_gpu_div=1):
    """K back-to-back steps (the step time), then K more with events around the attention launch
    (its own duration, for the roofline), with clocks sampled throughout. Returns a dict."""
    with ClockSampler(local) as clk:
        # the step as a user runs it: kernels back to back, chained by programmatic dependent launch
        total_ms, _ = time_steps(step, lens, K, W_, world, kernel_events=False)
        # the same steps again with CUDA events around each attention launch (on the launching
        # stream) for the kernel's own duration; events between kernels break the launch overlap,
        # so this loop is not the step time
        _, kern_ms = time_steps(step, lens, K, 0, world, kernel_events=True)
    st = int(step.status.item())
    if st:
        raise RuntimeError(f"device status {st:#x} during the timed region")
    total_ms = max_over_ranks(total_ms, world)
    kern_ms = max_over_ranks(kern_ms, world)
    bytes_step = float(np.mean([W.algorithmic_bytes(spec, i % spec.steps) for i in range(spec.steps)]))
    peak, peak_kind = load_peaks()
    achieved = bytes_step / per_gpu_div / (kern_ms / 1e3) / 1e9
    return {"total_ms": total_ms, "kern_ms": kern_ms, "bytes_step": bytes_step, "K": K, "W": W_,
            "value": jobs * bytes_step * K / (total_ms / 1e3) / 1e9, "ms_step": total_ms / K,
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                         "frac_of_nominal_8000": round(achieved / 8000.0, 4), "kernel_us": round(1000 * kern_ms, 2)},
            "clocks": clk.summary()}


OTHER_WORKLOADS = ("uniform", "heavy", "fp8", "heavy_q4")


def other_workload(B, args, name, dev, G, world, local):
    """The same measurement on another named workload (single-launch path; the FP8 workload runs
    the prologue kernel in front of it), for the workloads object of the JSON line. heavy_q4 is
    the heavy-tailed batch with four new tokens per request, on the library's default kernel for
    them (the tcgen05 several-token kernel)."""
    from dataclasses import replace
    q_len = 4 if name == "heavy_q4" else 1
    base = "heavy" if name == "heavy_q4" else name
    spec = W.config_spec(base)
    if q_len > 1:
        spec = replace(spec, q_len=q_len, name=f"{spec.name}, {q_len} new tokens per request")
    case = W.make_case(spec)
    dc = device_case(case, dev)
    del case
    step = Step(B, spec, dc, G, spec.tile_len, fused=True, item_cost=args.item_cost, e4m3_kernel=args.e4m3_kernel)
    lens = step_lengths(dc, spec)
    est_ms = W.algorithmic_bytes(spec) / (6.0e9 if q_len == 1 else 4.0e9)
    K = int(min(5000, max(64, round(1500.0 / est_ms))))
    K -= K % spec.steps
    m = measure(step, spec, lens, K, 20, world, local)
    text = WORKLOAD_TEXT[base] + (f"; {q_len} new tokens per request, causal among themselves" if q_len > 1 else "")
    kernel = "decode_attention_tcm_kernel (tcgen05)" if q_len > 1 else "decode_attention_kernel<fused>"
    out = {"workload": text, "steps": K, "warmup": 20, "us_per_step": round(1000 * m["ms_step"], 2),
           "value": round(m["value"], 2), "unit": "GB/s",
           "roofline": dict(m["roofline"], kernel=kernel, traffic=load_traffic(traffic_key(base, q_len))),
           "clocks": m["clocks"], "gpu_launches": step.launches * K,
           "path": "single launch" + (" after the prologue kernel (PDL)" if spec.prologue else "")}
    if spec.steps > 1:
        out["note"] = f"{spec.steps} decode steps cycled (lengths +1 per step, re-planned on the device each step)"
    del step, dc
    torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, local):
    from load_balanced_split_step_b200 import binding as B
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    spec = workload_spec(args)
    case = W.make_case(spec)
    dc = device_case(case, dev, args.layout)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    tl = args.tile_len or spec.tile_len
    G = sms * args.ctas_per_sm
    lens = step_lengths(dc, spec)
    if args.shard:
        if spec.prologue or spec.q_len != 1 or args.layout != "HND":
            raise SystemExit("--shard runs one-token workloads without the prologue, HND cache")
        step = ShardStep(B, spec, dc, G, tl, rank, world, lens)
    else:
        step = Step(B, spec, dc, G, tl, fused=args.path == "fused", folded=args.path == "folded",
                    layout=args.layout, item_cost=args.item_cost, e4m3_kernel=args.e4m3_kernel,
                    multi_kernel=args.multi_kernel)
    K, W_ = args.steps, max(3, args.warmup)
    jobs = 1 if args.shard else world  # sharded: the ranks share one batch
    m = measure(step, spec, lens, K, W_, world, local, jobs=jobs, per_gpu_div=world if args.shard else 1)
    total_ms, kern_ms, bytes_step = m["total_ms"], m["kern_ms"], m["bytes_step"]
    value, ms_step = m["value"], m["ms_step"]
    clocks = m["clocks"]

    extra = {}
    if not args.no_extras and not args.shard:
        # graph replay of the same step (host launch overhead removed)
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            step(lens[0])
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        with torch.cuda.graph(g):
            step(lens[0])
        for _ in range(5):
            g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(K):
            g.replay()
        b.record()
        torch.cuda.synchronize()
        extra["graph_us_per_step"] = round(1000.0 * a.elapsed_time(b) / K, 2)
        del g
        extra["step_time_distribution"] = step_distribution(step, lens, max(50, 8 * len(lens)), world)
        if spec.q_len == 1:  # the static plan drives the three-launch path, which takes one new token
            extra["static_split_k"] = static_leg(B, spec, dc, tl, max(50, K // 10), sms, args.layout)
            extra["speedup_vs_static_split_k"] = round(extra["static_split_k"]["us_per_step"] / (1000 * ms_step),
                                                       3)
    e2e_steps = max(50, K // 4)
    if args.shard:
        e2e_ms, h2d, d2h = shard_e2e_leg(step, case, dc, e2e_steps, world)
    else:
        e2e_ms, h2d, d2h = e2e_leg(B, spec, case, dc, tl, G, e2e_steps, world, fused=args.path != "split",
                                   layout=args.layout, folded=args.path == "folded", multi_kernel=args.multi_kernel)
    e2e_ms = max_over_ranks(e2e_ms, world)
    e2e_val = jobs * bytes_step * e2e_steps / (e2e_ms / 1e3) / 1e9

    cpu = None
    if rank == 0 and world == 1 and not args.no_extras:
        cpu = cpu_baseline(spec, case)
    others = None
    if (world == 1 and not args.no_extras and not args.shard and args.workload == "extreme" and spec.q_len == 1
            and not args.requests and args.path == "fused" and args.layout == "HND"):
        del dc, case
        if not isinstance(step, ShardStep):
            step.dc = None
        torch.cuda.empty_cache()
        others = {name: other_workload(B, args, name, dev, G, world, local) for name in OTHER_WORKLOADS}

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": W_,
        "ms_per_step": round(ms_step, 5), "us_per_step": round(1000 * ms_step, 2), "higher_is_better": True,
        "scaling": "strong" if args.shard else "weak", "vs_baseline": None,
        "dtype": "bf16" if spec.kv_dtype == "bf16" else "e4m3/f16",
        "data": "synthetic (seeded N(0,1), bf16-rounded; random page permutation)",
        "config": {"workload": WORKLOAD_TEXT[args.workload] + qlen_text(args), "tile_len": tl, "num_ctas": G,
                   "plan": "dynamic (re-planned on the device every step)"
                   + ("; the single launch plans while the previous step's kernel finishes (seq_lens_ready: no "
                      "kernel writes the lengths)" if args.path in ("fused", "folded") and not args.shard else ""),
                   "path": ({"fused": "single launch: in-kernel plan, attention, ticket merge"
                                      + (" (after the prologue kernel, PDL)" if spec.prologue else ""),
                             "folded": "single launch: prologue, in-kernel plan, attention, ticket merge",
                             "split": "plan, attention and merge kernels chained by PDL"
                                      + (" after the prologue kernel" if spec.prologue else "")}[args.path]),
                   "kv_layout": args.layout,
                   "l2": f"inputs larger than L2 ({bytes_step / 1e9:.2f} GB per step), no flush",
                   "parallelism": (f"one batch request-sharded over {world} GPU(s): one all-gather of (out, lse), "
                                   "log-sum-exp merge of split requests") if args.shard
                   else f"{world} independent replica(s), no collective"},
        "roofline": dict(m["roofline"],
                         kernel="decode_attention_tcm_kernel (tcgen05)" if uses_tcgen05_multi(spec, args.multi_kernel)
                         else "decode_attention_kernel" + {"fused": "<fused>", "folded": "<fused, prologue>",
                                                           "split": ""}[args.path],
                         traffic=load_traffic(traffic_key(args.workload, args.q_len))
                         if not args.requests and (args.q_len == 1 or args.multi_kernel == "default") else None),
        "cpu_baseline": cpu,
        "e2e": {"value": round(e2e_val, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "us_per_step": round(1000 * e2e_ms / e2e_steps, 2)},
        "gpu_launches": step.launches * K,
        "clocks": clocks,
    }
    line.update(extra)
    if others:
        line["workloads"] = others
    return line


def run_reference(args, rank, world):
    """The reference arm: the fp64 CPU oracle as it stands, timed on the host cores over the same
    stratified sample as the cpu_baseline leg, one pass per step."""
    if rank != 0:
        return None
    spec = workload_spec(args)
    case = W.make_case(spec)
    K, W_ = max(1, min(args.steps, 5)), min(max(args.warmup, 0), 1)
    cb = CpuBaseline(spec, case)
    try:
        for _ in range(W_):
            cb.run()
        runs = [cb.run() for _ in range(K)]
    finally:
        cb.close()
    el = sum(e for _, e in runs)
    v = cb.bytes * K / el / 1e9
    bytes_step = W.algorithmic_bytes(spec)
    return {
        "impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": W_, "ms_per_step": round(1000 * bytes_step / (v * 1e9), 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT[args.workload] + qlen_text(args), "tile_len": spec.tile_len,
                   "plan": "none (exact)", "parallelism": f"{cb.workers} host processes"},
        "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": cb.workers, "kind": "oracle",
                         "sample": cb.describe(el / K) + f"; {K} timed passes", "cpu_model": cpu_model(),
                         "host_cores": os.cpu_count()},
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_trace(args, local):
    """Per-CTA load evidence from the HPC_TRACE build: for each of R single-launch steps, every
    CTA's entry, plan-ready, first-stage, last-item and producer-end stamps (%globaltimer, ns) with
    its item and stage counts. Summarised per step: the launch span (first entry to last end),
    each CTA's idle tail (span end minus its last item end, as a share of the span, averaged
    over CTAs), the spread of CTA end times, the plan and first-data latencies. Stamps perturb
    the kernel a little; the bench line, not this, gives the step time."""
    from load_balanced_split_step_b200 import binding as B
    from load_balanced_split_step_b200 import build as BLD
    B.use_library(BLD.build_trace())
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    spec = workload_spec(args)
    case = W.make_case(spec)
    dc = device_case(case, dev, args.layout)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    tl = args.tile_len or spec.tile_len
    G = sms * args.ctas_per_sm
    if args.path == "split":
        raise SystemExit("--trace summarises the single-launch step")
    step = Step(B, spec, dc, G, tl, fused=True, folded=args.path == "folded", layout=args.layout,
                item_cost=args.item_cost, e4m3_kernel=args.e4m3_kernel)
    trace = torch.zeros((G, B.TRACE_WORDS), dtype=torch.int64, device=dev)
    step.trace = trace
    lens = step_lengths(dc, spec)
    for i in range(max(3, args.warmup)):
        step(lens[i % len(lens)])
    R = max(1, min(args.steps, 64))
    per = []
    for i in range(R):
        trace.zero_()
        step(lens[i % len(lens)])
        torch.cuda.synchronize()
        t = trace.cpu().numpy().astype(np.int64)
        busy = t[:, 5] > 0
        start = t[:, 1].min()  # the first CTA past the wait on the previous launch
        end = max(t[:, 4].max(), t[busy, 3].max())
        span = end - start
        tail = (end - t[busy, 3]) / span  # idle after a CTA's last item, share of the span
        per.append({"span_us": span / 1e3, "idle_tail_mean": float(tail.mean()),
                    "idle_tail_p90": float(np.percentile(tail, 90)), "idle_tail_max": float(tail.max()),
                    "end_spread_us": float((end - t[busy, 3].min()) / 1e3),
                    "wait_and_plan_us_median": float(np.median(t[:, 1] - t[:, 0]) / 1e3),
                    "plan_ready_spread_us": float((t[:, 1].max() - start) / 1e3),
                    "first_data_us_median": float(np.median(t[busy, 2] - t[busy, 1]) / 1e3),
                    "items_max": int(t[:, 5].max()), "items_median": float(np.median(t[busy, 5])),
                    "stages_max": int(t[:, 6].max()), "stages_min_busy": int(t[busy, 6].min()),
                    "ctas_busy": int(busy.sum())})
    st = int(step.status.item())
    if st:
        raise RuntimeError(f"device status {st:#x}")
    keys = per[0].keys()
    summary = {k: round(float(np.median([p[k] for p in per])), 4) for k in keys}
    return {"trace": summary, "steps": R, "workload": WORKLOAD_TEXT[args.workload] + qlen_text(args), "num_ctas": G,
            "item_cost": args.item_cost if args.item_cost is not None else "default",
            "note": "medians over the traced steps; span = first CTA past the wait on the previous launch to the last "
                    "CTA's end; idle tail = (span end - a busy CTA's last item end) / span"}


def main(argv=None):
    args = parse_args(argv)
    rank, world, local = dist_init(args)
    try:
        if args.record_traffic:
            line = record_traffic(args)
        elif args.trace:
            line = run_trace(args, local)
        elif args.impl == "reference":
            line = run_reference(args, rank, world)
        else:
            line = run_ours(args, rank, world, local)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        dist_done(world)


if __name__ == "__main__":
    main()
