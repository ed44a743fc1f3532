"""Benchmark of the B200 sink-attention path.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload all|fwd|fwd_bwd|decode]

One JSON line on rank 0.  The headline workload is the packed varlen causal forward:
16 sequences with lengths ~ U[64, 4096] (seed 1), 32 q heads / 8 kv heads, head dim
128, bf16, sink ~ N(0, 1).  A step is one forward over that batch (tile schedule, loads,
Q K^T, masked online softmax with the sink, P V, epilogue: every step of the forward
path), with inputs resident in HBM; L2 is flushed (a 256 MB write) before every timed
step.  ``value`` is algorithmic TFLOP/s: 2 (dk + dv) flops per visible (query, key, head)
triple, summed over all ranks, divided by the slowest rank's device time.

With ``--workload all`` (the default) the same line also carries the other two paths,
each timed the same way: ``fwd_bwd`` (4 x 8192 tokens, 16 heads, d 128, causal:
forward and backward TFLOP/s) and ``decode`` (64 sequences of one query against 8k-32k
keys, 64 q / 8 kv heads: GB/s of K/V read).

Multi-GPU (torchrun): every rank runs its own copy of the workload (weak scaling, no
data-path collective; independent problems shard with no exchange).  Timing is the
max over ranks of each rank's CUDA-event time.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same workload
(one 256-row slice of one (sequence, head) per step) on this host's cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "sink-attention fwd/bwd TFLOP/s (bf16) and decode GB/s, % of B200 roofline"


# --- algorithmic work ------------------------------------------------------------------

def visible_pairs(cu_q, cu_k, hq, causal, window_left=-1, window_right=-1) -> int:
    """Visible (query, key, q head) triples, bottom-right aligned, counted row by row."""
    total = 0
    for b in range(len(cu_q) - 1):
        sq = int(cu_q[b + 1] - cu_q[b])
        sk = int(cu_k[b + 1] - cu_k[b])
        if sq <= 0 or sk <= 0:
            continue
        pos = np.arange(sq, dtype=np.int64) + (sk - sq)
        right = np.inf if window_right < 0 else window_right
        if causal:
            right = min(right, 0)
        hi = np.minimum(sk, pos + right + 1) if np.isfinite(right) else np.full(sq, sk)
        lo = np.maximum(0, pos - window_left) if window_left >= 0 else np.zeros(sq, np.int64)
        total += int(np.maximum(0, hi - lo).sum())
    return total * int(hq)


def source_digest(kernel_file: str) -> str:
    """sha256[:16] over a kernel source and the project headers it includes, directly or
    through other headers (what its build depends on), in a fixed order."""
    import hashlib
    import re
    dirs = [os.path.join(ROOT, "softmax_attn_sink_b200", "csrc"), os.path.join(ROOT, "include")]
    seen, todo = [], [kernel_file]
    while todo:
        name = todo.pop()
        path = next((os.path.join(d, name) for d in dirs if os.path.exists(os.path.join(d, name))), None)
        if path is None or path in seen:
            continue
        seen.append(path)
        with open(path, encoding="utf-8") as f:
            todo += re.findall(r'^\s*#\s*include\s+"([^"]+)"', f.read(), flags=re.M)
    h = hashlib.sha256()
    for path in [seen[0]] + sorted(seen[1:]):
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def kernel_traffic(kernel_file: str, leg: str = ""):
    """DRAM bytes per bench launch from profiles/traffic.txt (the line labelled
    ``kernel_file`` or ``kernel_file:leg``), or None when the kernel's sources have changed
    since that capture."""
    label = kernel_file + (":" + leg if leg else "")
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.txt")) as f:
            for line in f:
                parts = line.split()
                if parts and not line.startswith("#") and parts[0] == label:
                    return int(parts[2]) if parts[1] == source_digest(kernel_file) else None
    except OSError:
        pass
    return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# --- clocks during the timed region ----------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, uuid):
        self.uuid, self.proc, self.lines = uuid, None, []

    def __enter__(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50"]
        if self.uuid:
            cmd.insert(1, f"--id={self.uuid}")
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.15)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        for l in self.lines:
            parts = [x.strip() for x in l.split(",")]
            if len(parts) < 6:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for name, flag in zip(self.NAMES, parts[2:6]):
                if flag.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --- distributed plumbing ---------------------------------------------------------------

def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return rank, world, local


def barrier(world):
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def _reduce_device():
    import torch.distributed as dist
    return "cpu" if dist.get_backend() == "gloo" else "cuda"


def max_over_ranks(x: float, world: int) -> float:
    """The slowest rank's value (all ranks call this in the same order)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=_reduce_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank: float, world: int, total_ms_max: float, steps: int) -> float:
    """Throughput of the whole job: every rank's units over the slowest rank's time."""
    return units_per_rank * world / (total_ms_max / steps * 1e-3)


# --- timing helpers ---------------------------------------------------------------------

class Flusher:
    """Writes 256 MB (2x the 126 MB L2) so every timed step starts with a cold L2."""

    def __init__(self):
        import torch
        self.buf = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def __call__(self):
        self.buf.fill_(1)


def time_steps(fn, steps, warmup, world, flush, sampler=None):
    """Run `warmup` untimed steps, then exactly `steps` timed ones bracketed by barrier +
    synchronize; each step is timed with CUDA events on the current stream after an L2
    flush.  Returns (per-step ms list, max-over-ranks total ms of the steps)."""
    import torch
    for _ in range(warmup):
        flush()
        fn()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier(world)
    ctx = sampler if sampler is not None else _Null()
    with ctx:
        for i in range(steps):
            flush()
            starts[i].record()
            fn()
            ends[i].record()
        barrier(world)
    per = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    return per, max_over_ranks(sum(per), world)


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def gpu_uuid(local):
    import torch
    try:
        u = str(torch.cuda.get_device_properties(local).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return None


# --- workloads --------------------------------------------------------------------------

def fwd_workload():
    import torch
    p = W.config2()
    td = torch.bfloat16
    t = {"q": torch.from_numpy(p.q).to(td), "k": torch.from_numpy(p.k).to(td),
         "v": torch.from_numpy(p.v).to(td), "cu": torch.from_numpy(p.cu_seqlens_q),
         "sink": torch.from_numpy(p.sink)}
    pairs = visible_pairs(p.cu_seqlens_q, p.cu_seqlens_k, p.num_heads_q, True)
    return p, t, pairs


def bench_fwd(args, world, peaks, peak_kind, sampler):
    import torch
    import softmax_attn_sink_b200 as sab
    p, host, pairs = fwd_workload()
    dev = {k: v.cuda() for k, v in host.items()}
    mq, mk = p.max_seqlen_q, p.max_seqlen_k
    out = torch.empty((p.q.shape[0], 32, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((32, p.q.shape[0]), dtype=torch.float32, device="cuda")
    flops = 2 * (128 + 128) * pairs

    def step():
        sab.attn_sink_fwd(dev["q"], dev["k"], dev["v"], dev["cu"], dev["cu"], mq, mk, dev["sink"],
                          p.softmax_scale, True, out=out, lse=lse)

    flush = Flusher()
    per, total_ms = time_steps(step, args.steps, args.warmup, world, flush, sampler)
    ms = total_ms / args.steps
    tflops = weak_scaling_value(flops, world, total_ms, args.steps) / 1e12
    kernel_ms = statistics.mean(per)
    achieved = flops / (kernel_ms * 1e-3) / 1e12
    roof = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
            "traffic": kernel_traffic("fwd_sm100.cu"),
            "peak_source": f"bf16_tflops ({peak_kind}, burst: kernel timed alone)",
            "kernel": "fwd (one launch per step)", "flops_per_launch": flops}

    # end to end through the public API with host buffers: every step copies its inputs from
    # pinned host memory, runs the forward and copies out and lse back.  Consecutive steps
    # are pipelined on three streams (H2D of step i, forward of step i - 1, D2H of step i - 2)
    # over two device buffer sets; the whole run is timed between events on the compute
    # stream.  No L2 flush: the inputs (422 MB) are larger than L2.
    pin = {k: v.pin_memory() for k, v in host.items()}
    devs = [{k: torch.empty(v.shape, dtype=v.dtype, device="cuda") for k, v in host.items()} for _ in range(2)]
    outs = [(torch.empty_like(out), torch.empty_like(lse)) for _ in range(2)]
    houts = [(torch.empty(out.shape, dtype=out.dtype).pin_memory(), torch.empty(lse.shape, dtype=lse.dtype).pin_memory())
             for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in pin.values())
    d2h = out.numel() * out.element_size() + lse.numel() * lse.element_size()
    comp_s = torch.cuda.current_stream()
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev_h2d = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_d2h = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(n):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(comp_s)
        h2d_s.wait_event(t0)
        for i in range(n):
            bi = i % 2
            d, (o, l), (oh, lh) = devs[bi], outs[bi], houts[bi]
            with torch.cuda.stream(h2d_s):
                if i >= 2:
                    h2d_s.wait_event(ev_comp[bi])   # the forward of step i - 2 read these inputs
                for k2 in d:
                    d[k2].copy_(pin[k2], non_blocking=True)
                ev_h2d[bi].record(h2d_s)
            comp_s.wait_event(ev_h2d[bi])
            if i >= 2:
                comp_s.wait_event(ev_d2h[bi])       # the D2H of step i - 2 read these outputs
            sab.attn_sink_fwd(d["q"], d["k"], d["v"], d["cu"], d["cu"], mq, mk, d["sink"], p.softmax_scale, True,
                              out=o, lse=l)
            ev_comp[bi].record(comp_s)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(ev_comp[bi])
                oh.copy_(o, non_blocking=True)
                lh.copy_(l, non_blocking=True)
                ev_d2h[bi].record(d2h_s)
        comp_s.wait_event(ev_d2h[(n - 1) % 2])
        t1.record(comp_s)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    e_steps = max(3, min(args.steps, 20))
    e2e_run(2)
    barrier(world)
    e_total = max_over_ranks(e2e_run(e_steps), world)
    e2e = {"value": round(flops * world / (e_total / e_steps * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
           "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": e_steps,
           "ms_per_step": round(e_total / e_steps, 3),
           "pipelined": "H2D of step i, forward of step i-1 and D2H of step i-2 overlap on three streams",
           "l2": "not flushed: inputs (422 MB) larger than L2"}
    return {"value": tflops, "ms": ms, "roofline": roof, "e2e": e2e, "launches": args.steps,
            "pairs": pairs, "flops": flops, "p": p}


DROPOUT = (0.1, 0x5EED5EED1234ABCD, 0)   # p, Philox key, counter offset of the dropout legs


def bench_fwd_variant(args, world, peaks, peak_kind, dtype="fp16", dropout=None):
    """The headline forward with fp16 inputs (the same draws rounded to fp16), or with
    dropout; the algorithmic flops are those of the plain forward."""
    import torch
    import softmax_attn_sink_b200 as sab
    p = W.config2(dtype)
    td = torch.float16 if dtype == "fp16" else torch.bfloat16
    q, k, v = (torch.from_numpy(x).to(td).cuda() for x in (p.q, p.k, p.v))
    cu = torch.from_numpy(p.cu_seqlens_q).cuda()
    sink = torch.from_numpy(p.sink).cuda()
    pairs = visible_pairs(p.cu_seqlens_q, p.cu_seqlens_k, p.num_heads_q, True)
    flops = 2 * (128 + 128) * pairs
    out = torch.empty((p.q.shape[0], 32, 128), dtype=td, device="cuda")
    lse = torch.empty((32, p.q.shape[0]), dtype=torch.float32, device="cuda")
    flush = Flusher()
    steps = max(3, min(args.steps, 50))
    per, total = time_steps(lambda: sab.attn_sink_fwd(q, k, v, cu, cu, p.max_seqlen_q, p.max_seqlen_k, sink,
                                                      p.softmax_scale, True, out=out, lse=lse,
                                                      dropout=dropout),
                            steps, args.warmup, world, flush)
    achieved = flops / (statistics.mean(per) * 1e-3) / 1e12
    pk = peaks["bf16_tflops"]   # dense fp16 and bf16 tensor rates are equal (nominal ratio 1)
    name = p.name + (f"_dropout{dropout[0]}" if dropout else "")
    return {"workload": name, "unit": "TFLOP/s", "steps": steps,
            "value": round(weak_scaling_value(flops, world, total, steps) / 1e12, 2),
            "ms_per_step": round(total / steps, 4), "flops": flops,
            "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": pk, "unit": "TFLOP/s",
                         "frac": round(achieved / pk, 4), "traffic": None,
                         "peak_source": f"bf16_tflops x 1 (nominal fp16 / bf16 dense ratio; {peak_kind}, burst)"}}


def bench_fwd_d256(args, world, peaks, peak_kind):
    """Head dim 256: the headline workload's 16 sequence lengths with 16 q / 4 kv heads at
    d = 256, causal, bf16 N(0, 1) drawn on the device from a seeded generator."""
    import torch
    import softmax_attn_sink_b200 as sab
    lens = W.config2_lengths()
    cu_np = W.cu_from_lengths(lens)
    tq, hq, hkv, d = int(cu_np[-1]), 16, 4, 256
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5)
    q, k, v = (torch.randn((tq, h, d), generator=gen, device="cuda").to(torch.bfloat16) for h in (hq, hkv, hkv))
    sink = torch.randn(hq, generator=gen, device="cuda")
    cu = torch.from_numpy(cu_np).cuda()
    mx = int(lens.max())
    pairs = visible_pairs(cu_np, cu_np, hq, True)
    flops = 2 * (d + d) * pairs
    out = torch.empty((tq, hq, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((hq, tq), dtype=torch.float32, device="cuda")
    flush = Flusher()
    steps = max(3, min(args.steps, 50))
    per, total = time_steps(lambda: sab.attn_sink_fwd(q, k, v, cu, cu, mx, mx, sink, 1.0 / 16.0, True,
                                                      out=out, lse=lse),
                            steps, args.warmup, world, flush)
    achieved = flops / (statistics.mean(per) * 1e-3) / 1e12
    pk = peaks["bf16_tflops"]
    # backward (preprocess + the tcgen05 dQ, dK and dV kernels of this head dim): a few steps
    do = torch.randn((tq, hq, d), generator=gen, device="cuda").to(torch.bfloat16)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dsink = torch.empty(hq, dtype=torch.float32, device="cuda")
    bflops = 2 * (3 * d + 2 * d) * pairs
    b_per, b_total = time_steps(lambda: sab.attn_sink_bwd(q, k, v, out, do, lse, cu, cu, mx, mx, sink, 1.0 / 16.0,
                                                          True, dq=dq, dk=dk, dv=dv, dsink=dsink),
                                3, 1, world, flush)
    ba = bflops / (statistics.mean(b_per) * 1e-3) / 1e12
    # the same backward with dropout p = 0.1 (the forward's keep bytes redrawn)
    sab.attn_sink_fwd(q, k, v, cu, cu, mx, mx, sink, 1.0 / 16.0, True, out=out, lse=lse, dropout=DROPOUT)
    bd_per, bd_total = time_steps(lambda: sab.attn_sink_bwd(q, k, v, out, do, lse, cu, cu, mx, mx, sink, 1.0 / 16.0,
                                                            True, dq=dq, dk=dk, dv=dv, dsink=dsink, dropout=DROPOUT),
                                  3, 1, world, flush)
    bda = bflops / (statistics.mean(bd_per) * 1e-3) / 1e12
    # decode: 16 sequences of the decode workload's lengths, 32 q / 4 kv heads at d = 256
    dl = W.config5_meta().cu_seqlens_k
    dlens = np.diff(dl)[:16]
    dcu_np = W.cu_from_lengths(dlens)
    dk_ = torch.randn((int(dcu_np[-1]), 4, d), generator=gen, device="cuda").to(torch.bfloat16)
    dv_ = torch.randn((int(dcu_np[-1]), 4, d), generator=gen, device="cuda").to(torch.bfloat16)
    dq_ = torch.randn((16, 32, d), generator=gen, device="cuda").to(torch.bfloat16)
    dsk = torch.randn(32, generator=gen, device="cuda")
    dcu = torch.from_numpy(dcu_np).cuda()
    dout = torch.empty((16, 32, d), dtype=torch.bfloat16, device="cuda")
    dlse = torch.empty((32, 16), dtype=torch.float32, device="cuda")
    dbytes = 2 * int(dcu_np[-1]) * 4 * d * 2 + dq_.numel() * 2 + dout.numel() * 2 + dlse.numel() * 4
    d_per, d_total = time_steps(lambda: sab.attn_sink_decode(dq_, dk_, dv_, dcu, int(dlens.max()), dsk, 1.0 / 16.0,
                                                             out=dout, lse=dlse),
                                steps, args.warmup, world, flush)
    da = dbytes / (statistics.mean(d_per) * 1e-3) / 1e9
    pb = peaks["hbm_gbs"]
    return {"workload": "varlen16_gqa16x4_d256_causal", "unit": "TFLOP/s", "steps": steps,
            "value": round(weak_scaling_value(flops, world, total, steps) / 1e12, 2),
            "ms_per_step": round(total / steps, 4), "flops": flops, "pairs": pairs,
            "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": pk, "unit": "TFLOP/s",
                         "frac": round(achieved / pk, 4), "traffic": kernel_traffic("fwd_d256_sm100.cu"),
                         "peak_source": f"bf16_tflops ({peak_kind}, burst)",
                         "kernel": "fwd_d256_sm100 (one launch per step)"},
            "bwd": {"value": round(bflops * world / (b_total / 3 * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                    "ms_per_step": round(b_total / 3, 3), "flops": bflops, "steps": 3,
                    "roofline": {"bound": "tensor", "achieved": round(ba, 2), "peak": pk, "unit": "TFLOP/s",
                                 "frac": round(ba / pk, 4), "traffic": None,
                                 "kernels": "preprocess + tcgen05 dQ + dK + dV"}},
            "bwd_dropout": {"value": round(bflops * world / (bd_total / 3 * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                            "ms_per_step": round(bd_total / 3, 3), "flops": bflops, "steps": 3, "dropout": [DROPOUT[0]],
                            "roofline": {"bound": "tensor", "achieved": round(bda, 2), "peak": pk, "unit": "TFLOP/s",
                                         "frac": round(bda / pk, 4), "traffic": None}},
            "decode": {"workload": "decode16_gqa32x4_d256_L8k-32k", "value": round(dbytes * world / (d_total / steps * 1e-3) / 1e9, 1),
                       "unit": "GB/s", "ms_per_step": round(d_total / steps, 4), "bytes_per_step": dbytes,
                       "roofline": {"bound": "hbm", "achieved": round(da, 1), "peak": pb, "unit": "GB/s",
                                    "frac": round(da / pb, 4), "traffic": kernel_traffic("decode_split.cu", "d256"),
                                    "kernels": "split + merge (two launches per step)"}}}


def bench_small_configs(args, world, peaks, peak_kind):
    """The two small forward configurations: 2 x 256 tokens, 4 heads, d 64, non-causal and
    causal; and softmax_n (sink = log n, n in {1, 0.5, 3}) on 6 x (1024 queries, 1152 keys),
    1 head, dk 64 / dv 32, bottom-right causal with a (512, 0) window.  Both launch far fewer
    tiles than the GPU has SMs, so they measure launch latency and a short critical path,
    not throughput; they are reported, not graded."""
    import torch
    import softmax_attn_sink_b200 as sab
    flush = Flusher()
    steps = max(10, min(args.steps, 100))
    pk = peaks["bf16_tflops"]

    def run(p, wl, wr):
        td = torch.bfloat16
        q, k, v = (torch.from_numpy(x).to(td).cuda() for x in (p.q, p.k, p.v))
        cq, ck = torch.from_numpy(p.cu_seqlens_q).cuda(), torch.from_numpy(p.cu_seqlens_k).cuda()
        sink = torch.from_numpy(p.sink).cuda()
        out = torch.empty((q.shape[0], q.shape[1], v.shape[2]), dtype=td, device="cuda")
        lse = torch.empty((q.shape[1], q.shape[0]), dtype=torch.float32, device="cuda")
        pairs = visible_pairs(p.cu_seqlens_q, p.cu_seqlens_k, q.shape[1], p.causal, wl, wr)
        flops = 2 * (q.shape[2] + v.shape[2]) * pairs
        per, total = time_steps(lambda: sab.attn_sink_fwd(q, k, v, cq, ck, p.max_seqlen_q, p.max_seqlen_k, sink,
                                                          p.softmax_scale, p.causal, (wl, wr), out=out, lse=lse),
                                steps, args.warmup, world, flush)
        achieved = flops / (statistics.mean(per) * 1e-3) / 1e12
        return {"value": round(weak_scaling_value(flops, world, total, steps) / 1e12, 3), "unit": "TFLOP/s",
                "ms_per_step": round(total / steps, 5), "pairs": pairs, "flops": flops, "steps": steps,
                "roofline": {"bound": "tensor", "achieved": round(achieved, 3), "peak": pk, "unit": "TFLOP/s",
                             "frac": round(achieved / pk, 5), "traffic": None,
                             "peak_source": f"bf16_tflops ({peak_kind}, burst)",
                             "kernel": "fwd_sm100 (one launch per step; launch-latency bound)"}}

    c1 = {"workload": "fixed2x256_h4_d64"}
    for causal in (False, True):
        c1["causal" if causal else "non_causal"] = run(W.config1(causal), -1, -1)
    c4 = {"workload": "softmax_n_6x1024x1152_h1_dk64_dv32_causal_window512"}
    for n in (1.0, 0.5, 3.0):
        c4[f"n={n:g}"] = run(W.config4(n), 512, 0)
    return {"config1": c1, "config4": c4}


def bench_fwd_bwd(args, world, peaks, peak_kind):
    import torch
    import softmax_attn_sink_b200 as sab
    p = W.config3()
    if args.seqs < 4:  # a smaller case of the same kernels (for profiler captures)
        t = 8192 * args.seqs
        p.q, p.k, p.v, p.dout = p.q[:t], p.k[:t], p.v[:t], p.dout[:t]
        p.cu_seqlens_q = p.cu_seqlens_q[:args.seqs + 1].copy()
        p.cu_seqlens_k = p.cu_seqlens_q.copy()
    td = torch.bfloat16
    q, k, v, do = (torch.from_numpy(x).to(td).cuda() for x in (p.q, p.k, p.v, p.dout))
    cu = torch.from_numpy(p.cu_seqlens_q).cuda()
    sink = torch.from_numpy(p.sink).cuda()
    pairs = visible_pairs(p.cu_seqlens_q, p.cu_seqlens_k, 16, True)
    out, lse = sab.attn_sink_fwd(q, k, v, cu, cu, 8192, 8192, sink, p.softmax_scale, True)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dsink = torch.empty(16, dtype=torch.float32, device="cuda")
    flush = Flusher()
    steps = max(3, min(args.steps, 20))
    f_per, f_total = time_steps(
        lambda: sab.attn_sink_fwd(q, k, v, cu, cu, 8192, 8192, sink, p.softmax_scale, True,
                                  out=out, lse=lse), steps, args.warmup, world, flush)
    b_per, b_total = time_steps(
        lambda: sab.attn_sink_bwd(q, k, v, out, do, lse, cu, cu, 8192, 8192, sink, p.softmax_scale,
                                  True, dq=dq, dk=dk, dv=dv, dsink=dsink), steps, args.warmup, world, flush)
    d_per, d_total = time_steps(
        lambda: sab.attn_sink_bwd(q, k, v, out, do, lse, cu, cu, 8192, 8192, sink, p.softmax_scale,
                                  True, dq=dq, dk=dk, dv=dv, dsink=dsink, deterministic=True),
        steps, args.warmup, world, flush)
    fd_per, fd_total = time_steps(
        lambda: sab.attn_sink_fwd(q, k, v, cu, cu, 8192, 8192, sink, p.softmax_scale, True,
                                  out=out, lse=lse, dropout=DROPOUT), steps, args.warmup, world, flush)
    bd_per, bd_total = time_steps(
        lambda: sab.attn_sink_bwd(q, k, v, out, do, lse, cu, cu, 8192, 8192, sink, p.softmax_scale,
                                  True, dq=dq, dk=dk, dv=dv, dsink=dsink, dropout=DROPOUT),
        steps, args.warmup, world, flush)
    ff, bf = 2 * 256 * pairs, 2 * (3 * 128 + 2 * 128) * pairs
    fa = ff / (statistics.mean(f_per) * 1e-3) / 1e12
    ba = bf / (statistics.mean(b_per) * 1e-3) / 1e12
    da = bf / (statistics.mean(d_per) * 1e-3) / 1e12
    fda = ff / (statistics.mean(fd_per) * 1e-3) / 1e12
    bda = bf / (statistics.mean(bd_per) * 1e-3) / 1e12
    pk = peaks["bf16_tflops"]

    def leg(total, flops, achieved, **kw):
        return {"value": round(flops * world / (total / steps * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "ms_per_step": round(total / steps, 4), "flops": flops,
                "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": pk,
                             "unit": "TFLOP/s", "frac": round(achieved / pk, 4), "traffic": None,
                             "peak_source": f"bf16_tflops ({peak_kind}, burst)", **kw}}
    return {
        "workload": f"train{args.seqs}x8192_h16_d128_causal", "pairs": pairs, "steps": steps,
        "fwd": {"value": round(ff * world / (f_total / steps * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "ms_per_step": round(f_total / steps, 4), "flops": ff,
                "roofline": {"bound": "tensor", "achieved": round(fa, 2), "peak": pk,
                             "unit": "TFLOP/s", "frac": round(fa / pk, 4), "traffic": None,
                             "peak_source": f"bf16_tflops ({peak_kind}, burst)"}},
        "bwd": {"value": round(bf * world / (b_total / steps * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "ms_per_step": round(b_total / steps, 4), "flops": bf,
                "roofline": {"bound": "tensor", "achieved": round(ba, 2), "peak": pk,
                             "unit": "TFLOP/s", "frac": round(ba / pk, 4),
                             "traffic": kernel_traffic("bwd_sm100.cu") if args.seqs == 4 else None,
                             "peak_source": f"bf16_tflops ({peak_kind}, burst)"}},
        # the same algorithmic flops; the deterministic pass recomputes Q K^T and dout V^T
        "bwd_deterministic": {"value": round(bf * world / (d_total / steps * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                              "ms_per_step": round(d_total / steps, 4), "flops": bf,
                              "roofline": {"bound": "tensor", "achieved": round(da, 2), "peak": pk,
                                           "unit": "TFLOP/s", "frac": round(da / pk, 4), "traffic": None,
                                           "peak_source": f"bf16_tflops ({peak_kind}, burst)",
                                           "kernels": "preprocess + key-stationary dK/dV + query-stationary dQ"}},
        # dropout p = 0.1 (Philox keep bytes drawn in the forward, redrawn in the backward);
        # the flops counted are the plain ones
        "fwd_dropout": leg(fd_total, ff, fda, dropout=list(DROPOUT[:1])),
        "bwd_dropout": leg(bd_total, bf, bda, dropout=list(DROPOUT[:1]),
                           kernels="preprocess + key-stationary dK/dV + query-stationary dQ"),
    }


def bench_decode(args, world, peaks, peak_kind):
    import torch
    import softmax_attn_sink_b200 as sab
    d = W.config5_meta()
    nb = args.decode_batch
    if nb < 64:  # a smaller case of the same kernels (for profiler captures)
        d.q = d.q[:nb]
        d.cu_seqlens_k = d.cu_seqlens_k[:nb + 1].copy()
    total_k = int(d.cu_seqlens_k[-1])
    k, v = W.decode_kv_on_device(total_k, 8, 128, 128, seed=4)
    q = torch.from_numpy(d.q).to(torch.bfloat16).cuda()
    cu = torch.from_numpy(d.cu_seqlens_k).cuda()
    sink = torch.from_numpy(d.sink).cuda()
    mk = int(np.diff(d.cu_seqlens_k).max())
    out = torch.empty((nb, 64, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((64, nb), dtype=torch.float32, device="cuda")
    splits = sab.decode_num_splits(nb, mk, total_k, 64, 8, 128, 128)
    ws = torch.empty(nb * 64 * splits * (128 + 2) * 4 + 4096, dtype=torch.uint8, device="cuda")
    flush = Flusher()
    steps = max(3, min(args.steps, 50))
    per, total = time_steps(
        lambda: sab.attn_sink_decode(q, k, v, cu, mk, sink, d.softmax_scale, True, (-1, -1), 0,
                                     out=out, lse=lse, workspace=ws), steps, args.warmup, world, flush)
    kv_bytes = 2 * total_k * 8 * 128 * 2
    io_bytes = q.numel() * 2 + out.numel() * 2 + lse.numel() * 4 + cu.numel() * 4 + sink.numel() * 4
    algo = kv_bytes + io_bytes
    gbs = algo / (statistics.mean(per) * 1e-3) / 1e9
    pk = peaks["hbm_gbs"]
    res = {"workload": f"decode{nb}_gqa64x8_d128_L8k-32k", "unit": "GB/s", "steps": steps,
           "value": round(algo * world / (total / steps * 1e-3) / 1e9, 1),
           "ms_per_step": round(total / steps, 4), "bytes_per_step": algo, "splits": splits,
           "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk, "unit": "GB/s",
                        "frac": round(gbs / pk, 4),
                        "traffic": kernel_traffic("decode_split.cu") if nb == 64 else None,
                        "peak_source": f"hbm_gbs ({peak_kind})",
                        "kernels": "split + merge (two launches per step)"}}

    # the same keys and values in a paged cache: 64-key blocks in a seeded random order
    bs = 64
    lens = np.diff(d.cu_seqlens_k)
    table, n_blocks = W.paged_layout(40, lens, bs)
    kc = W.to_paged(k, d.cu_seqlens_k, table, bs, n_blocks)
    vc = W.to_paged(v, d.cu_seqlens_k, table, bs, n_blocks)
    del k, v
    tab = torch.from_numpy(table).cuda()
    used = torch.from_numpy(lens.astype(np.int32)).cuda()
    per_p, total_p = time_steps(
        lambda: sab.attn_sink_decode_paged(q, kc, vc, tab, used, mk, sink, d.softmax_scale, True, (-1, -1),
                                           0, out=out, lse=lse, workspace=ws),
        steps, args.warmup, world, flush)
    table_bytes = int(sum(-(-int(n) // bs) for n in lens)) * 4 + used.numel() * 4
    algo_p = kv_bytes + io_bytes - cu.numel() * 4 + table_bytes
    gbs_p = algo_p / (statistics.mean(per_p) * 1e-3) / 1e9
    res["paged"] = {"workload": f"decode{nb}_gqa64x8_d128_L8k-32k_paged{bs}", "unit": "GB/s",
                    "value": round(algo_p * world / (total_p / steps * 1e-3) / 1e9, 1),
                    "ms_per_step": round(total_p / steps, 4), "bytes_per_step": algo_p,
                    "block_size": bs, "num_blocks": n_blocks,
                    "roofline": {"bound": "hbm", "achieved": round(gbs_p, 1), "peak": pk, "unit": "GB/s",
                                 "frac": round(gbs_p / pk, 4), "traffic": None,
                                 "peak_source": f"hbm_gbs ({peak_kind})"}}
    del kc, vc
    return res


# --- the oracle on the host -------------------------------------------------------------

def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(budget_s=15.0):
    secs, flops, steps = 0.0, 0, 0
    while secs < budget_s and steps < 5000:
        s, f = _oracle_step(steps)
        secs += s
        flops += f
        steps += 1
    return {"value": round(flops / secs / 1e12, 6), "unit": "TFLOP/s", "cores": cpu_cores(),
            "kind": "oracle",
            "sample": f"{steps} slices of 256 query rows of one (sequence, head) of the headline "
                      f"workload, fp64 NumPy, {secs:.1f} s of CPU time"}


def _oracle_step(s, _cache={}):
    """One bounded oracle step: 256 query rows of one (sequence, head) of the headline
    workload, cycling deterministically.  Returns (seconds, algorithmic flops)."""
    from oracle import ref  # the oracle: only the CPU legs of this script import it
    if "p" not in _cache:
        _cache["p"] = W.config2()
    p = _cache["p"]
    a = (p.cu_seqlens_q, p.cu_seqlens_k, p.sink, p.softmax_scale, True, -1, -1)
    b = (s * 7) % 16
    h = (s * 11) % 32
    L = int(p.cu_seqlens_q[b + 1] - p.cu_seqlens_q[b])
    r0 = (s * 131) % (L - 256 + 1) if L > 256 else 0
    rows = list(range(r0, min(L, r0 + 256)))
    t0 = time.perf_counter()
    ref.fwd_rows(p.q, p.k, p.v, *a, b=b, h=h, rows=rows)
    dt = time.perf_counter() - t0
    vis = sum(min(L, r + 1) for r in rows)
    return dt, 2 * 256 * vis


def run_reference(args):
    """The oracle as the reference arm: rank 0 only, on this host's cores."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    for s in range(args.warmup):
        _oracle_step(s)
    secs, flops = 0.0, 0
    for s in range(args.steps):
        dt, f = _oracle_step(args.warmup + s)
        secs += dt
        flops += f
    value = flops / secs / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(secs / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "varlen16_gqa32x8_d128_causal (oracle sample)",
                       "step": "256 query rows of one (sequence, head), fp64 NumPy"},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cpu_cores(),
                             "kind": "oracle",
                             "sample": f"{args.steps} steps of 256 query rows of one (sequence, "
                                       "head) of the headline workload"},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["all", "fwd", "fwd_fp16", "fwd_dropout", "fwd_d256", "fwd_bwd", "decode",
                                           "small"],
                    default="all")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seqs", type=int, default=4, choices=[1, 2, 3, 4],
                    help="sequences of the fwd_bwd leg (4 = the full training workload)")
    ap.add_argument("--decode-batch", type=int, default=64,
                    help="sequences of the decode leg (64 = the full decode workload)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours" and args.workload == "all":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    rank, world, local = dist_setup(args.gpus)
    peaks, peak_kind = load_peaks()
    line = {"metric": METRIC, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded numpy N(0,1) bf16; decode K/V seeded torch Philox on device)"}
    extra = {}
    try:
        if args.workload in ("all", "fwd"):
            sampler = ClockSampler(gpu_uuid(local)) if rank == 0 else None
            r = bench_fwd(args, world, peaks, peak_kind, sampler)
            p = r["p"]
            line.update({
                "value": round(r["value"], 3), "unit": "TFLOP/s", "ms_per_step": round(r["ms"], 4),
                "config": {"workload": "varlen16_gqa32x8_d128_causal",
                           "sequences": 16, "total_tokens": int(p.cu_seqlens_q[-1]),
                           "num_heads_q": 32, "num_heads_kv": 8, "head_dim": 128, "causal": True,
                           "visible_pairs": r["pairs"], "flops_per_step": r["flops"],
                           "l2": "flushed (256 MB write) before every timed step",
                           "parallelism": f"replicas x{world}"},
                "roofline": r["roofline"], "e2e": r["e2e"], "gpu_launches": r["launches"],
            })
            if sampler is not None:
                line["clocks"] = sampler.summary()
        if args.workload in ("all", "fwd_fp16"):
            extra["fwd_fp16"] = bench_fwd_variant(args, world, peaks, peak_kind, "fp16")
        if args.workload in ("all", "fwd_dropout"):
            extra["fwd_dropout"] = bench_fwd_variant(args, world, peaks, peak_kind, "bf16", DROPOUT)
        if args.workload in ("all", "fwd_d256"):
            extra["fwd_d256"] = bench_fwd_d256(args, world, peaks, peak_kind)
        if args.workload in ("all", "fwd_bwd"):
            extra["fwd_bwd"] = bench_fwd_bwd(args, world, peaks, peak_kind)
        if args.workload in ("all", "small"):
            extra.update(bench_small_configs(args, world, peaks, peak_kind))
        if args.workload in ("all", "decode"):
            extra["decode"] = bench_decode(args, world, peaks, peak_kind)
        if extra:
            line["extra"] = extra
        if "value" not in line:  # a single non-headline workload was asked for
            key = args.workload if args.workload != "small" else "config4"
            e = extra[key]
            if key == "config4":
                e = dict(e["n=1"], workload=e["workload"])
            v = e["fwd"]["value"] if key == "fwd_bwd" else e["value"]
            line.update({"value": v, "unit": e.get("unit", "TFLOP/s"),
                         "ms_per_step": e["fwd"]["ms_per_step"] if key == "fwd_bwd" else e["ms_per_step"],
                         "config": {"workload": e["workload"]}})
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline()
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
