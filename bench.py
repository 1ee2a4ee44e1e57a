#!/usr/bin/env python3
"""Decode-step benchmark: KV tokens scanned per second over a prunable INT2
KV cache on B200, with achieved HBM bandwidth against the measured peak.

One step = one decode step of the whole hot path: append the new token per
(sequence, KV head) (transform + quantize + pack), transform the query and
select channels, channel-skipping split-context attention and the merge.
Inputs are device resident and L2 is cold for every step: when a step reads
enough, several copies of the cache (each with its own transforms) are used
in turn and the steps run back to back; otherwise L2 is flushed between steps
(a 256 MiB write, outside the timed events).  `e2e` repeats the loop through
the Python binding with the step's inputs copied from pinned host memory and
the output copied back inside the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun every rank runs the same per-GPU workload (weak scaling, no
data-path collective); the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from long_context_decode_dual_b200 import workloads as W  # noqa: E402

METRIC = "KV tokens scanned/s per decode step (INT2, 40% pruned); % of HBM peak GB/s"
UNIT = "KV tokens scanned/s"
DEFAULT_WORKLOAD = "longctx_b1_128k"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20
L2_BYTES = 126 << 20                # B200 L2
MAX_ROTATED_CACHES = 8
CSRC = os.path.join(ROOT, "long_context_decode_dual_b200", "csrc")
PROFILES = os.path.join(ROOT, "profiles")


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ---------------------------------------------------------------- helpers
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def decode_source_hash() -> str:
    """Hash of the sources of the decode kernels whose DRAM traffic profiles/
    records (the fused step and the three-call decode in kvq_decode_mma.cu,
    the CUDA-core decode in kvq_decode_simt.cu, the internal header)."""
    h = hashlib.sha256()
    for name in sorted(os.listdir(CSRC)):
        if name in ("kvq_decode_mma.cu", "kvq_decode_simt.cu") or name.endswith(".cuh"):
            with open(os.path.join(CSRC, name), "rb") as f:
                h.update(name.encode())
                h.update(f.read())
    return h.hexdigest()[:16]


def committed_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from a committed ncu summary
    (profiles/traffic_<kernel>_<workload>.txt, the workload name carrying its
    cache format), if it was taken on the current kernel source."""
    try:
        kv = {}
        with open(os.path.join(PROFILES, f"traffic_{kernel}_{workload}.txt")) as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    a, b = line.split(":", 1)
                    kv[a.strip()] = b.strip()
        if kv.get("kernel_source_sha") != decode_source_hash():
            return None, "stale"
        return float(kv["dram_bytes_per_launch"]), kv.get("note", "")
    except Exception:
        return None, "absent"


def algorithmic_step_bytes(wl: W.Workload, k: int, length: int, protect=(0, 0)) -> int:
    """Bytes one fused step launch must move: the decode bytes over `length`
    tokens, A^{-T} of every KV head and the A columns the appending CTAs read
    (float64, 128 x 128 each), the query rows and the new token's key and
    value (bf16 or f32); with a value rotation, its matrix once for the
    appending CTAs and once per (sequence, KV head) for the merge; with a
    refinement, its 128 scales per KV head."""
    elem = 2 if wl.dtype == "bf16" else 4
    transforms = 2 * wl.n_kv_heads * 128 * 128 * 8
    if wl.rotate_values:
        transforms += (wl.n_kv_heads + wl.batch * wl.n_kv_heads) * 128 * 128 * 8
    if wl.refine:
        transforms += wl.n_kv_heads * 128 * 8
    inputs = wl.batch * (wl.n_q_heads + 2 * wl.n_kv_heads) * 128 * elem
    return algorithmic_decode_bytes(wl, k, length, protect) + transforms + inputs


# fp64 FMA throughput of a B200 from its unit counts and clock (not measured):
# 64 fp64 FMA lanes per SM and clock, 148 SMs, 1965 MHz maximum SM clock
FP64_FMA_PEAK_PER_S = 64 * 148 * 1965e6


def prefill_roofline(wl: W.Workload, prefill_ms: float) -> dict:
    """The prefill append is bound by its fixed-order fp64 transforms: per
    token and KV head, K' = K A (128 x 128 fma), and with a value rotation V Rv
    as many again.  Achieved fp64 FMA/s over the derived peak."""
    per_token = 128 * 128 * (2 if wl.rotate_values else 1)
    fmas = wl.batch * wl.n_kv_heads * wl.n_ctx * per_token
    achieved = fmas / (prefill_ms * 1e-3)
    return {"bound": "alu", "unit": "fp64 FMA/s", "fma_per_token_head": per_token,
            "achieved": achieved, "peak": FP64_FMA_PEAK_PER_S, "frac": achieved / FP64_FMA_PEAK_PER_S,
            "peak_source": "derived: 64 fp64 FMA lanes/SM/clock x 148 SMs x 1965 MHz"}


def algorithmic_decode_bytes(wl: W.Workload, k: int, length: int, protect=(0, 0)) -> int:
    """Bytes one decode launch must read: per (sequence, KV head) and page of
    coded tokens, the k-1 selected key rows, the value codes, channel 0 and
    both metadata blocks; with a protected tier (n_sink, n_recent), the pages
    cover only the coded tokens and each protected token adds its k selected
    BF16 key channels and its 128 BF16 values.  The selection inputs and the
    partial outputs are ignored (< 0.1%); so is the value rotation's matrix
    that the merge reads (128 KB per sequence and KV head)."""
    n_sink, n_recent = protect
    R = 128 * wl.bits // 8
    meta = 4 * 128 * (128 // wl.quant_group)            # bytes of one metadata block
    per_page = (k - 1) * R + 128 * R + 256 + 2 * meta
    sink_end = min(n_sink, length)
    recent_start = max(sink_end, length - n_recent)
    n_pages = (recent_start + 127) // 128
    n_prot = sink_end + (length - recent_start)
    return wl.batch * wl.n_kv_heads * (n_pages * per_page + n_prot * (2 * k + 256))


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.proc = None
        self.uuid = uuid

    def __enter__(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.uuid:
            cmd.insert(1, f"--id={self.uuid}")
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self):
        rows = [r.split(", ") for r in (self.out or "").strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.strip() == "Active"})
        hi = sorted(sm)[len(sm) // 2:] if sm else []
        return {"sm_mhz": statistics.median(hi) if hi else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------ oracle (CPU)
def oracle_sample(wl: W.Workload, n_steps: int, budget_s: float = 30.0, skip_first: int = 1, protect=(0, 0)):
    """Time the fp64 CPU oracle on a bounded sample of the workload: one
    (sequence 0, KV head 0) unit with the full context, n_steps decode steps
    (append one token, transform the query and select, attend), with the
    workload's format (group, value rotation and clip, refinement, protected
    tier)."""
    from oracle import oracle as orc
    A, Ai = (x[0] for x in W.make_transforms(wl.with_(n_kv_heads=1)))
    delta = W.make_deltas(wl.with_(n_kv_heads=1))
    delta = None if delta is None else delta[0]
    Rv = W.make_value_rotations(wl.with_(n_kv_heads=1))
    Rv = None if Rv is None else Rv[0]
    vals = (lambda v: v) if Rv is None else (lambda v: orc.value_rotate(v, Rv))
    rope = W.make_rope(wl)
    if rope is None:
        keys = lambda k, pos0: orc.transform(k, A)                          # noqa: E731
    else:
        keys = lambda k, pos0: orc.bucket_keys(k, A, rope, wl.bucket, pos0)  # noqa: E731
    n_sink, n_recent = protect
    K, V = W.make_kv_unit(wl, 0, 0)
    gq = wl.quant_group
    unit = orc.new_unit(wl.capacity, wl.bits, gq)
    slots = orc.new_slots(n_sink, n_recent)
    Kp, Vr = keys(W.as_float(K, wl.dtype), 0), vals(W.as_float(V, wl.dtype))
    orc.append_unit(unit, wl.bits, 0, Kp, Vr, group=gq, vclip=wl.v_clip)
    length = wl.n_ctx
    if n_sink + n_recent:
        orc.protect_store(slots, n_sink, n_recent, 0, Kp, Vr, length)
    g = wl.group_size
    times, tokens = [], []
    t_start = time.perf_counter()
    for i in range(n_steps):
        kn, vn = W.make_step_kv(wl, i)
        q = W.make_q(wl, i)
        t0 = time.perf_counter()
        kp, vr = keys(W.as_float(kn[0, 0], wl.dtype), length), vals(W.as_float(vn[0, 0], wl.dtype))
        orc.append_unit(unit, wl.bits, length, kp, vr, group=gq, vclip=wl.v_clip)
        length += 1
        if rope is not None:
            if n_sink + n_recent:
                orc.protect_store(slots, n_sink, n_recent, length - 1, kp, vr, length)
            qpb = orc.bucket_queries(W.as_float(q[0, :g], wl.dtype), Ai, rope, -(-length // wl.bucket))
            orc.decode_unit_buckets(unit, wl.bits, length, qpb, wl.sparsity, wl.bucket, gq, delta=delta, Rv=Rv,
                                    slots=slots, n_sink=n_sink, n_recent=n_recent)
            times.append(time.perf_counter() - t0)
            tokens.append(length)
            if time.perf_counter() - t_start > budget_s and i >= 1:
                break
            continue
        qp = orc.transform(W.as_float(q[0, :g], wl.dtype), Ai)
        if n_sink + n_recent:
            orc.protect_store(slots, n_sink, n_recent, length - 1, kp, vr, length)
            orc.decode_unit_protected(unit, slots, wl.bits, length, qp, wl.sparsity, n_sink, n_recent, gq,
                                      delta=delta, Rv=Rv)
        else:
            orc.decode_unit(unit, wl.bits, length, qp, wl.sparsity, gq, delta=delta, Rv=Rv)
        times.append(time.perf_counter() - t0)
        tokens.append(length)
        if time.perf_counter() - t_start > budget_s and i >= 1:
            break
    skip = min(skip_first, len(times) - 1)
    value = sum(tokens[skip:]) / sum(times[skip:])
    sample = (f"1 of {wl.batch * wl.n_kv_heads} (sequence, KV head) units, full {wl.n_ctx}-token "
              f"context, {len(times) - skip} timed decode steps (append+select+attend), fp64, "
              f"single thread")
    return value, times[skip:], sample


# ------------------------------------------------------------ reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = W.workload(args.workload, **({"sparsity": args.sparsity} if args.sparsity is not None else {}),
                    bits=args.bits, n_steps=args.warmup + args.steps + 1, **format_overrides(args))
    from oracle import oracle as orc
    k = orc.num_selected(wl.sparsity)
    protect = protect_of(args)
    value, times, sample = oracle_sample(wl, args.warmup + args.steps, budget_s=1e9,
                                         skip_first=args.warmup, protect=protect)
    tokens_per_s = value
    line = {
        "impl": "reference", "metric": METRIC, "value": tokens_per_s, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.mean(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(wl, k, protect),
        "cpu_baseline": {"value": tokens_per_s, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample, "host": host_cpu()},
        "e2e": {"value": tokens_per_s, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


L2_FLUSHED = "flushed between steps (256 MiB write, outside the timed events)"


def config_dict(wl: W.Workload, k: int, protect=(0, 0), l2: str = L2_FLUSHED):
    d = {"workload": wl.name, "batch": wl.batch, "n_q_heads": wl.n_q_heads,
         "n_kv_heads": wl.n_kv_heads, "context": wl.n_ctx, "head_dim": 128, "bits": wl.bits,
         "group": wl.quant_group, "sparsity": wl.sparsity, "k": k, "input_dtype": wl.dtype,
         "arithmetic": "f16 x f16 -> f32 tensor-core products of exact codes, f32 softmax, f64 transforms",
         "step": "append 1 token + query transform/select + decode + merge",
         "l2": l2}
    if protect != (0, 0):
        d["protected_bf16"] = {"sink": protect[0], "recent": protect[1]}
    if wl.rotate_values:
        d["value_rotation"] = {"clip": wl.v_clip}
    if wl.refine:
        d["diagonal_refinement"] = True
    if wl.bucket:
        d["rope_bucket"] = wl.bucket
    return d


def host_cpu() -> dict:
    """The host the CPU baseline ran on: logical CPUs and model name."""
    model = ""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "model": model}


def format_overrides(args) -> dict:
    """Workload fields of the cache format the flags ask for."""
    d = {"quant_group": args.group, "bucket": args.bucket}
    if args.rotate_values:
        d.update(rotate_values=True, v_clip=0.92)
    if args.refine:
        d["refine"] = True
    return d


def protect_of(args):
    return (64, 256) if args.protect else (0, 0)


def format_tag(wl: W.Workload, protect=(0, 0)) -> str:
    """Suffix naming a cache format other than the default (groups of 32,
    no tier, no rotation, no refinement, no RoPE buckets): the pages' whole
    recipe is "_pages", anything else lists its parts."""
    parts = [p for p, on in (("g128", wl.quant_group == 128), ("tier", protect != (0, 0)),
                             ("rot", wl.rotate_values), ("ref", wl.refine), (f"bkt{wl.bucket}", wl.bucket > 0)) if on]
    if len(parts) == 5 and wl.bucket == 2048:
        return "_pages"
    return "_" + "-".join(parts) if parts else ""


# ------------------------------------------------------------- ranks
# More than one GPU runs independent replicas (weak scaling): rank r decodes
# its own sequences (the workload's seed offset by r), no data crosses GPUs,
# and the job's time is the slowest rank's.
def rank_workload(wl: W.Workload, rank: int) -> W.Workload:
    return wl if rank == 0 else wl.with_(seed=wl.seed + 7919 * rank)


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest x over all ranks (every rank calls this, in the same order)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: float, max_ms: float, world: int) -> float:
    """Units all ranks processed per second, over the slowest rank's time."""
    return world * tokens_per_rank / (max_ms * 1e-3)


# ------------------------------------------------------------- our arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    from long_context_decode_dual_b200 import kvq

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    kvq.lib()

    n_pool = 8
    total_steps = args.warmup + args.steps
    n_appends = total_steps * (2 if args.e2e else 1) + 1
    over = {"bits": args.bits, "n_steps": n_appends, **format_overrides(args)}
    if args.sparsity is not None:
        over["sparsity"] = args.sparsity
    if args.batch is not None:
        over["batch"] = args.batch
    wl = rank_workload(W.workload(args.workload, **over), rank)
    B, Hq, Hkv = wl.batch, wl.n_q_heads, wl.n_kv_heads

    t0 = time.perf_counter()
    A_np, Ai_np = W.make_transforms(wl)
    K_np, V_np = W.make_kv(wl)
    log(f"[bench] inputs generated in {time.perf_counter() - t0:.1f}s")

    def dev_in(x):
        if wl.dtype == "f32":
            return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(dev)
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(dev).view(torch.bfloat16)

    A = torch.from_numpy(A_np).to(dev)
    Ai = torch.from_numpy(Ai_np).to(dev)
    Kd, Vd = dev_in(K_np), dev_in(V_np)
    stream = torch.cuda.current_stream(dev)

    protect = protect_of(args)
    Rv_np, delta_np = W.make_value_rotations(wl), W.make_deltas(wl)
    Rv = None if Rv_np is None else torch.from_numpy(Rv_np).to(dev)
    delta = None if delta_np is None else torch.from_numpy(delta_np).to(dev)
    rope_np = W.make_rope(wl)
    rope = None if rope_np is None else torch.from_numpy(rope_np).to(dev)
    k = kvq.num_selected(wl.sparsity)
    alg_fn = algorithmic_step_bytes if args.fused else algorithmic_decode_bytes
    # Cold L2 for every timed step: when one step reads enough, R copies of
    # the cache (each with its own transforms) are used in turn, so the R - 1
    # steps between two uses of a copy move more than twice the L2 through it
    # and the steps run back to back; otherwise L2 is flushed before each step.
    step_bytes = alg_fn(wl, k, wl.n_ctx, protect)
    n_rot = int(np.ceil(2 * L2_BYTES / max(step_bytes, 1))) + 1
    rotate = n_rot <= MAX_ROTATED_CACHES
    n_copies = n_rot if rotate else 1
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    caches, steps = [], []
    prefill_ms = None
    for r in range(n_copies):
        cache = kvq.new_cache(B, Hkv, wl.capacity, wl.bits, device=dev, n_sink=protect[0], n_recent=protect[1],
                              group=wl.quant_group, v_rot=Rv, v_clip=wl.v_clip, bucket=wl.bucket, rope=rope)
        Ar, Air = (A, Ai) if r == 0 else (A.clone(), Ai.clone())
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record()
        kvq.append(cache, Kd, Vd, Ar)
        ev1.record()
        torch.cuda.synchronize(dev)
        # the fastest of the copies' prefills (the first call also loads the module)
        ms = ev0.elapsed_time(ev1)
        prefill_ms = ms if prefill_ms is None else min(prefill_ms, ms)
        assert kvq.read_status(cache) == 0
        caches.append(cache)
        steps.append(kvq.DecodeStep(cache, Ar, Air, wl.sparsity, Hq, tdt, fused=args.fused, delta=delta))
    cache, step = caches[0], steps[0]
    log(f"[bench] {n_copies} cache cop{'ies' if n_copies > 1 else 'y'}, "
        f"{'rotated' if rotate else 'L2 flushed between steps'}")

    q_pool = [dev_in(W.make_q(wl, i)) for i in range(n_pool)]
    kv_pool = [tuple(dev_in(t) for t in W.make_step_kv(wl, i)) for i in range(n_pool)]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def stage(st, i):
        st.q.copy_(q_pool[i % n_pool])
        st.k_new.copy_(kv_pool[i % n_pool][0])
        st.v_new.copy_(kv_pool[i % n_pool][1])

    # step: one kvq_decode_step call = one fused launch (with RoPE buckets
    # three: the append, the per-bucket choice as its programmatic dependent,
    # the decode as the choice's); unfused: one-token append (with its length
    # advance), select, decode (with its merge)
    launches_per_step = (3 if wl.bucket else 1) if args.fused else 3
    lengths = [wl.n_ctx] * n_copies
    for st in steps:
        st.time_decode()
    for i in range(max(args.warmup, n_copies)):
        r = i % n_copies
        stage(steps[r], i)
        steps[r].run()
        lengths[r] += 1
        if i < n_copies and args.graph:
            torch.cuda.synchronize(dev)
            steps[r].capture()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()

    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    a, b_ = E(), E()
    step_ms, dec_ms, alg_bytes, tokens = [], [], [], []
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    # The K steps are queued back to back, each bracketed by its own pair of
    # events on the launching stream (the next step's inputs, and the L2
    # flush when the copies are not rotated, between them outside the
    # events); one synchronize at the end.  (A synchronize after every step
    # would leave the GPU idle before each launch and add the host's launch
    # latency to every step; a serving loop keeps launches queued ahead of the
    # GPU in the same way.)
    step_ev = [(E(), E()) for _ in range(args.steps)]
    dec_ev = [(E(), E()) for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    with ClockSampler(uuid) as clocks:
        # a head start for the host: a clock-counting kernel keeps the GPU busy
        # (outside every step's events) while the K steps are submitted, so
        # the GPU then runs them without waiting for the host between them
        torch.cuda._sleep(int(2e6 * max(5, args.steps)))
        for i in range(args.steps):
            j = max(args.warmup, n_copies) + i
            r = j % n_copies
            st = steps[r]
            stage(st, j)
            if not rotate:
                flush.fill_(i & 0xFF)
            st.decode_events = dec_ev[i]
            step_ev[i][0].record()
            st.run()
            step_ev[i][1].record()
            lengths[r] += 1
            alg_bytes.append(alg_fn(wl, k, lengths[r], protect))
            tokens.append(B * Hkv * lengths[r])
        torch.cuda.synchronize(dev)
    step_ms = [x.elapsed_time(y) for x, y in step_ev]
    dec_ms = [x.elapsed_time(y) for x, y in dec_ev]
    if world > 1:
        dist.barrier()
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    value = job_throughput(sum(tokens), total_ms, world)
    assert kvq.read_status(cache) == 0

    # roofline of the dominant kernel (decode partial + merge, timed together;
    # a bucketed step's preparation kernel runs under the decode's first
    # pages, so there the events bracket both launches)
    hbm_peak, peak_src = measured_peaks()
    alg_bytes = [alg_fn(wl, k, tok // (B * Hkv), protect) for tok in tokens]
    # bytes over time of all timed launches (not a mean of per-step ratios)
    achieved = sum(alg_bytes) / (sum(dec_ms) * 1e-3) / 1e9
    traffic, traffic_note = committed_traffic("step_mma" if args.fused else "decode_mma",
                                              wl.name + format_tag(wl, protect))

    # end to end through the Python binding with host buffers
    e2e = None
    if args.e2e:
        npdt = np.int16 if wl.dtype == "bf16" else np.float32
        pin = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(npdt)).pin_memory()  # noqa: E731
        as_t = (lambda t: t.view(torch.bfloat16)) if wl.dtype == "bf16" else (lambda t: t)
        qh = [as_t(pin(W.make_q(wl, i))) for i in range(n_pool)]
        kvh = [tuple(as_t(pin(t)) for t in W.make_step_kv(wl, i)) for i in range(n_pool)]
        e_tok, e_ms = [], 0.0
        length = lengths[0]
        torch.cuda.synchronize(dev)
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            a.record()
            j = i % n_pool
            # inputs from pinned host memory in one copy, the step, the
            # result back to pinned host memory in one copy (one graph replay)
            step.run_host(qh[j], kvh[j][0], kvh[j][1])
            b_.record()
            torch.cuda.synchronize(dev)
            e_ms += a.elapsed_time(b_)
            length += 1
            e_tok.append(B * Hkv * length)
        e_ms = max_over_ranks(e_ms, world, dev)
        e2e = {"value": job_throughput(sum(e_tok), e_ms, world), "unit": UNIT,
               "h2d_bytes_per_step": step.h2d_bytes, "d2h_bytes_per_step": step.d2h_bytes}

    # the unpruned BF16 comparator on the same keys and values
    comparator = None
    if args.comparator and wl.dtype == "bf16":
        n_tok = wl.n_ctx
        qc = q_pool[0]
        cws = kvq.alloc_workspace(kvq.bf16_workspace_bytes(B, Hq, Hkv, n_tok), dev)
        cout = torch.empty(B, Hq, 128, dtype=torch.float32, device=dev)
        for _ in range(3):
            kvq.bf16_decode_attn(qc, Kd, Vd, out=cout, ws=cws)
        # its keys and values (512 B per token and KV head) are larger than L2
        # by themselves: calls back to back, each between its own events
        n_cmp = max(5, min(args.steps, 20))
        c_ev = [(E(), E()) for _ in range(n_cmp)]
        torch.cuda.synchronize(dev)
        torch.cuda._sleep(int(4e6 * n_cmp))
        for i in range(n_cmp):
            c_ev[i][0].record()
            kvq.bf16_decode_attn(qc, Kd, Vd, out=cout, ws=cws)
            c_ev[i][1].record()
        torch.cuda.synchronize(dev)
        c_ms = [x.elapsed_time(y) for x, y in c_ev]
        cb = B * Hkv * n_tok * 512
        cm = statistics.mean(c_ms)
        comparator = {"kernel": "bf16 unpruned decode attention", "ms": cm,
                      "tokens_per_s": B * Hkv * n_tok / (cm * 1e-3),
                      "achieved_gbs": cb / (cm * 1e-3) / 1e9, "frac_of_peak": cb / (cm * 1e-3) / 1e9 / hbm_peak,
                      "speedup_of_int2_decode": cm / statistics.mean(dec_ms)}

    # CPU baseline: the oracle on a bounded sample (rank 0, one GPU only)
    cpu = None
    if args.cpu_baseline and world == 1:
        cv, ct, sample = oracle_sample(wl.with_(n_steps=8), 6, budget_s=25.0, protect=protect)
        cpu = {"value": cv, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample,
               "host": host_cpu()}

    csum = clocks.summary()
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": config_dict(wl, k, protect, l2=(
            f"inputs larger than L2: {n_copies} copies of the cache ({n_copies} x {caches[0].pages.numel() >> 20} MiB, "
            f"each with its own transforms) used in turn, steps back to back" if rotate else L2_FLUSHED)),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "traffic": traffic,
                     "kernel": ("fused step (kvq_decode_step: append + select + decode + merge)" if args.fused
                                else "decode partial + merge (kvq_decode_attn)"),
                     "peak_source": f"{peak_src} hbm_gbs", "traffic_note": traffic_note},
        "ms_per_step_median": statistics.median(step_ms),
        "decode_ms": statistics.mean(dec_ms),
        "step_launch": "cuda graph" if args.graph else "eager",
        "decode_alg_bytes": statistics.mean(alg_bytes),
        "prefill_ms": prefill_ms,
        "prefill_roofline": prefill_roofline(wl, prefill_ms),
        # the prefill reads K and V once and writes the pages (and slots)
        "prefill_gbs": (Kd.numel() * Kd.element_size() * 2 + cache.pages.numel()) / (prefill_ms * 1e-3) / 1e9,
        "seq_tokens_per_s": world * B * statistics.mean(tokens) / (B * Hkv) / (total_ms / args.steps * 1e-3),
        "gpu_launches": launches_per_step * args.steps,
        "clocks": csum,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "comparator": comparator,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(W.WORKLOADS))
    ap.add_argument("--sparsity", type=float, default=None)
    ap.add_argument("--batch", type=int, default=None,
                    help="sequences per step (default: the workload's); for smaller profiling captures")
    ap.add_argument("--bits", type=int, default=2, choices=[2, 4])
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--no-comparator", dest="comparator", action="store_false")
    ap.add_argument("--group", type=int, default=32, choices=[32, 128],
                    help="channels per quantization group (128: the pages' one grid per token)")
    ap.add_argument("--protect", action="store_true",
                    help="keep the first 64 and the last 256 tokens in BF16 (the pages' protected tier)")
    ap.add_argument("--rotate-values", action="store_true",
                    help="rotate the values before quantization, clip their grids at 0.92, rotate the output back")
    ap.add_argument("--refine", action="store_true",
                    help="fold a diagonal refinement into the transforms; select on the base queries")
    ap.add_argument("--bucket", type=int, default=0,
                    help="tokens per bucket of bucket-relative RoPE (the pages use 2048; 0: none)")
    ap.add_argument("--pages-recipe", action="store_true",
                    help="the pages' whole format: --group 128 --protect --rotate-values --refine --bucket 2048")
    ap.add_argument("--unfused", dest="fused", action="store_false",
                    help="run the step as three launches (append, select, decode) instead of one")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="launch the step's kernels eagerly instead of replaying a CUDA graph")
    args = ap.parse_args()
    if args.pages_recipe:
        args.group, args.protect, args.rotate_values, args.refine = 128, True, True, True
        args.bucket = 2048
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
