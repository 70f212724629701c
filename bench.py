"""Benchmark of the paged decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload llama7b|llama3_8b|beam|long32k|tiny|swap] [--seed S]

One step is the whole hot path once over one batch: copy-on-write block
copies (when the workload has any), the cache write of the step's new tokens,
and paged decode attention of every sequence. The default workload is the
LLaMA-7B-shaped decode batch (64 sequences, 32 heads, head_dim 128,
block_size 16, fp16, contexts uniform in [128, 2048]); its KV cache (~1.1 GB
read per step) is larger than the 126 MB L2, so no L2 flush is needed.

Under torchrun every rank runs its own replica of the workload on its own GPU
(weak scaling, no collective on the data path); rank 0 prints one JSON line
with the max-over-ranks device time.

--impl reference times the fp64 CPU oracle on the host cores over a bounded
sample of the same workload (rank 0 only). --workload swap measures
pa_swap_blocks between the GPU pools and page-locked host memory instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention: seqs/s and KV GB/s as % of B200 HBM peak, 1 GPU"
FALLBACK_HBM_GBS = 6650.0
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama7b")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--partition", type=int, default=None)
    ap.add_argument("--kv", default="auto", choices=["auto", "fp8", "e4m3h", "int8", "e4m3b", "int8b"],
                    help="fp8: E4M3 KV cache, one scale per tensor (pa_reshape_and_cache_fp8 + pa_decode_fp8); "
                         "e4m3h / int8: E4M3 / INT8 codes with one scale per KV head, spanning 100x "
                         "(pa_reshape_and_cache_quant + pa_decode_quant); e4m3b / int8b: one scale per "
                         "(block, KV head), spanning 100x (pa_reshape_and_cache_quant_blocks + "
                         "pa_decode_quant_blocks)")
    ap.add_argument("--unfused", action="store_true",
                    help="separate cache-write launch instead of pa_decode_append")
    ap.add_argument("--share", default="auto", choices=["auto", "on", "off"],
                    help="pa_decode_shared (blocks shared by several sequences streamed once per group); "
                         "auto: on when the workload's tables share blocks")
    ap.add_argument("--block-size", type=int, default=None,
                    help="llama7b / llama3_8b at another block size (16, 32 or 64)")
    ap.add_argument("--head-dim", type=int, default=None,
                    help="llama7b / llama3_8b at another head size (64 or 128)")
    ap.add_argument("--kv-heads", type=int, default=None,
                    help="llama3_8b with another KV head count (32 query heads: 4 gives 8 per KV head)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    return ap.parse_args()


def shape_args(args) -> dict:
    kw = {}
    if args.block_size is not None:
        kw["block_size"] = args.block_size
    if args.head_dim is not None:
        kw["head_dim"] = args.head_dim
    if kw and args.workload not in ("llama7b", "llama3_8b"):
        raise SystemExit("--block-size / --head-dim apply to llama7b and llama3_8b")
    if getattr(args, "kv_heads", None) is not None:
        if args.workload != "llama3_8b":
            raise SystemExit("--kv-heads applies to llama3_8b")
        kw["kv_heads"] = args.kv_heads
    return kw


def describe(wl) -> dict:
    st = wl.steps[0]
    ctx = st.context_lens
    return {"workload": wl.name, "num_seqs": int(len(ctx)), "num_heads": wl.num_heads,
            "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim, "block_size": wl.block_size,
            "num_blocks": wl.num_blocks, "context_mean": float(ctx.mean()),
            "context_min": int(ctx.min()), "context_max": int(ctx.max()),
            "new_tokens_per_step": int(len(st.slot_mapping)),
            "copy_pairs_per_step": int(len(st.copy_pairs)),
            "kv_bytes_per_step": int(wl.kv_bytes()), "kv_bytes_unique_per_step": int(wl.kv_bytes_unique()),
            "steps_in_plan": len(wl.steps),
            "l2": "L2 flushed before every step (256 MiB written, then another 256 MiB read, so that the "
                  "lines left are clean), outside the step's events"
            if needs_flush(wl) else
            "no flush: KV read per step (%.2f GB) exceeds the 126 MB L2" % (wl.kv_bytes_unique() / 1e9)}


L2_BYTES = 126 * 1024 * 1024
FP8_SCALE = 0.0375  # N(0,1) values / 0.0375 stay well inside E4M3's +-448
INT8_SCALE = 0.035  # about max |N(0,1)| / 127 over a pool


def block_scales(nb: int, n: int, base: float, seed: int) -> torch.Tensor:
    """Per-(block, KV head) scales from base / 10 to base * 10, seeded."""
    g = torch.Generator().manual_seed(seed)
    return (base * 10.0 ** (2.0 * torch.rand((nb, n), generator=g, dtype=torch.float64) - 1.0)).float()


def head_scales(n: int, base: float) -> torch.Tensor:
    """Per-KV-head scales from base / 10 to base * 10 (100x), neighbours apart."""
    s = base * 10.0 ** np.linspace(-1.0, 1.0, n)
    order = np.argsort(np.arange(n) % 2 * n + np.arange(n))
    return torch.tensor(s[order], dtype=torch.float32)


def non_kv_bytes(wl, P: int, fused: bool, shared: bool) -> dict:
    """Bytes a decode call moves besides the K/V rows of valid tokens, from the
    workload's shapes (the mean over its steps): the query rows read and the
    output rows written, the block-table entries and context lengths, the fp32
    partials of split sequences (written by the attention kernel and read by
    the merge: per partition and query head D floats and a (max, sum) pair;
    with shared-prefix units one more partition per sequence, an upper bound),
    and the new K/V rows the fused append reads and writes."""
    H, Hkv, D, bs = wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size
    e = 2
    acc = {"q_and_out": 0.0, "tables_and_contexts": 0.0, "partials": 0.0, "appended_rows": 0.0}
    for st in wl.steps:
        B = len(st.context_lens)
        ctx = st.context_lens.astype(np.int64)
        acc["q_and_out"] += 2 * B * H * D * e
        acc["tables_and_contexts"] += 4 * int((-(-ctx // bs)).sum()) + 4 * B
        nparts = -(-ctx // P) + (1 if shared else 0)
        split = nparts[nparts > 1]
        acc["partials"] += 2 * int(split.sum()) * H * (D * 4 + 8)
        if fused:
            acc["appended_rows"] += 2 * 2 * B * Hkv * D * e
    n = len(wl.steps)
    return {k: int(v / n) for k, v in acc.items()}


def needs_flush(wl) -> bool:
    return wl.kv_bytes_unique() < 4 * L2_BYTES


def appends_at_last_positions(wl) -> bool:
    """True when every step's first num_seqs new tokens are each sequence's
    last position, so the fused append + decode entry point applies."""
    for st in wl.steps:
        B = st.q.shape[0]
        for s in range(B):
            n = int(st.context_lens[s])
            if n == 0 or st.slot_mapping[s] != st.block_tables[s, (n - 1) // wl.block_size] * wl.block_size + \
                    (n - 1) % wl.block_size:
                return False
    return True


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# The files that define the decode kernels and how they are launched.
KERNEL_SOURCES = ("pa_common.cuh", "pa_decode.cuh", "pa_decode_mma.cuh", "pa_launch.cuh")


def code_only(text: str) -> str:
    """C++ source without comments and blank space: edits to comments leave
    the compiled kernels, and so their digest, unchanged."""
    out, i, n = [], 0, len(text)
    while i < n:
        if text.startswith("//", i):
            i = text.find("\n", i)
            i = n if i < 0 else i
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif text[i] == '"':  # string literal, kept as is
            j = i + 1
            while j < n and text[j] != '"':
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            out.append(text[i])
            i += 1
    return " ".join("".join(out).split())


def source_digest() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_372_b200", "csrc")
    for name in KERNEL_SOURCES:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + code_only(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the decode kernel from a committed ncu capture,
    only while the kernel sources are unchanged since that capture."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            d = json.load(f)
        e = d.get(workload)
        if e and e.get("source_digest") == source_digest():
            return e["dram_bytes_per_launch"]
    except Exception:
        pass
    return None


class Clocks:
    """nvidia-smi sampling during the timed region."""

    def __init__(self, index: int):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(index),
                 "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            return None
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 7:
                continue
            try:
                sm.append(float(f[0]))
                mx = max(mx, float(f[1]))
            except ValueError:
                continue
            for n, v in zip(names, f[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


# ------------------------------------------------------------------------------
def run_ours(args, world, rank, local, extras=True):
    """The hot path of args.workload timed on this rank's GPU; with `extras`
    also the end-to-end figure and (rank 0, one GPU) the CPU baseline."""
    import paged_kv_cache_372_b200 as pa
    from paged_kv_cache_372_b200 import build, workloads
    build.build()
    dev = torch.device("cuda", local if world > 1 else 0)
    wl = workloads.build(args.workload, args.seed + rank, **shape_args(args))
    st0 = wl.steps[0]
    B = int(len(st0.context_lens))
    kp, vp = wl.k_pool.to(dev), wl.v_pool.to(dev)
    P = wl.partition_size if args.partition is None else args.partition
    max_ctx = max(int(s.context_lens.max()) for s in wl.steps)
    ws = pa.alloc_workspace(B, wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size, max_ctx, P, dev)
    nsteps = len(wl.steps)
    dev_steps = []
    for st in wl.steps:
        dev_steps.append(dict(
            q=st.q.to(dev), out=torch.empty_like(st.q, device=dev),
            tables=torch.from_numpy(st.block_tables).to(dev), ctx=torch.from_numpy(st.context_lens).to(dev),
            k=st.k_new.to(dev), v=st.v_new.to(dev), slots=torch.from_numpy(st.slot_mapping).to(dev),
            pairs=torch.from_numpy(st.copy_pairs).to(dev)))
    stream = torch.cuda.current_stream(dev)
    flush = needs_flush(wl)
    flush_w = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if flush else None
    flush_r = torch.zeros(2 * L2_BYTES // 8, dtype=torch.int64, device=dev) if flush else None

    def flush_l2(i):
        """Evict the previous step's blocks from L2: write a buffer twice the
        L2's size, then read another as large, so that the dirty lines the
        write leaves are written back here and not during the next step."""
        flush_w.fill_(i & 0xff)
        flush_r.sum()

    kv8 = args.kv in ("fp8", "e4m3h", "int8", "e4m3b", "int8b")
    quant = args.kv in ("e4m3h", "int8", "e4m3b", "int8b")
    per_block = args.kv in ("e4m3b", "int8b")
    qfmt = {"e4m3h": "e4m3", "int8": "int8", "e4m3b": "e4m3", "int8b": "int8"}.get(args.kv)
    if quant:
        base = INT8_SCALE if qfmt == "int8" else FP8_SCALE
        if per_block:
            ksc = block_scales(kp.shape[0], wl.num_kv_heads, base, args.seed + 61).to(dev)
            vsc = block_scales(kp.shape[0], wl.num_kv_heads, base, args.seed + 62).to(dev)
        else:
            ksc = head_scales(wl.num_kv_heads, base).to(dev)
            vsc = head_scales(wl.num_kv_heads, base).flip(0).contiguous().to(dev)
    write_quant = pa.pa_reshape_and_cache_quant_blocks if per_block else pa.pa_reshape_and_cache_quant
    if kv8:
        ws = pa.alloc_workspace(B, wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size, max_ctx, P, dev,
                                fp8=True)
    fused = not args.unfused and not kv8 and appends_at_last_positions(wl)
    share = ((quant and not per_block) or not kv8) and (args.share == "on" or
                                     (args.share == "auto" and wl.kv_bytes_unique() < wl.kv_bytes()))
    if share:
        ws = pa.alloc_workspace(B, wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size, max_ctx, P, dev,
                                shared=True)
    if kv8:
        # The whole cache quantised once by the library's own E4M3 cache write.
        NB, Hkv, bs, D = kp.shape
        k8 = torch.empty((NB, Hkv, bs, D), dtype=torch.uint8, device=dev)
        v8 = torch.empty_like(k8)
        all_slots = torch.arange(NB * bs, dtype=torch.int64, device=dev)
        krows = kp.permute(0, 2, 1, 3).reshape(NB * bs, Hkv, D).contiguous()
        vrows = vp.permute(0, 2, 1, 3).reshape(NB * bs, Hkv, D).contiguous()
        if quant:
            write_quant(krows, vrows, k8, v8, all_slots, qfmt, ksc, vsc)
        else:
            pa.pa_reshape_and_cache_fp8(krows, vrows, k8, v8, all_slots, FP8_SCALE, FP8_SCALE)
        del krows, vrows
        del kp, vp
        kp, vp = k8, v8
    for d in dev_steps:
        d["k_dec"], d["v_dec"] = d["k"][:B].contiguous(), d["v"][:B].contiguous()
        d["k_extra"], d["v_extra"], d["slots_extra"] = d["k"][B:], d["v"][B:], d["slots"][B:]

    def step(i, ev=None):
        d = dev_steps[i % nsteps]
        if d["pairs"].shape[0]:
            pa.pa_copy_blocks([kp, vp], d["pairs"])
        if quant:
            write_quant(d["k"], d["v"], kp, vp, d["slots"], qfmt, ksc, vsc)
        elif kv8:
            pa.pa_reshape_and_cache_fp8(d["k"], d["v"], kp, vp, d["slots"], FP8_SCALE, FP8_SCALE)
        elif fused:
            if d["slots_extra"].shape[0]:
                pa.pa_reshape_and_cache(d["k_extra"], d["v_extra"], kp, vp, d["slots_extra"])
        else:
            pa.pa_reshape_and_cache(d["k"], d["v"], kp, vp, d["slots"])
        if ev is not None:
            ev[0].record(stream)
        if quant and share:
            pa.pa_decode_shared_quant(d["out"], d["q"], kp, vp, d["tables"], d["ctx"], wl.scale, max_ctx, qfmt,
                                      ksc, vsc, P, ws)
        elif quant and per_block:
            pa.pa_decode_quant_blocks(d["out"], d["q"], kp, vp, d["tables"], d["ctx"], wl.scale, max_ctx, qfmt, ksc,
                                      vsc, P, ws)
        elif quant:
            pa.pa_decode_quant(d["out"], d["q"], kp, vp, d["tables"], d["ctx"], wl.scale, max_ctx, qfmt, ksc, vsc,
                               P, ws)
        elif kv8:
            pa.pa_decode_fp8(d["out"], d["q"], kp, vp, d["tables"], d["ctx"], wl.scale, max_ctx, FP8_SCALE,
                             FP8_SCALE, P, ws)
        elif share:
            kw = dict(k_new=d["k_dec"], v_new=d["v_dec"]) if fused else {}
            pa.pa_decode_shared(d["out"], d["q"], kp, vp, d["tables"], d["ctx"], wl.scale, max_ctx, P, ws, **kw)
        elif fused:
            pa.pa_decode_append(d["out"], d["q"], d["k_dec"], d["v_dec"], kp, vp, d["tables"], d["ctx"], wl.scale,
                                max_ctx, P, ws)
        else:
            pa.pa_decode(d["out"], d["q"], kp, vp, d["tables"], d["ctx"], wl.scale, max_ctx, P, ws)
        if ev is not None:
            ev[1].record(stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    assert pa.pa_device_errors() == 0

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    step_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(args.steps)] if flush else None
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = Clocks(dev.index) if rank == 0 else None
    barrier(world)
    torch.cuda.synchronize(dev)
    launches0 = pa.pa_launch_count()
    # The K steps of the headline figure: no event between the kernels of a
    # step (an event record between two kernels idles the GPU for a moment),
    # unless the L2 flush has to be kept out of the step's time.
    start.record(stream)
    for i in range(args.steps):
        if flush:
            flush_l2(i)
            step_evs[i][0].record(stream)
        step(i)
        if flush:
            step_evs[i][1].record(stream)
    stop.record(stream)
    launches = pa.pa_launch_count() - launches0  # this library's kernels in the K steps
    torch.cuda.synchronize(dev)
    barrier(world)
    total_ms = (sum(a.elapsed_time(b) for a, b in step_evs) if flush else start.elapsed_time(stop))
    # The same K steps again with an event pair around each decode call: the
    # call's own time (decode_ms, the roofline figure) and its spread.
    for i in range(args.steps):
        if flush:
            flush_l2(i)
        step(i, evs[i])
    torch.cuda.synchronize(dev)
    barrier(world)
    clk = clocks.stop() if clocks else None
    dec = np.array([a.elapsed_time(b) for a, b in evs])
    decode_ms = float(dec.mean())
    unflushed = None
    if flush:
        # The same steps with the blocks of the previous step left in L2.
        m = min(args.steps, 200)
        for i in range(m):
            step(i, evs[i])
        torch.cuda.synchronize(dev)
        u = float(np.mean([a.elapsed_time(b) for a, b in evs[:m]]))
        unflushed = {"steps": m, "decode_ms": u}
    total_ms = max_over_ranks(total_ms, world)
    decode_ms_max = max_over_ranks(decode_ms, world)
    ms_per_step = total_ms / args.steps
    seqs = B * world
    value = seqs / (ms_per_step / 1e3)

    eb = 0.5 if kv8 else 1.0   # kv_bytes counts 2-byte elements
    kv_bytes = eb * float(np.mean([wl.kv_bytes(i % nsteps) for i in range(args.steps)]))
    uniq = [wl.kv_bytes_unique(i) for i in range(nsteps)]
    kv_unique = eb * float(np.mean([uniq[i % nsteps] for i in range(args.steps)]))
    peak, peak_kind = measured_peaks()
    achieved = kv_unique / (decode_ms * 1e-3) / 1e9
    result = {
        "metric": METRIC, "value": value, "unit": "seqs/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": (f"{qfmt} KV cache (per-block scales), {wl.dtype} q/out" if per_block else
                                       f"{qfmt} KV cache (per-head scales), {wl.dtype} q/out" if quant else
                                       f"e4m3 KV cache, {wl.dtype} q/out" if kv8 else wl.dtype),
        "data": "synthetic (seeded N(0,1) K/V/Q, shuffled block pool)",
        "config": describe(wl),
        "kv_gbs": kv_unique * world / (ms_per_step * 1e-3) / 1e9,
        "decode_ms": decode_ms_max,
        "decode_ms_p10_p50_p90": [float(x) for x in np.percentile(dec, [10, 50, 90])],
        "decode_kv_gbs": achieved,
        "decode_kv_gbs_logical": kv_bytes / (decode_ms * 1e-3) / 1e9,
        "hbm_frac_of_%s" % peak_kind: achieved / peak,
        "hbm_frac_of_nominal_8000": achieved / 8000.0,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": peak_kind,
                     "kernel": ("pa_decode_shared_quant call (grouping plan + attention launches; split merge "
                                "in a launch of its own)" if quant and share else
                                "pa_decode_quant_blocks call (plan + attention launches; split merge fused up to 16 "
                                "partitions)" if per_block else
                                "pa_decode_quant call (plan + attention launches; split merge fused up to 16 "
                                "partitions)" if quant else
                                "pa_decode_fp8 call (plan + attention launches; split merge fused)" if kv8 else
                                "pa_decode_shared call (grouping plan + attention launches; cache write fused, "
                                "split merge in a launch of its own)" if share and fused else
                                "pa_decode_shared call (grouping plan + attention launches; split merge in a "
                                "launch of its own)" if share else
                                "pa_decode_append call (plan + attention launches; cache write fused, split "
                                "merge fused up to 16 partitions, a launch of its own beyond)" if fused else
                                "pa_decode call (plan + attention launches; split merge fused up to 16 "
                                "partitions, a launch of its own beyond)"),
                     "bytes": "unique K+V bytes of valid tokens per call",
                     "traffic": profiled_traffic(wl.name + (f"@{args.kv}" if kv8 else "") + ("@shared" if share else "")
                                                 + ("" if args.partition is None else f"@P{args.partition}"))},
        "gpu_launches": launches,
        "step": ("pa_copy_blocks (if any), pa_reshape_and_cache_quant, pa_decode_shared_quant" if quant and share
                 else "pa_copy_blocks (if any), pa_reshape_and_cache_quant_blocks, pa_decode_quant_blocks"
                 if per_block else "pa_copy_blocks (if any), pa_reshape_and_cache_quant, pa_decode_quant" if quant else
                 "pa_copy_blocks (if any), pa_reshape_and_cache_fp8, pa_decode_fp8" if kv8 else
                 "pa_copy_blocks (if any), pa_reshape_and_cache of extra tokens (if any), pa_decode_shared with "
                 "the new tokens" if share and fused else
                 "pa_copy_blocks (if any), pa_reshape_and_cache, pa_decode_shared" if share else
                 "pa_copy_blocks (if any), pa_reshape_and_cache of extra tokens (if any), pa_decode_append"
                 if fused else "pa_copy_blocks (if any), pa_reshape_and_cache, pa_decode"),
        "clocks": clk,
    }
    result["shared_prefix_units"] = bool(share)
    B0, mx = wl.num_seqs, int(max(int(st.context_lens.max()) for st in wl.steps))
    part_fn = (pa.pa_decode_shared_partition_size if share else pa.pa_decode_fp8_partition_size if kv8
               else pa.pa_decode_partition_size)
    P_used = part_fn(B0, wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size, mx, P)
    result["non_kv_bytes_per_call"] = non_kv_bytes(wl, P_used, fused, share) if P_used > 0 else None
    result["partition_size"] = P_used
    if unflushed is not None:
        unflushed["decode_kv_gbs"] = kv_unique / (unflushed["decode_ms"] * 1e-3) / 1e9
        unflushed["decode_kv_gbs_logical"] = kv_bytes / (unflushed["decode_ms"] * 1e-3) / 1e9
        result["unflushed"] = unflushed
    if per_block:
        result["config"]["kv_cache"] = (f"{qfmt} codes, one scale per (block, KV head): {base / 10:g} to "
                                        f"{base * 10:g} (100x), drawn per block and head")
        result["config"]["kv_bytes_per_step"] = int(kv_bytes)
    elif quant:
        result["config"]["kv_cache"] = (f"{qfmt} codes, one scale per KV head: {base / 10:g} to {base * 10:g} "
                                        "(100x), keys and values in opposite head order")
        result["config"]["kv_bytes_per_step"] = int(kv_bytes)
    elif kv8:
        result["config"]["kv_cache"] = f"E4M3 codes, k_scale = v_scale = {FP8_SCALE}"
        result["config"]["kv_bytes_per_step"] = int(kv_bytes)
    if extras and not args.no_e2e and not kv8:
        e2e = run_e2e(args, wl, pa, kp, vp, ws, P, max_ctx, dev, world, fused, share)
        if rank == 0:
            result["e2e"] = e2e
    pa.pa_device_errors()
    if extras and rank == 0 and world == 1 and not args.no_cpu and not kv8:
        result["cpu_baseline"] = cpu_baseline(wl)
    return result


# After the default (LLaMA-7B-shaped) line, the Llama-3-8B-shaped GQA batch is
# timed the same way on the same GPU and reported under its own key, so that
# one run covers both decode batches the throughput target names.
# Workloads timed after the default line, in the same run: the Llama-3-8B GQA
# batch, the long-context batch at its own 512-token partitions, and the
# shared-prefix beam batch (each with its own L2 rule).
SECONDARY = {"llama7b": ("llama3_8b", "long32k", "beam")}
SECONDARY_STEPS = 300


def run_secondary(args, world, rank, local, name):
    sub = argparse.Namespace(**vars(args))
    sub.workload, sub.steps = name, min(args.steps, SECONDARY_STEPS)
    r = run_ours(sub, world, rank, local, extras=False)
    keep = ("value", "unit", "steps", "warmup", "ms_per_step", "dtype", "config", "decode_ms",
            "decode_ms_p10_p50_p90", "decode_kv_gbs", "decode_kv_gbs_logical", "roofline", "gpu_launches",
            "clocks", "step", "shared_prefix_units", "unflushed", "non_kv_bytes_per_call", "partition_size")
    return {k: r[k] for k in keep if k in r}


def run_e2e(args, wl, pa, kp, vp, ws, P, max_ctx, dev, world, fused, share=False):
    """Same metric through the public API with host buffers: every step copies its
    inputs from pinned host memory and reads the output back. The copies run on
    a second stream into double buffers, so step i+1's inputs travel while step
    i decodes and step i's output comes back while step i+1 runs (the way a
    serving loop would pipeline them); all of it is inside the timed region."""
    nsteps = len(wl.steps)
    keys = ("q", "k", "v", "slots", "tables", "ctx", "pairs")

    def staged(st):
        """A step's inputs in one pinned host buffer (256-byte aligned parts),
        so that one copy per step moves them all."""
        parts = dict(q=st.q, k=st.k_new, v=st.v_new, slots=torch.from_numpy(st.slot_mapping),
                     tables=torch.from_numpy(st.block_tables), ctx=torch.from_numpy(st.context_lens),
                     pairs=torch.from_numpy(st.copy_pairs))
        layout, off = {}, 0
        for k in keys:
            t = parts[k].contiguous()
            layout[k] = (off, t.dtype, tuple(t.shape), t.numel() * t.element_size())
            off += (layout[k][3] + 255) // 256 * 256
        buf = torch.zeros(max(off, 256), dtype=torch.uint8).pin_memory()
        for k in keys:
            o, _, _, n = layout[k]
            if n:
                buf[o:o + n].copy_(parts[k].contiguous().reshape(-1).view(torch.uint8))
        return buf, layout

    def views(buf, layout):
        return {k: buf[o:o + n].view(dt).view(shape) if n else torch.empty(shape, dtype=dt, device=buf.device)
                for k, (o, dt, shape, n) in layout.items()}

    host = []
    for st in wl.steps:
        buf, layout = staged(st)
        host.append(dict(buf=buf, layout=layout, out=torch.empty_like(st.q).pin_memory()))
    B = int(len(wl.steps[0].context_lens))
    h0 = host[0]
    h2d = h0["buf"].numel()
    d2h = h0["out"].numel() * h0["out"].element_size()
    # Device copies of each step's staging buffer, two sets (double buffering),
    # with the inputs as views into it, and two outputs.
    dbuf = {}
    for j in range(nsteps):
        for b in (0, 1):
            raw = torch.empty_like(host[j]["buf"], device=dev)
            dbuf[(j, b)] = dict(raw=raw, **views(raw, host[j]["layout"]))
    outs = [torch.empty_like(h0["out"], device=dev) for _ in (0, 1)]
    stream = torch.cuda.current_stream(dev)
    cs = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in (0, 1)]     # inputs of the set have arrived
    ev_done = [torch.cuda.Event() for _ in (0, 1)]   # decode using the set has finished
    ev_back = [torch.cuda.Event() for _ in (0, 1)]   # output of the set is on the host
    for e in ev_done + ev_back:
        e.record(stream)

    def upload(i):
        b = i % 2
        d, h = dbuf[(i % nsteps, b)], host[i % nsteps]
        with torch.cuda.stream(cs):
            cs.wait_event(ev_done[b])  # the set's previous user has finished
            d["raw"].copy_(h["buf"], non_blocking=True)
            ev_in[b].record(cs)

    def download(i):
        b = i % 2
        with torch.cuda.stream(cs):
            cs.wait_event(ev_done[b])
            host[i % nsteps]["out"].copy_(outs[b], non_blocking=True)
            ev_back[b].record(cs)

    def compute(i):
        b = i % 2
        d = dbuf[(i % nsteps, b)]
        out = outs[b]
        stream.wait_event(ev_in[b])
        stream.wait_event(ev_back[b])  # the output buffer has been read back
        if d["pairs"].shape[0]:
            pa.pa_copy_blocks([kp, vp], d["pairs"])
        if share:
            kw = {}
            if fused:
                if d["slots"].shape[0] > B:
                    pa.pa_reshape_and_cache(d["k"][B:], d["v"][B:], kp, vp, d["slots"][B:])
                kw = dict(k_new=d["k"][:B], v_new=d["v"][:B])
            else:
                pa.pa_reshape_and_cache(d["k"], d["v"], kp, vp, d["slots"])
            pa.pa_decode_shared(out, d["q"], kp, vp, d["tables"], d["ctx"], wl.scale, max_ctx, P, ws, **kw)
        elif fused:
            if d["slots"].shape[0] > B:
                pa.pa_reshape_and_cache(d["k"][B:], d["v"][B:], kp, vp, d["slots"][B:])
            pa.pa_decode_append(out, d["q"], d["k"][:B], d["v"][:B], kp, vp, d["tables"], d["ctx"], wl.scale,
                                max_ctx, P, ws)
        else:
            pa.pa_reshape_and_cache(d["k"], d["v"], kp, vp, d["slots"])
            pa.pa_decode(out, d["q"], kp, vp, d["tables"], d["ctx"], wl.scale, max_ctx, P, ws)
        ev_done[b].record(stream)

    def run(n):
        upload(0)
        for i in range(n):
            if i + 1 < n:
                upload(i + 1)
            compute(i)
            download(i)
        stream.wait_stream(cs)

    run(args.warmup)
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    a.record(stream)
    cs.wait_event(a)
    run(args.steps)
    b.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    ms = max_over_ranks(a.elapsed_time(b) / args.steps, world)
    return {"value": B * world / (ms / 1e3), "unit": "seqs/s", "ms_per_step": ms,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "overlap": "inputs of step i+1 copied (one staging buffer, one copy) and step i's output read back "
                       "on a second stream while step i / i+1 decode (double buffers)"}


def bits_of(t: torch.Tensor) -> np.ndarray:
    """Raw 16-bit patterns of a CPU fp16/bf16 tensor (the oracle's input format)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# Sequences of the workload's first step that the oracle decodes per timed
# run, in the CPU baseline and in the reference arm alike.
ORACLE_SAMPLE_SEQS = 32


def oracle_sample(wl, n_seqs):
    """A bounded slice of the workload's first step for the oracle: n_seqs
    sequences with their tables, the pools as 16-bit patterns, and the
    algorithmic K+V bytes those sequences read."""
    st = wl.steps[0]
    ctx = st.context_lens[:n_seqs]
    kv = int(ctx.astype(np.int64).sum()) * wl.num_kv_heads * wl.head_dim * 2 * 2
    return dict(q=bits_of(st.q[:n_seqs]), kp=bits_of(wl.k_pool), vp=bits_of(wl.v_pool),
                tables=st.block_tables[:n_seqs], ctx=ctx,
                k=bits_of(st.k_new), v=bits_of(st.v_new), slots=st.slot_mapping, kv_bytes=kv)


def oracle_run(wl, s, kp, vp, threads):
    """One oracle step over the sample: the cache write, then fp64 attention."""
    import oracle
    oracle.reshape_and_cache(s["k"], s["v"], kp, vp, s["slots"])
    oracle.paged_attention(s["q"], kp, vp, s["tables"], s["ctx"], wl.scale, wl.dtype, threads)


def cpu_baseline(wl, repeats=3):
    """The oracle as it stands on this host's cores: the same sample timed on
    one core and on all of them, best of `repeats` wall-clock runs each."""
    import oracle
    B = int(len(wl.steps[0].context_lens))
    n = min(B, ORACLE_SAMPLE_SEQS)
    s = oracle_sample(wl, n)
    kp, vp = s["kp"].copy(), s["vp"].copy()
    cores = oracle.max_threads()
    best = {}
    for threads in (1, cores):
        t = []
        for _ in range(repeats):
            t0 = time.perf_counter()
            oracle_run(wl, s, kp, vp, threads)
            t.append(time.perf_counter() - t0)
        best[threads] = min(t)
    entry = lambda dt: {"seqs_per_s": n / dt, "kv_gbs": s["kv_bytes"] / dt / 1e9, "s_per_run": dt}
    return {"value": n / best[cores], "unit": "seqs/s", "cores": cores, "kind": "oracle",
            "kv_gbs": s["kv_bytes"] / best[cores] / 1e9,
            "cores_1": entry(best[1]), "cores_all": entry(best[cores]),
            "sample": f"{n} of {B} sequences of the first step (cache write + fp64 attention), "
                      f"best of {repeats} runs on 1 core and on all {cores}"}


def run_swap(args, world, rank, local):
    """pa_swap_blocks between the GPU pools and a page-locked host pool: a
    shuffled set of whole blocks out and back, against one contiguous
    cudaMemcpyAsync of the same bytes over the same link (the roofline)."""
    import paged_kv_cache_372_b200 as pa
    from paged_kv_cache_372_b200 import build, inputs
    build.build()
    dev = torch.device("cuda", local if world > 1 else 0)
    nb, hkv, bs, d = 8192, 8, 16, 128                      # llama3_8b-shaped blocks, 32 KiB per pool
    gen = inputs.generator(args.seed + 7000)
    kp = inputs.normal((nb, hkv, bs, d), "bf16", gen).to(dev)
    vp = inputs.normal((nb, hkv, bs, d), "bf16", gen).to(dev)
    hk = torch.empty((nb, hkv, bs, d), dtype=torch.bfloat16).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    n = nb // 2                                           # half the pool moves each way
    src = torch.tensor(inputs.choice(nb, n, gen), dtype=torch.int64)
    dst = torch.tensor(inputs.choice(nb, n, gen), dtype=torch.int64)
    out_pairs = torch.stack([src, dst], 1).to(dev)
    in_pairs = torch.stack([dst, src], 1).to(dev)
    moved = 2 * n * kp[0].numel() * 2
    stream = torch.cuda.current_stream(dev)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / args.steps

    ms_out = timed(lambda: pa.pa_swap_blocks([hk, hv], [kp, vp], out_pairs))
    ms_in = timed(lambda: pa.pa_swap_blocks([kp, vp], [hk, hv], in_pairs))
    assert pa.pa_device_errors() == 0
    flat_d = torch.empty(moved, dtype=torch.uint8, device=dev)
    flat_h = torch.empty(moved, dtype=torch.uint8).pin_memory()
    ms_d2h = timed(lambda: flat_h.copy_(flat_d, non_blocking=True))
    ms_h2d = timed(lambda: flat_d.copy_(flat_h, non_blocking=True))
    gbs = lambda ms: moved / (ms * 1e-3) / 1e9
    value = 2 * moved / ((ms_out + ms_in) * 1e-3) / 1e9
    link = 2 * moved / ((ms_d2h + ms_h2d) * 1e-3) / 1e9
    return {"metric": "block swap GPU<->page-locked host (pa_swap_blocks), GB/s", "value": value, "unit": "GB/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_out + ms_in,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": {"workload": "swap", "blocks_each_way": n, "block_bytes_per_pool":
                                            kp[0].numel() * 2, "pools": 2, "bytes_each_way": moved},
            "swap_out_gbs": gbs(ms_out), "swap_in_gbs": gbs(ms_in),
            "roofline": {"bound": "host link", "achieved": value, "peak": link, "unit": "GB/s",
                         "frac": value / link,
                         "peak_source": "measured: one contiguous cudaMemcpyAsync of the same bytes each way",
                         "memcpy_d2h_gbs": gbs(ms_d2h), "memcpy_h2d_gbs": gbs(ms_h2d)},
            "gpu_launches": 2 * args.steps}


def run_reference(args, world, rank):
    """The oracle, as it stands, on all host cores: each step is the same
    bounded sample of the workload that the CPU baseline times."""
    import oracle
    from paged_kv_cache_372_b200 import workloads
    wl = workloads.build(args.workload, args.seed, **shape_args(args))
    B = int(len(wl.steps[0].context_lens))
    n = min(B, ORACLE_SAMPLE_SEQS)
    s = oracle_sample(wl, n)
    kp, vp = s["kp"].copy(), s["vp"].copy()
    cores = oracle.max_threads()
    for _ in range(args.warmup):
        oracle_run(wl, s, kp, vp, cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_run(wl, s, kp, vp, cores)
    dt = (time.perf_counter() - t0) / args.steps
    value = n / dt
    sample = f"{n} of {B} sequences of the first step per step (cache write + fp64 attention), all {cores} cores"
    return {"metric": METRIC, "value": value, "unit": "seqs/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": describe(wl),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "seqs/s", "cores": cores, "kind": "oracle",
                             "kv_gbs": s["kv_bytes"] / dt / 1e9, "sample": sample},
            "e2e": {"value": value, "unit": "seqs/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            if rank == 0:
                print(json.dumps(run_reference(args, world, rank)), flush=True)
            return
        res = run_swap(args, world, rank, local) if args.workload == "swap" else run_ours(args, world, rank, local)
        if (args.workload in SECONDARY and world == 1 and args.kv == "auto" and args.partition is None
                and not shape_args(args)):
            res["secondary_workloads"] = {name: run_secondary(args, world, rank, local, name)
                                          for name in SECONDARY[args.workload]}
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
