#!/usr/bin/env python
"""Benchmark of one paged decode step on B200: reshape_and_cache of each sequence's new token, then
paged attention over the whole batch, on the 7B-shape decode workload (64 sequences, context lengths
uniform in [512, 2048], 32 query / 32 kv heads, head size 128, block size 16, bf16, blocks shuffled
across a 16384-block pool).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]

Prints one JSON line (rank 0). `value` is the achieved KV-read bandwidth: the ideal bytes of every
valid token's K and V row read once, divided by the device time of a step, summed over ranks and
divided by the slowest rank's time. Multi-GPU runs shard independent sequences (one batch per rank,
no collective on the data path; weak scaling). `--impl reference` times the CPU oracle instead.
"""
import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "paged decode attention: achieved KV-read HBM GB/s & % of peak; tokens/s"
KERNEL_SOURCES = ("pa_attention.cuh", "pa_device.cuh", "pa_launch.cuh")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "paged_attention_main_traffic.json")
THROTTLE_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
                 0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
                 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


def bits16(t):
    """Raw uint16 bits of a CPU fp16/bf16 tensor (how the oracle takes 16-bit arrays)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def measured_peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except OSError:
        return None


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "pagedattention_paged_kv_attention_b200", "csrc")
    for name in KERNEL_SOURCES:
        h.update(open(os.path.join(csrc, name), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """DRAM bytes per launch of the attention kernel from the committed ncu summary, if it was taken
    on the current kernel source and this workload; else None."""
    try:
        rec = json.load(open(TRAFFIC_FILE))
    except (OSError, ValueError):
        return None
    rec = rec.get(workload)
    if not rec or rec.get("kernel_source_hash") != kernel_source_hash():
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms while the timed region runs."""

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    def summary(self):
        sm, mx, reasons = [], [], set()
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 3:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
                bits = int(parts[2], 16)
            except ValueError:
                continue
            for b, name in THROTTLE_BITS.items():
                if bits & b and name != "gpu_idle":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_selector(dev):
    """nvidia-smi -i argument for the physical GPU behind a CUDA device (its UUID when known)."""
    props = torch.cuda.get_device_properties(dev)
    uuid = getattr(props, "uuid", None)
    if uuid is not None:
        u = str(uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    return str(dev.index)


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl != "reference":
        torch.cuda.set_device(local)  # before NCCL comes up, so each rank's collectives use its own GPU
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl" if args.impl != "reference" else "gloo",
                                             timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def reduce_max(x, world, device):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(x, world, device):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def run_reference(args, cfg, world, rank):
    """The CPU oracle timed on the machine's host cores (rank 0 only): --warmup untimed passes, then
    --steps timed passes over the same deterministic sample as the GPU arm's cpu_baseline leg."""
    if rank != 0:
        return
    rec = oracle_decode_timing(cfg, passes=args.steps, warmup=args.warmup)
    lens = decode_lengths(cfg, cfg.seed)
    line = {"metric": METRIC, "value": rec["value"], "unit": "GB/s", "impl": "reference", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(rec["pass_s"]["median"] * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": decode_config(cfg, lens, world),
            "tokens_per_s": rec["tokens_per_s"],
            "cpu_baseline": rec,
            "e2e": {"value": rec["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--op", default="decode", choices=["decode", "prefill", "swap", "layers", "plan", "trace"],
                    help="decode: the decode step (default); prefill: the causal prefill step; swap: swap_blocks "
                         "host<->device; layers: multi-layer cache ops; plan: the block manager's decode plan; "
                         "trace: per-CTA and per-item timing of the decode kernel (trace build)")
    ap.add_argument("--workload", default=None, choices=list(W.CONFIGS) + list(W.PREFILL_CONFIGS),
                    help="default: 7b (decode ops), prefill_7b (--op prefill)")
    ap.add_argument("--partition-size", type=int, default=None,
                    help="tokens per split-K partition (default: the workload's, else the library's choice)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--num-seqs", type=int, default=None,
                    help="smaller batch of the same workload (profiling cases); default: the workload's")
    ap.add_argument("--pool-blocks", type=int, default=None,
                    help="override the pool size in blocks (profiling cases that must stay small)")
    ap.add_argument("--cpu-seconds", type=float, default=8.0)
    ap.add_argument("--trace-out", default=None, help="trace op: also save the raw records of the last launch (.npz)")
    ap.add_argument("--no-extra-configs", action="store_true",
                    help="time only --workload (by default the 7B line also carries a 70B-GQA sub-record)")
    args = ap.parse_args()
    assert args.warmup >= 3, "at least 3 warm-up steps"
    if args.workload is None:
        args.workload = "prefill_7b" if args.op == "prefill" else "7b"
    if args.op == "prefill":
        world, rank, local = dist_setup(args)
        run_prefill(args, W.PREFILL_CONFIGS[args.workload], world, rank)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    cfg = W.CONFIGS[args.workload]
    if args.pool_blocks is not None:
        import dataclasses
        cfg = dataclasses.replace(cfg, num_blocks=args.pool_blocks)
    world, rank, local = dist_setup(args)

    if args.op in ("swap", "layers", "plan", "trace"):
        if rank == 0:
            {"swap": run_swap, "layers": run_layers, "plan": run_plan, "trace": run_trace}[args.op](args, cfg)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    if args.impl == "reference":
        run_reference(args, cfg, world, rank)
        if world > 1:
            torch.distributed.destroy_process_group()
        return

    from pagedattention_paged_kv_attention_b200 import pagedattn as P

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks = measured_peaks()
    peak = peaks["hbm_gbs"] if peaks else 6650.0
    rec = measure_decode(args, cfg, P, dev, rank, world, peak, peaks is not None, checks=True)
    extra = {}
    if (args.workload == "7b" and not args.no_extra_configs and args.num_seqs is None and args.pool_blocks is None
            and args.partition_size is None):
        # The second configuration the bandwidth target names, in the same run and process.
        extra["70b_gqa"] = measure_decode(args, W.CONFIGS["70b_gqa"], P, dev, rank, world, peak, peaks is not None,
                                          checks=False)
    if rank == 0:
        line = {
            "metric": METRIC, "value": rec["value"], "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": rec["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if cfg.dtype == "bf16" else "f16",
            "data": "synthetic",
            "config": decode_config(cfg, decode_lengths(cfg, cfg.seed)[:args.num_seqs or cfg.num_seqs], world),
        }
        line.update({k: v for k, v in rec.items() if k not in ("value", "ms_per_step")})
        if extra:
            line["configs"] = {name: {k: v for k, v in r.items() if k not in ("gpu_launches",)}
                               for name, r in extra.items()}
            for name, r in extra.items():
                line["configs"][name]["config"] = decode_config(W.CONFIGS[name], decode_lengths(W.CONFIGS[name],
                                                                W.CONFIGS[name].seed), world)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = oracle_decode_timing(cfg, seconds=args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def timed_launches(fn, reps=10, warmup=3):
    """Median CUDA-event time (ms) of one call of fn on the current stream."""
    for _ in range(warmup):
        fn()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    torch.cuda.synchronize()
    for a, b in evs:
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    return float(np.median([a.elapsed_time(b) for a, b in evs]))


def read_ceilings(P, dev, key_cache, value_cache, block_tables, context_lens, kv_bytes):
    """Read-only ceilings measured in this process (include/pa_probe.h): a sequential stream over 2 GiB
    (HBM), the same 16-byte loads over the batch's own K/V rows through its block table (no compute),
    and a 32 MiB buffer read 64 times over (L2)."""
    sink = torch.zeros(1, dtype=torch.int64, device=dev)
    big = torch.empty(2 << 30, dtype=torch.uint8, device=dev)
    t_stream = timed_launches(lambda: P.probe_stream_read(big, 1, sink))
    del big
    small = torch.empty(32 << 20, dtype=torch.uint8, device=dev)
    t_l2 = timed_launches(lambda: P.probe_stream_read(small, 64, sink))
    del small
    t_paged = timed_launches(lambda: P.probe_paged_read(key_cache, value_cache, block_tables, context_lens, sink))
    return {"hbm_read_stream_gbs": round((2 << 30) / (t_stream * 1e-3) / 1e9, 1),
            "paged_read_gbs": round(kv_bytes / (t_paged * 1e-3) / 1e9, 1),
            "l2_read_gbs": round(64 * (32 << 20) / (t_l2 * 1e-3) / 1e9, 1),
            "method": "pa_probe_stream_read over 2 GiB once (HBM) and over 32 MiB 64 times (L2); "
                      "pa_probe_paged_read over this batch's valid K/V rows; median of 10 event-timed launches"}


def measure_decode(args, cfg, P, dev, rank, world, peak, peak_measured, checks):
    """One workload's decode step timed on the device (K steps after W warm-ups, back to back), through
    the public API end to end, and with its roofline; with checks, also the read ceilings and an L2-flush
    check of the attention call."""
    w = W.make_workload(cfg, seed=cfg.seed + 1000 * rank, device=dev, num_seqs=args.num_seqs)
    S, H, d = w.query.shape
    kv_bytes = 1 if cfg.kv_dtype.startswith("fp8") else 2
    ks = vs = None
    key_cache, value_cache = w.key_values, w.value_values
    if cfg.kv_dtype.startswith("fp8"):
        # The product's own quantiser fills the FP8 pools from the drawn values.
        NB, bs, Hkv, _ = key_cache.shape
        ks, vs = w.k_scale.to(dev), w.v_scale.to(dev)
        kq = torch.empty((NB, bs, Hkv, d), dtype=torch.uint8, device=dev)
        vq = torch.empty_like(kq)
        slots = torch.arange(NB * bs, dtype=torch.int64, device=dev)
        P.reshape_and_cache(key_cache.view(NB * bs, Hkv, d), value_cache.view(NB * bs, Hkv, d), kq, vq, slots, ks, vs)
        key_cache, value_cache = kq, vq
        del slots
        w.key_values = w.value_values = None
    lens = w.context_lens.cpu().numpy()
    mcl = int(lens.max())
    ideal = W.ideal_bytes(lens, cfg.num_kv_heads, d, kv_bytes, cfg.block_size, H, 2)
    part_req = args.partition_size if args.partition_size is not None else cfg.partition_size
    ps = P.partition_size(S, H, cfg.num_kv_heads, mcl, part_req)
    parts = max(1, -(-mcl // ps))
    ws = P.make_workspace(S, H, cfg.num_kv_heads, d, mcl, part_req, device=dev)
    out = torch.empty_like(w.query)
    stream = torch.cuda.current_stream(dev)

    def step(q, nk, nv, slots, tables, clens, o, ev=None):
        if w.cow_mapping.shape[0]:      # copy-on-write first, so a copied block then takes its new token
            P.copy_blocks(key_cache, value_cache, w.cow_mapping)
        P.reshape_and_cache(nk, nv, key_cache, value_cache, slots, ks, vs)
        if ev is not None:
            ev[0].record(stream)
        P.paged_attention(o, q, key_cache, value_cache, tables, clens, cfg.softmax_scale, mcl, ws, ks, vs,
                          partition_size=part_req)
        if ev is not None:
            ev[1].record(stream)

    inputs = (w.query, w.new_key, w.new_value, w.slot_mapping, w.block_tables, w.context_lens)
    launches_per_step = 2 + (1 if parts > 1 else 0) + (1 if w.cow_mapping.shape[0] else 0)

    # ---- device-resident timing: K steps back to back (the K/V read per step is larger than L2) ----
    for _ in range(args.warmup):
        step(*inputs, out)
    kernel_events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                     for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(gpu_selector(dev)) as clocks:
        start.record(stream)
        for i in range(args.steps):
            step(*inputs, out, kernel_events[i])
        stop.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    step_ms = start.elapsed_time(stop) / args.steps
    attn_ms = float(np.mean([a.elapsed_time(b) for a, b in kernel_events]))
    assert P.get_device_error(ws) == 0, "device error word set"
    max_step_ms = reduce_max(step_ms, world, dev)
    total_kv = reduce_sum(float(ideal["kv"]), world, dev)
    total_seqs = reduce_sum(float(S), world, dev)
    total_ctx = reduce_sum(float(np.sum(lens)), world, dev)
    value = total_kv / (max_step_ms * 1e-3) / 1e9

    # ---- end to end through the API: pinned host inputs in, output back to pinned host ----
    # Each step uploads its inputs as ONE copy of a packed pinned buffer (every tensor at a 256-byte
    # aligned offset) and reads its output back. Two device input slots: step i+1's upload (copy stream)
    # overlaps step i's kernels; the read-back runs on a third stream. Every copy is inside the timed
    # region, which ends after the last read-back.
    offs, total = [], 0
    for t in inputs:
        offs.append(total)
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    host_packed = torch.empty(total, dtype=torch.uint8).pin_memory()
    for t, o in zip(inputs, offs):
        nb = t.numel() * t.element_size()
        host_packed[o:o + nb].copy_(t.contiguous().view(-1).view(torch.uint8).cpu())
    dev_packed = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(2)]
    views = [[dp[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape) for t, o in zip(inputs, offs)]
             for dp in dev_packed]
    outs = [torch.empty_like(out) for _ in range(2)]
    host_out = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in inputs)
    d2h = host_out[0].numel() * host_out[0].element_size()
    copy_stream, back_stream = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]      # inputs of the slot uploaded
    ev_run = [torch.cuda.Event() for _ in range(2)]     # kernels of the slot done
    ev_back = [torch.cuda.Event() for _ in range(2)]    # output of the slot read back

    def e2e_step(i):
        slot = i % 2
        copy_stream.wait_event(ev_run[slot])            # the slot's previous kernels have read it
        with torch.cuda.stream(copy_stream):
            dev_packed[slot].copy_(host_packed, non_blocking=True)
        ev_in[slot].record(copy_stream)
        stream.wait_event(ev_in[slot])
        stream.wait_event(ev_back[slot])                # the slot's previous output has been read
        step(*views[slot], outs[slot])
        ev_run[slot].record(stream)
        back_stream.wait_event(ev_run[slot])
        with torch.cuda.stream(back_stream):
            host_out[slot].copy_(outs[slot], non_blocking=True)
        ev_back[slot].record(back_stream)

    for i in range(args.warmup):
        e2e_step(i)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    copy_stream.wait_event(e0)
    for i in range(args.steps):
        e2e_step(i)
    stream.wait_event(ev_back[(args.steps - 1) % 2])
    stream.wait_event(ev_back[args.steps % 2])
    e1.record(stream)
    torch.cuda.synchronize()
    assert torch.equal(host_out[(args.steps - 1) % 2], outs[(args.steps - 1) % 2].cpu()), "read-back mismatch"
    e2e_ms = reduce_max(e0.elapsed_time(e1) / args.steps, world, dev)
    e2e_value = total_kv / (e2e_ms * 1e-3) / 1e9

    achieved = ideal["total"] / (attn_ms * 1e-3) / 1e9
    rec = {
        "value": round(value, 2), "ms_per_step": round(max_step_ms, 4),
        "plan": {"partition_size": ps, "partitions": parts, "num_seqs": S},
        "tokens_per_s": round(total_seqs / (max_step_ms * 1e-3), 1),
        "context_tokens_per_s": round(total_ctx / (max_step_ms * 1e-3), 1),
        "pct_of_measured_hbm_peak": round(100 * value / peak, 2),
        "pct_of_8tbs": round(100 * value / 8000.0, 2),
        "roofline": {"kernel": "paged_attention (pa_paged_attention call: main kernel%s)" %
                     (" + split-K reduce" if parts > 1 else ""),
                     "bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_source": "measured" if peak_measured else "fallback",
                     "algorithmic_bytes_per_launch": ideal["total"], "avg_launch_ms": round(attn_ms, 4),
                     "traffic": recorded_traffic(cfg.name)},
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
                "copies": "one packed pinned upload per step (overlapping the previous step's kernels) "
                          "and the output read back on its own stream, all inside the timed region"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks.summary(),
    }
    del dev_packed, views, outs, host_out, host_packed
    if rank == 0:
        # Read ceilings in this process, and the attention call's fraction of each.
        ceil = read_ceilings(P, dev, key_cache, value_cache, w.block_tables, w.context_lens, ideal["kv"])
        rec["ceilings"] = ceil
        rec["roofline"]["frac_of_read_stream"] = round(achieved / ceil["hbm_read_stream_gbs"], 4)
        rec["roofline"]["frac_of_paged_read"] = round(achieved / ceil["paged_read_gbs"], 4)
        if cfg.shared_prefix_tokens:
            # Every sequence reads the shared prefix blocks: most logical bytes come from L2 (the unique
            # bytes are a fifth of them), so the bound for the logical bytes is the L2 read ceiling.
            rec["roofline"].update({"bound": "l2", "peak": ceil["l2_read_gbs"],
                                    "frac": round(achieved / ceil["l2_read_gbs"], 4),
                                    "peak_source": "measured in this run (pa_probe_stream_read, 32 MiB read 64 times)",
                                    "frac_of_measured_hbm_copy": round(achieved / peak, 4)})
        if checks:
            # L2 flush check: the same attention call with L2 flushed (a write of twice the L2 size)
            # before each step, per-step event timing; against the back-to-back figure above.
            l2 = torch.cuda.get_device_properties(dev).L2_cache_size
            flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            for i in range(args.steps):
                flush.fill_(i & 0xFF)
                step(*inputs, out, evs[i])
            torch.cuda.synchronize()
            flushed_ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
            rec["l2_flush_check"] = {"flush_bytes": 2 * l2, "attn_ms_flushed": round(flushed_ms, 4),
                                     "attn_ms_back_to_back": round(attn_ms, 4),
                                     "back_to_back_over_flushed": round(flushed_ms / attn_ms, 4)}
            del flush
    del key_cache, value_cache, w
    torch.cuda.empty_cache()
    return rec


def run_prefill(args, cfg, world, rank):
    """The prefill step: reshape_and_cache of every chunk's keys and values, then causal paged prefill
    attention. value = causal attention FLOPs (4 * d per visible (query head, key) pair) / device step
    time; each rank runs its own batch (weak scaling). The roofline is the attention call's FLOPs over
    its event-timed duration against the measured dense bf16 tensor peak."""
    if args.impl == "reference":
        return run_prefill_reference(args, cfg, world, rank)
    from pagedattention_paged_kv_attention_b200 import pagedattn as P
    dev = torch.device("cuda", torch.cuda.current_device())
    w = W.make_prefill_workload(cfg, seed=cfg.seed + 1000 * rank, device=dev, num_seqs=args.num_seqs)
    H, d = cfg.num_heads, cfg.head_size
    flops = 4.0 * d * H * w.causal_pairs()
    key_cache, value_cache = w.key_values, w.value_values
    ks = vs = None
    if cfg.cache_dtype.startswith("fp8"):
        # The product's own quantiser fills the FP8 pools from the drawn values.
        NB, bs, Hkv, _ = key_cache.shape
        ks, vs = w.k_scale.to(dev), w.v_scale.to(dev)
        kq = torch.empty((NB, bs, Hkv, d), dtype=torch.uint8, device=dev)
        vq = torch.empty_like(kq)
        slots = torch.arange(NB * bs, dtype=torch.int64, device=dev)
        P.reshape_and_cache(key_cache.view(NB * bs, Hkv, d), value_cache.view(NB * bs, Hkv, d), kq, vq, slots, ks, vs)
        key_cache, value_cache = kq, vq
        del slots
    out = torch.empty_like(w.query)
    ws = torch.zeros(64, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    mq = w.max_q_len

    def step(q, nk, nv, slots, tables, lens, qs, o, ev=None):
        P.reshape_and_cache(nk, nv, key_cache, value_cache, slots, ks, vs)
        if ev is not None:
            ev[0].record(stream)
        P.paged_prefill(o, q, key_cache, value_cache, tables, lens, qs, cfg.softmax_scale, mq, ws, ks, vs)
        if ev is not None:
            ev[1].record(stream)

    inputs = (w.query, w.new_key, w.new_value, w.slot_mapping, w.block_tables, w.context_lens, w.q_start)
    for _ in range(args.warmup):
        step(*inputs, out)
    events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(gpu_selector(dev)) as clocks:
        start.record(stream)
        for i in range(args.steps):
            step(*inputs, out, events[i])
        stop.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    step_ms = start.elapsed_time(stop) / args.steps
    attn_ms = float(np.mean([a.elapsed_time(b) for a, b in events]))
    assert P.get_device_error(ws) == 0, "device error word set"
    max_ms = reduce_max(step_ms, world, dev)
    total_flops = reduce_sum(flops, world, dev)
    value = total_flops / (max_ms * 1e-3) / 1e12

    # end to end: pinned host inputs in, output back to pinned host memory
    host_in = [t.cpu().pin_memory() for t in inputs]
    dev_in = [torch.empty_like(t) for t in inputs]
    host_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = host_out.numel() * host_out.element_size()

    def e2e_step():
        for dst, src in zip(dev_in, host_in):
            dst.copy_(src, non_blocking=True)
        step(*dev_in, out)
        host_out.copy_(out, non_blocking=True)

    for _ in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    a1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(a0.elapsed_time(a1) / args.steps, world, dev)
    e2e_value = total_flops / (e2e_ms * 1e-3) / 1e12

    if rank != 0:
        return
    peaks = measured_peaks()
    peak = peaks.get("bf16_tflops") if peaks else 1590.0
    achieved = flops / (attn_ms * 1e-3) / 1e12
    T = w.query.shape[0]
    line = {"metric": "paged prefill attention: causal TFLOP/s", "value": round(value, 2), "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(max_ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": cfg.dtype if not cfg.cache_dtype.startswith("fp8") else "f16",
            "data": "synthetic",
            "config": {"workload": cfg.description, "name": cfg.name, "num_seqs": cfg.num_seqs, "query_tokens": T,
                       "causal_pairs_per_head": w.causal_pairs(), "num_heads": H, "num_kv_heads": cfg.num_kv_heads,
                       "head_size": d, "block_size": cfg.block_size, "kv_dtype": cfg.cache_dtype,
                       "l2": f"inputs larger than L2: {(w.query.numel() * 2 * 2 + key_cache.numel() * 4) / 1e9:.2f} GB "
                             "of query, output and K/V per step vs 126 MB L2",
                       "parallelism": f"dp{world} (independent batches)"},
            "tokens_per_s": round(reduce_sum(float(T), world, dev) / (max_ms * 1e-3), 1),
            "roofline": {"kernel": "paged_prefill_kernel (pa_paged_prefill call)", "bound": "tensor",
                         "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(achieved / peak, 4),
                         "peak_source": "measured bf16 burst" if peaks else "fallback",
                         "flops_per_launch": flops, "avg_launch_ms": round(attn_ms, 4), "traffic": None},
            "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4)},
            "gpu_launches": 2 * args.steps, "clocks": clocks.summary()}
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = prefill_cpu_baseline(cfg, args.cpu_seconds)
    print(json.dumps(line), flush=True)


def _prefill_sample(cfg, rows_wanted):
    """Sampled query rows of the prefill workload as one-token chunks over truncated contexts (the
    oracle's cost per row is its prefix length), with their FLOPs."""
    import dataclasses
    w = W.make_prefill_workload(cfg, num_seqs=min(cfg.num_seqs, 2))
    rng = np.random.default_rng(cfg.seed)
    q_start = w.q_start.numpy()
    lens = w.context_lens.numpy()
    rows = np.sort(rng.choice(w.query.shape[0], size=min(rows_wanted, w.query.shape[0]), replace=False))
    seq = np.searchsorted(q_start, rows, side="right") - 1
    n = q_start[seq + 1] - q_start[seq]
    pos = lens[seq] - n + (rows - q_start[seq])
    kc, vc = bits16(w.key_values), bits16(w.value_values)
    import oracle
    kd = cfg.cache_dtype
    ks = vs = None
    if kd.startswith("fp8"):   # the oracle's own quantiser fills its FP8 pools
        ks, vs = w.k_scale.numpy(), w.v_scale.numpy()
        quant = oracle.quantize_e4m3 if kd == "fp8_e4m3" else oracle.quantize_e4m3_blocks
        kc, vc = quant(kc, cfg.dtype, ks), quant(vc, cfg.dtype, vs)
    oracle.reshape_and_cache(bits16(w.new_key), bits16(w.new_value), cfg.dtype, kc, vc, kd, w.slot_mapping.numpy(),
                             ks, vs)
    inp = dict(query_bits=bits16(w.query)[rows], q_dtype=cfg.dtype, key_cache=kc, value_cache=vc,
               kv_dtype=kd, block_tables=w.block_tables.numpy()[seq], context_lens=(pos + 1).astype(np.int32),
               q_start=np.arange(len(rows) + 1, dtype=np.int32), scale=cfg.softmax_scale, k_scale=ks, v_scale=vs)
    flops = 4.0 * cfg.head_size * cfg.num_heads * float((pos + 1).sum())
    return inp, flops, len(rows)


def prefill_cpu_baseline(cfg, seconds):
    import oracle
    rows = 4
    while True:
        inp, flops, n = _prefill_sample(cfg, rows)
        t0 = time.perf_counter()
        oracle.paged_prefill(**inp)
        dt = time.perf_counter() - t0
        if dt >= seconds / 3 or rows >= 4096:
            break
        rows = min(4096, max(rows * 2, int(rows * seconds / 3 / max(dt, 1e-3))))
    reps, total = 0, 0.0
    while total < seconds * 2 / 3 or reps == 0:
        t0 = time.perf_counter()
        oracle.paged_prefill(**inp)
        total += time.perf_counter() - t0
        reps += 1
    t = total / reps
    return {"value": round(flops / t / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.default_threads(),
            "kind": "oracle", "sample": f"{n} random query rows of the workload's first sequences, each over its "
                                        f"whole prefix, {reps} timed passes of {t:.2f} s, fp64"}


def run_prefill_reference(args, cfg, world, rank):
    """The oracle's prefill on a bounded sample, timed on the host cores (rank 0 only)."""
    if rank != 0:
        return
    import oracle
    rows = 4
    while True:
        inp, flops, n = _prefill_sample(cfg, rows)
        t0 = time.perf_counter()
        oracle.paged_prefill(**inp)
        dt = time.perf_counter() - t0
        if dt >= 0.5 or rows >= 4096:
            break
        rows = min(4096, max(rows * 2, int(rows * 1.0 / max(dt, 1e-3))))
    for _ in range(args.warmup):
        oracle.paged_prefill(**inp)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.paged_prefill(**inp)
        times.append(time.perf_counter() - t0)
    t = float(np.mean(times))
    value = flops / t / 1e12
    sample = f"{n} random query rows of the workload, each over its whole prefix, fp64 oracle"
    line = {"metric": "paged prefill attention: causal TFLOP/s", "value": round(value, 6), "unit": "TFLOP/s",
            "impl": "reference", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(t * 1e3, 3), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "config": {"workload": cfg.description, "name": cfg.name},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.default_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


TRACE_CTA_BASE, TRACE_MAX_CTAS = 8, 1024   # word offsets of the trace build's records (pa_attention.cuh)


def run_trace(args, cfg):
    """Where the decode kernel's time goes at the end of a launch. Builds the PA_TRACE variant of the
    library (same kernels; they also stamp %globaltimer into the workspace), runs the workload's decode
    step, and summarises one launch: per-CTA start/end, per-item start/finish, the split-K reduce's
    span; idle SM time after each CTA's last item, and in the last 10% of the launch."""
    from pagedattention_paged_kv_attention_b200 import build as B
    lib = B.build(defines=["PA_TRACE"], output=os.path.join(os.path.dirname(B.LIBRARY), "libpagedattn_trace.so"))
    os.environ["PA_LIBRARY_PATH"] = lib
    from pagedattention_paged_kv_attention_b200 import pagedattn as P
    dev = torch.device("cuda", torch.cuda.current_device())
    w = W.make_workload(cfg, seed=cfg.seed, device=dev, num_seqs=args.num_seqs)
    assert not cfg.kv_dtype.startswith("fp8"), "trace op: 16-bit caches"
    S, H, d = w.query.shape
    lens = w.context_lens.cpu().numpy()
    mcl = int(lens.max())
    part_req = args.partition_size if args.partition_size is not None else cfg.partition_size
    ps = P.partition_size(S, H, cfg.num_kv_heads, mcl, part_req)
    parts = max(1, -(-mcl // ps))
    ws = P.make_workspace(S, H, cfg.num_kv_heads, d, mcl, part_req, device=dev)
    nbytes = ws.numel() * ws.element_size()
    g_tile = 1
    while g_tile < H // cfg.num_kv_heads and g_tile < 8:
        g_tile *= 2
    items = parts * S * (-(-cfg.num_kv_heads // 8)) * (-(-(H // cfg.num_kv_heads) // g_tile))
    trace_words = 8 + 4 * TRACE_MAX_CTAS + 4 * items
    trace = ws.view(torch.uint8)[nbytes - ((trace_words * 8 + 255) // 256 * 256):].view(torch.int64)
    out = torch.empty_like(w.query)
    summaries = []
    for rep in range(args.warmup + args.steps):
        trace.zero_()
        P.reshape_and_cache(w.new_key, w.new_value, w.key_values, w.value_values, w.slot_mapping)
        P.paged_attention(out, w.query, w.key_values, w.value_values, w.block_tables, w.context_lens,
                          cfg.softmax_scale, mcl, ws, partition_size=part_req)
        torch.cuda.synchronize()
        if rep < args.warmup:
            continue
        t = trace.cpu().numpy().view(np.uint64).astype(np.float64)
        cta = t[TRACE_CTA_BASE:TRACE_CTA_BASE + 4 * TRACE_MAX_CTAS].reshape(-1, 4)
        cta = cta[cta[:, 0] > 0]
        it = t[TRACE_CTA_BASE + 4 * TRACE_MAX_CTAS:].reshape(-1, 4)[:items]
        it = it[it[:, 0] > 0]
        t0, t_end = cta[:, 0].min(), cta[:, 1].max()
        span = t_end - t0
        if args.trace_out:
            np.savez(args.trace_out, cta=cta, items=it, lens=lens, partition_size=ps, header=t[:8])
        ends = cta[:, 1]
        win = t_end - 0.1 * span
        busy_last10 = np.clip(ends - win, 0, None).sum() / (len(cta) * 0.1 * span)
        red_start = (2 ** 64 - 1) - t[0] if parts > 1 and t[0] > 0 else None
        summaries.append({
            "span_us": span / 1e3, "ctas": int(len(cta)), "items": int(len(it)),
            "cta_start_spread_us": (cta[:, 0].max() - t0) / 1e3,
            "cta_end_before_last_us": {q: float(np.percentile(t_end - ends, q)) / 1e3 for q in (10, 50, 90, 100)},
            "idle_after_last_item_frac": float((t_end - ends).sum() / (len(cta) * span)),
            "idle_in_last_10pct_frac": float(1 - busy_last10),
            "last_item_start_before_end_us": float((t_end - it[:, 0].max()) / 1e3),
            "item_us": {q: float(np.percentile(it[:, 1] - it[:, 0], q)) / 1e3 for q in (10, 50, 90, 100)},
            "item_tokens": {q: float(np.percentile(it[:, 3], q)) for q in (10, 50, 90, 100)},
            "reduce_start_after_main_end_us": None if red_start is None else float((red_start - t_end) / 1e3),
            "reduce_span_us": None if red_start is None else float((t[1] - red_start) / 1e3),
        })
    med = lambda key: float(np.median([x[key] for x in summaries]))
    line = {"metric": "decode kernel timeline (trace build)", "impl": "ours", "unit": "us", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "value": round(med("span_us"), 2),
            "config": {"workload": cfg.description, "name": cfg.name, "num_seqs": S, "partition_size": ps,
                       "partitions": parts, "items": items},
            "median": {k: round(med(k), 4) for k in ("span_us", "idle_after_last_item_frac",
                                                     "idle_in_last_10pct_frac", "last_item_start_before_end_us")},
            "launches": summaries}
    print(json.dumps(line), flush=True)


def run_swap(args, cfg, num_blocks=1024):
    """swap_blocks throughput: num_blocks random blocks of the workload's pool out to a pinned host pool
    and back in, each direction one launch, CUDA-event timed; beside it a plain copy of the same bytes
    between pinned host memory and the device (the link's ceiling for contiguous transfers)."""
    from pagedattention_paged_kv_attention_b200 import pagedattn as P
    dev = torch.device("cuda", torch.cuda.current_device())
    kv = torch.bfloat16 if cfg.kv_dtype == "bf16" else (torch.float16 if cfg.kv_dtype == "f16" else torch.uint8)
    shape = (cfg.num_blocks or 4096, cfg.block_size, cfg.num_kv_heads, cfg.head_size)
    dk = torch.randn(shape, device=dev).to(kv) if kv != torch.uint8 else torch.randint(0, 120, shape, device=dev, dtype=kv)
    dv = dk.clone()
    hk = torch.empty((num_blocks,) + shape[1:], dtype=kv).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    g = torch.Generator().manual_seed(cfg.seed)
    src = torch.randperm(shape[0], generator=g)[:num_blocks]
    out_map = torch.stack([src, torch.arange(num_blocks)], 1).to(dev)
    in_map = torch.stack([torch.arange(num_blocks), torch.randperm(shape[0], generator=g)[:num_blocks]], 1).to(dev)
    nbytes = 2 * hk.numel() * hk.element_size()

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.steps):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / args.steps

    t_out = timed(lambda: P.swap_blocks(hk, hv, dk, dv, out_map))
    t_in = timed(lambda: P.swap_blocks(dk, dv, hk, hv, in_map))
    flat_d = torch.empty(hk.numel() * 2, dtype=kv, device=dev)
    flat_h = torch.empty(hk.numel() * 2, dtype=kv).pin_memory()
    t_d2h = timed(lambda: flat_h.copy_(flat_d, non_blocking=True))
    t_h2d = timed(lambda: flat_d.copy_(flat_h, non_blocking=True))
    gbs = lambda ms: round(nbytes / (ms * 1e-3) / 1e9, 2)
    line = {"metric": "swap_blocks host<->device GB/s", "value": gbs((t_out + t_in) / 2), "unit": "GB/s",
            "impl": "ours", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
            "dtype": cfg.kv_dtype, "data": "synthetic",
            "config": {"workload": f"{num_blocks} random blocks of the {cfg.name} pool shape {list(shape[1:])}",
                       "bytes_per_direction": nbytes},
            "swap_out_gbs": gbs(t_out), "swap_in_gbs": gbs(t_in),
            "roofline": {"bound": "host link", "copy_d2h_gbs": gbs(t_d2h), "copy_h2d_gbs": gbs(t_h2d),
                         "frac_out": round(t_d2h / t_out, 3), "frac_in": round(t_h2d / t_in, 3)},
            "gpu_launches": 2 * args.steps}
    print(json.dumps(line), flush=True)


def run_layers(args, cfg, num_layers=32, pool_blocks=2048, cow_pairs=64):
    """The cache ops of one decode step over every layer of the model: reshape_and_cache of the batch's
    new tokens (distinct random slots) and copy_blocks of cow_pairs copy-on-write pairs, each as ONE
    launch covering all num_layers layers, CUDA-event timed; beside it the same work as one launch
    per layer. Bytes: each token's K and V row read and written, each pair's K and V block read and
    written, per layer. The step's data (over 0.5 GB) exceeds L2, so no flush is needed."""
    from pagedattention_paged_kv_attention_b200 import pagedattn as P
    dev = torch.device("cuda", torch.cuda.current_device())
    kv = torch.bfloat16 if cfg.kv_dtype == "bf16" else (torch.float16 if cfg.kv_dtype == "f16" else torch.uint8)
    it = torch.bfloat16 if cfg.dtype == "bf16" else torch.float16
    T, Hkv, d, bs = cfg.num_seqs, cfg.num_kv_heads, cfg.head_size, cfg.block_size
    shape = (pool_blocks, bs, Hkv, d)
    g = torch.Generator(device=dev).manual_seed(cfg.seed)
    kc = [torch.empty(shape, dtype=kv, device=dev) for _ in range(num_layers)]
    vc = [torch.empty(shape, dtype=kv, device=dev) for _ in range(num_layers)]
    for t in kc + vc:
        t.view(torch.uint8).random_(0, 120, generator=g)
    keys = [torch.randn((T, Hkv, d), generator=g, device=dev).to(it) for _ in range(num_layers)]
    values = [torch.randn((T, Hkv, d), generator=g, device=dev).to(it) for _ in range(num_layers)]
    fp8 = kv == torch.uint8
    ks = [torch.full((Hkv,), 0.01, device=dev) for _ in range(num_layers)] if fp8 else None
    vs = [torch.full((Hkv,), 0.01, device=dev) for _ in range(num_layers)] if fp8 else None
    perm = torch.randperm(pool_blocks * bs, generator=g, device=dev)
    slots = perm[:T].to(torch.int64)
    bperm = torch.randperm(pool_blocks, generator=g, device=dev)
    pairs = torch.stack([bperm[:cow_pairs], bperm[cow_pairs:2 * cow_pairs]], 1).to(torch.int64).contiguous()
    ptr = P.pointer_array
    arrays = [ptr(keys), ptr(values), ptr(kc), ptr(vc)]
    sarr = (ptr(ks), ptr(vs)) if fp8 else (None, None)
    ke, ve = kc[0].element_size(), it.itemsize
    reshape_bytes = num_layers * 2 * T * Hkv * d * (ve + ke)
    copy_bytes = num_layers * 2 * 2 * cow_pairs * bs * Hkv * d * ke
    lib, stream = P.lib, P._stream(None)
    code_in, code_kv = P.dtype_code(it), P.dtype_code(kv)

    def fused():
        # pointer arrays built once, as a caller holding its layers' caches would keep them
        P._check(lib.pa_reshape_and_cache_layers(
            arrays[0].data_ptr(), arrays[1].data_ptr(), code_in, arrays[2].data_ptr(), arrays[3].data_ptr(),
            code_kv, sarr[0].data_ptr() if fp8 else None, sarr[1].data_ptr() if fp8 else None, slots.data_ptr(),
            T, num_layers, Hkv, d, bs, pool_blocks, stream), "pa_reshape_and_cache_layers")
        P._check(lib.pa_copy_blocks_layers(arrays[2].data_ptr(), arrays[3].data_ptr(), num_layers, code_kv,
                                           pairs.data_ptr(), cow_pairs, Hkv, d, bs, pool_blocks, stream),
                 "pa_copy_blocks_layers")

    def per_layer():
        for l in range(num_layers):
            P.reshape_and_cache(keys[l], values[l], kc[l], vc[l], slots, ks[l] if fp8 else None,
                                vs[l] if fp8 else None)
            P.copy_blocks(kc[l], vc[l], pairs)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.steps):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / args.steps

    peaks = measured_peaks()
    peak = peaks.get("hbm_gbs") if peaks else None
    with ClockSampler(gpu_selector(dev)) as clocks:
        t_fused = timed(fused)
        t_loop = timed(per_layer)
    total = reshape_bytes + copy_bytes
    gbs = lambda nb, ms: round(nb / (ms * 1e-3) / 1e9, 2)
    line = {"metric": "multi-layer cache ops GB/s", "value": gbs(total, t_fused), "unit": "GB/s", "impl": "ours",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t_fused, 4),
            "higher_is_better": True, "dtype": cfg.kv_dtype, "data": "synthetic",
            "config": {"workload": f"{cfg.name} cache shape, {num_layers} layers, {T} new tokens, "
                                   f"{cow_pairs} copy-on-write pairs, pool {pool_blocks} blocks per layer",
                       "l2": "step data larger than L2", "bytes_per_step": total},
            "per_layer_launches": {"ms_per_step": round(t_loop, 4), "value": gbs(total, t_loop)},
            "roofline": {"bound": "hbm", "achieved": gbs(total, t_fused), "peak": peak, "unit": "GB/s",
                         "frac": round(gbs(total, t_fused) / peak, 3) if peak else None, "traffic": None,
                         "peak_source": "measured" if peak else None},
            "clocks": clocks.summary(), "gpu_launches": 2 * args.steps}
    print(json.dumps(line), flush=True)


def run_plan(args, cfg, plan_steps=200):
    """Host cost of the block manager per decode step: the workload's batch is admitted (prompts of
    its context lengths), then plan_steps decode plans (one new token for every sequence: slots,
    copy-on-write pairs, block tables, lengths, written into pinned buffers) are timed on the host
    clock. Beside it the oracle's manager doing the same steps (the reference arm of this part)."""
    from pagedattention_paged_kv_attention_b200.block_manager import BlockManager
    from oracle.block_manager import BlockManagerOracle
    lens = W._lengths(cfg, np.random.default_rng(W.sub_seeds(cfg.seed)[0]), cfg.num_seqs).tolist()
    S, bs = len(lens), cfg.block_size
    grow = plan_steps + args.warmup
    need = sum(-(-(L + grow) // bs) for L in lens)
    max_blocks = max(-(-(L + grow) // bs) for L in lens)
    ids = list(range(S))

    def admit(bm):
        for i, L in enumerate(lens):
            bm.add_sequence(i, int(L))

    bm = BlockManager(need + 16, bs)
    admit(bm)
    out = (torch.empty(S, dtype=torch.int64).pin_memory(), torch.empty((S, 2), dtype=torch.int64).pin_memory(),
           torch.empty((S, max_blocks), dtype=torch.int32).pin_memory(), torch.empty(S, dtype=torch.int32).pin_memory())
    for _ in range(args.warmup):
        bm.plan_decode(ids, max_blocks, 0, out)
    t0 = time.perf_counter()
    for _ in range(plan_steps):
        bm.plan_decode(ids, max_blocks, 0, out)
    t_native = (time.perf_counter() - t0) / plan_steps
    ref = BlockManagerOracle(need + 16, bs)
    admit(ref)
    ref_steps = max(1, plan_steps // 10)
    t0 = time.perf_counter()
    for _ in range(ref_steps):
        ref.append_slots(ids)
        ref.block_tables(ids, max_blocks)
    t_ref = (time.perf_counter() - t0) / ref_steps
    line = {"metric": "block-manager decode plan: sequences planned per second", "value": round(S / t_native),
            "unit": "seq/s", "impl": "ours", "n_gpus": 1, "steps": plan_steps, "warmup": args.warmup, "ms_per_step": round(t_native * 1e3, 4), "higher_is_better": True, "dtype": "int64",
            "data": "synthetic",
            "config": {"workload": f"{cfg.name} batch: {S} sequences, context {min(lens)}..{max(lens)}, block "
                                   f"{bs}, one token per sequence per step into pinned buffers"},
            "cpu_baseline": {"value": round(S / t_ref), "unit": "seq/s", "cores": 1, "kind": "oracle",
                             "sample": f"{ref_steps} steps of the oracle's manager on the same batch"},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def oracle_inputs(cfg, w):
    """The workload as oracle arrays (FP8 pools quantised by the oracle's own encoder)."""
    import oracle
    kb, vb = bits16(w.key_values), bits16(w.value_values)
    ks = vs = None
    if cfg.kv_dtype == "fp8_e4m3":
        ks, vs = w.k_scale.cpu().numpy(), w.v_scale.cpu().numpy()
        kb, vb = oracle.quantize_e4m3(kb, cfg.dtype, ks), oracle.quantize_e4m3(vb, cfg.dtype, vs)
    elif cfg.kv_dtype == "fp8_e4m3_block":
        ks, vs = w.k_scale.cpu().numpy(), w.v_scale.cpu().numpy()
        kb, vb = oracle.quantize_e4m3_blocks(kb, cfg.dtype, ks), oracle.quantize_e4m3_blocks(vb, cfg.dtype, vs)
    return dict(query_bits=bits16(w.query), q_dtype=cfg.dtype, key_cache=kb, value_cache=vb, kv_dtype=cfg.kv_dtype,
                block_tables=w.block_tables.cpu().numpy(), context_lens=w.context_lens.cpu().numpy(),
                scale=cfg.softmax_scale, k_scale=ks, v_scale=vs)


def host_cores():
    """Host CPU facts behind the oracle figures: logical CPUs, the CPUs this process may run on, and the
    cgroup CPU quota when one is set."""
    info = {"cpu_count": os.cpu_count()}
    try:
        info["affinity"] = len(os.sched_getaffinity(0))
    except AttributeError:
        info["affinity"] = os.cpu_count()
    try:
        quota, period = open("/sys/fs/cgroup/cpu.max").read().split()[:2]
        info["cgroup_quota_cpus"] = None if quota == "max" else round(int(quota) / int(period), 2)
    except (OSError, ValueError):
        info["cgroup_quota_cpus"] = None
    return info


def oracle_threads():
    """Threads for the all-core oracle figure: the CPUs this process may use (and no more than the
    cgroup quota allows)."""
    h = host_cores()
    n = h["affinity"] or 1
    if h["cgroup_quota_cpus"]:
        n = min(n, max(1, int(h["cgroup_quota_cpus"])))
    return n


ORACLE_ALL_CORE_GFLOP = 2.0    # work of one all-core oracle pass (about a second on 16 cores)
ORACLE_ONE_CORE_GFLOP = 0.15   # work of one single-thread pass


def decode_lengths(cfg, seed):
    """The batch's context lengths, as make_workload draws them (no values are generated)."""
    return W._lengths(cfg, np.random.default_rng(W.sub_seeds(seed)[0]), cfg.num_seqs)


def decode_config(cfg, lens, world):
    """The workload's description in the JSON line; both arms print the same one."""
    kv = W.ideal_bytes(lens, cfg.num_kv_heads, cfg.head_size, 1 if cfg.kv_dtype.startswith("fp8") else 2,
                       cfg.block_size, cfg.num_heads, 2)["kv"]
    return {"workload": cfg.description, "name": cfg.name, "num_seqs": len(lens), "num_heads": cfg.num_heads,
            "num_kv_heads": cfg.num_kv_heads, "head_size": cfg.head_size, "block_size": cfg.block_size,
            "kv_dtype": cfg.kv_dtype, "context_tokens": int(np.sum(lens)), "max_context_len": int(np.max(lens)),
            "seed": cfg.seed,
            "l2": "inputs larger than L2: %.2f GB of K/V read per step vs 126 MB L2" % (kv / 1e9),
            "parallelism": f"dp{world} (independent sequence batches)"}


def first_sequences(cfg, lens, gflop):
    """How many leading sequences of the batch fit in `gflop` of attention work (at least one)."""
    work = np.cumsum(np.asarray(lens, dtype=np.float64) * cfg.num_heads * 4 * cfg.head_size)
    return int(max(1, min(len(lens), np.searchsorted(work, gflop * 1e9, side="right"))))


def time_passes(fn, passes, warmup):
    for _ in range(warmup):
        fn()
    times = []
    for _ in range(passes):
        t0 = time.perf_counter()
        fn()
        times.append(time.perf_counter() - t0)
    return times


def oracle_decode_timing(cfg, passes=None, warmup=1, seconds=8.0):
    """The oracle, as it stands, on a deterministic sample of the decode workload: the first sequences
    of the batch (seed cfg.seed) that fit in ORACLE_ALL_CORE_GFLOP, on all usable host cores; and the
    first ones that fit in ORACLE_ONE_CORE_GFLOP on one thread. Each figure is the K/V bytes of its
    sample over the median pass time. passes=None fills about `seconds` with passes (at least 3)."""
    import dataclasses
    import oracle
    threads = oracle_threads()
    lens = decode_lengths(cfg, cfg.seed)
    cfg_s = dataclasses.replace(cfg, num_blocks=None)   # the sample's pool: 1.2x its blocks (placement only)
    kv_elem = 1 if cfg.kv_dtype.startswith("fp8") else 2

    def case(n, nthreads):
        w = W.make_workload(cfg_s, seed=cfg.seed, num_seqs=n, prefilled=True)
        inp = oracle_inputs(cfg, w)
        kv = W.ideal_bytes(w.context_lens.numpy(), cfg.num_kv_heads, cfg.head_size, kv_elem, cfg.block_size,
                           cfg.num_heads, 2)["kv"]
        return (lambda: oracle.paged_attention(**inp, num_threads=nthreads)), kv, int(w.context_lens.sum())

    n_all = first_sequences(cfg, lens, ORACLE_ALL_CORE_GFLOP)
    fn, kv, tokens = case(n_all, threads)
    if passes is None:
        t0 = time.perf_counter()
        fn()
        passes = max(3, int(seconds / max(time.perf_counter() - t0, 1e-3)))
        warmup = max(0, warmup - 1)
    times = time_passes(fn, passes, warmup)
    t = float(np.median(times))
    n_one = first_sequences(cfg, lens, ORACLE_ONE_CORE_GFLOP)
    fn1, kv1, tokens1 = case(n_one, 1)
    times1 = time_passes(fn1, 3, 1)
    t1 = float(np.median(times1))
    stats = lambda ts: {"median": round(float(np.median(ts)), 4), "min": round(min(ts), 4),
                        "max": round(max(ts), 4), "passes": len(ts)}
    return {"value": round(kv / t / 1e9, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"first {n_all} of {cfg.num_seqs} sequences ({tokens} context tokens, {kv} K/V bytes), "
                      f"fp64, {threads} threads, median of {len(times)} passes",
            "tokens_per_s": round(n_all / t, 3), "pass_s": stats(times), "host": host_cores(),
            "single_thread": {"value": round(kv1 / t1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                              "sample": f"first {n_one} sequences ({tokens1} context tokens, {kv1} K/V bytes), "
                                        f"fp64, 1 thread, median of 3 passes",
                              "pass_s": stats(times1)}}


if __name__ == "__main__":
    main()
