#!/usr/bin/env python
"""Throughput of PACE periodic low-bit recurrent-state decode on one node.

    python bench.py [--gpus N --steps K --warmup W] [--impl pace|reference]

One *step* is one period of the hot path over the whole pool: P decode
launches (one token for each of the B x H heads) followed by one commit
launch.  The default workload is the concurrency-stress configuration
(B=4096 sequences, H=48 heads, d_k=d_v=128, P=8, 25% INT8 heads, bf16 io),
whose 2.06 GB state pool is far larger than the 126 MB L2, so no L2 flush is
needed between steps.  The state is first warmed by a 512-token unquantised
fp32 prefill (pace_gdn_step_f32), then encoded into the pool.

Printed: one JSON line (rank 0).  ``value`` is head-tokens/s over all ranks
(each rank holds its own full pool: weak scaling; no collective on the data
path).  Kernel durations come from CUDA events on the launching stream.
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
sys.path.insert(0, ROOT)

HBM_FALLBACK_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=128, help="timed periods (128 x P=8 = 1024 tokens)")
    ap.add_argument("--warmup", type=int, default=3, help="untimed periods before timing")
    ap.add_argument("--impl", choices=["pace", "reference"], default="pace")
    ap.add_argument("--workload", default="concurrency_stress")
    ap.add_argument("--period", type=int, default=None, help="override P")
    ap.add_argument("--axis", choices=["col", "row"], default=None, help="override the scale axis")
    ap.add_argument("--commit-engine", choices=["tcgen05", "mma"], default="tcgen05",
                    help="period-commit kernel (tcgen05 falls back to mma for shapes it is not built for)")
    ap.add_argument("--prefill-tokens", type=int, default=64,
                    help="tokens of the chunked fp32 prefill measured after the decode (0: skip)")
    ap.add_argument("--commit-threshold", default=None,
                    help="also measure the adaptive period with this threshold on the accumulated "
                         "update's Frobenius norm ('auto': the median after 3 tokens)")
    ap.add_argument("--window", action="store_true",
                    help="also measure the pure-write window (pace_window_step, window = P)")
    ap.add_argument("--bits-from-gates", action="store_true",
                    help="choose the 8-bit heads from the prefill gates (slowest mean decay) "
                         "instead of the workload's seeded choice")
    ap.add_argument("--slots", type=int, default=None, help="override B (smaller profiling case)")
    ap.add_argument("--prefill", type=int, default=None, help="warm-up prefill tokens (default: workload's)")
    ap.add_argument("--e2e-steps", type=int, default=4)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time the periods from eager launches only (by default the headline value is "
                         "from replays of one captured CUDA graph of a period; the eager timing is "
                         "reported beside it under 'lockstep')")
    ap.add_argument("--no-compare", action="store_true", help="skip the bf16-state comparison path")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-period-sweep", action="store_true",
                    help="skip the period sweep (B=512, H=32, P in 1,2,4,8,16 with fp32-trajectory drift)")
    ap.add_argument("--sweep-tokens", type=int, default=1024, help="decode tokens per period in the sweep")
    ap.add_argument("--cpu-sample-slots", type=int, default=32)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--schedule", choices=["staggered", "lockstep"], default="lockstep",
                    help="phases of the slot groups for the headline value (per-kernel numbers "
                         "always come from a lockstep pass)")
    ap.add_argument("--stagger-blocks", default="2,2",
                    help="blocks per SM of the decode and the commit launches in the staggered schedule")
    return ap.parse_args()


# ----------------------------------------------------------------------------- helpers

def tensor_peak():
    """Dense bf16/f16 tensor peak in TFLOP/s for a kernel timed inside a long
    step (the sustained figure of MEASURED_PEAKS.json; fallback 1400)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 1400.0, "fallback"


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return HBM_FALLBACK_GBS, "fallback"


KERNEL_SOURCES = {"decode_step": "decode_kernels.cu", "commit": "commit_tc_kernels.cu"}
COMMIT_SOURCES = {"tcgen05": "commit_tc_kernels.cu", "mma": "commit_kernels.cu"}


def _code_only(text: str) -> str:
    """C++ source without comments and with whitespace collapsed: edits to
    comments do not change what a traffic record was measured on."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_digest(kernel: str, source: str = None) -> str:
    """sha256 (16 hex digits) of a kernel's source file and every csrc header
    it includes, directly or not, comments left out: what a DRAM-traffic
    record depends on."""
    import re
    csrc = os.path.join(ROOT, "bit_recurrent_state_pace_b200", "csrc")
    todo, seen = [source or KERNEL_SOURCES[kernel]], []
    while todo:
        fn = todo.pop()
        if fn in seen or not os.path.exists(os.path.join(csrc, fn)):
            continue
        seen.append(fn)
        with open(os.path.join(csrc, fn)) as f:
            todo += re.findall(r'^#include "([^"/]+)"', f.read(), flags=re.M)
    h = hashlib.sha256()
    for fn in sorted(seen):
        with open(os.path.join(csrc, fn)) as f:
            h.update(fn.encode() + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, digest: str):
    """DRAM bytes per launch recorded by an ncu capture of the same kernel
    sources (profiles/*.txt lines 'traffic <kernel> <bytes> <digest>')."""
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None
    for fn in sorted(os.listdir(pdir)):
        if not fn.endswith(".txt"):
            continue
        with open(os.path.join(pdir, fn)) as f:
            for line in f:
                tok = line.split()
                if len(tok) == 4 and tok[0] == "traffic" and tok[1] == kernel and tok[3] == digest:
                    return float(tok[2])
    return None


class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons while timing."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.06)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            p = [x.strip() for x in line.split(",")]
            if len(p) < 8:
                continue
            try:
                sm.append(float(p[0]))
                mx.append(float(p[1]))
            except ValueError:
                continue
            for name, val in zip(names, p[4:8]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def oracle_sample_rate(w, bits, slots: int, seed: int):
    """The fp64 oracle as it stands, on `slots` whole sequences (all H heads)
    for one period of P tokens plus the commit; head-tokens per second."""
    import numpy as np
    import torch
    import oracle as orc
    import pace_synth
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        cores = os.cpu_count() or 1
    sub = w.replace(B=slots)
    heads = [(b, h) for b in range(slots) for h in range(w.H)]
    S0 = pace_synth.random_state(len(heads), w.d_v, w.d_k, seed=seed).numpy()
    state, _ = orc.PoolState.from_fp32(S0, [bits[h] for _, h in heads], w.axis)
    toks = []
    for t in range(w.P):
        inp = pace_synth.token_inputs(sub, t, seed=seed)
        toks.append({k: v.reshape(len(heads), -1).double().numpy().squeeze(-1) if v.dim() == 2
                     else v.reshape(len(heads), -1).double().numpy() for k, v in inp.items()})
    t0 = time.perf_counter()
    orc.period_reference(state, toks, w.P)
    dt = time.perf_counter() - t0
    units = len(heads) * w.P
    return {"value": units / dt, "unit": "head-tokens/s", "cores": int(cores), "kind": "oracle",
            "sample": f"{slots} slots x {w.H} heads ({len(heads)} heads), one period of P={w.P} "
                      f"tokens plus its commit, fp64 numpy, {dt:.1f} s"}


def alg_bytes(w, bits, n: int):
    """Algorithmic DRAM bytes of one decode launch at buffer position n
    (1..P) and of one commit launch (every head commits)."""
    import bit_recurrent_state_pace_b200 as pace
    rec = [pace.pace_pool_bytes(1, 1, w.d_k, w.d_v, w.P, 0, 0, [b])[0] for b in bits]
    esz = 2 if w.io_dtype == "bf16" else 4
    row = (w.d_k + w.d_v + 2) * esz            # buffered k, v, alpha, beta
    inp = (2 * w.d_k + w.d_v + 2) * esz        # q, k, v, alpha, beta of the token
    per_head = inp + (n - 1) * row + row + 4 * w.d_v + 8   # + buffer row write + o + fill r/w
    decode = w.B * sum(rec) + w.B * w.H * per_head
    commit = 2 * w.B * sum(rec) + w.B * w.H * (w.P * row + 8)
    return decode, commit


# ----------------------------------------------------------------------------- arms

def run_reference(args, rank: int, world: int):
    if rank != 0:
        return
    import pace_synth
    w = pace_synth.workload(args.workload)
    if args.period:
        w = w.replace(P=args.period)
    bits = pace_synth.head_bits(w, args.seed)
    samples = []
    # each step: one whole sequence (all H heads) for one period, so that the
    # default --steps/--warmup run stays within a few minutes of CPU time
    for _ in range(args.warmup):
        oracle_sample_rate(w, bits, 1, args.seed)
    for _ in range(args.steps):
        samples.append(oracle_sample_rate(w, bits, 1, args.seed))
    val = statistics.median(s["value"] for s in samples)
    base = samples[0]
    # each timed step is one whole sequence (all H heads) for one period: the
    # time of that sample, not of the full pool; the rate is per head-token
    sample_ms = 1000.0 * w.H * w.P / val
    line = {
        "impl": "reference", "metric": "decode head-tokens/s (B x H heads, 4-bit state, P=%d)" % w.P,
        "value": val, "unit": "head-tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": sample_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_config(w, bits, state_bytes_of(w, bits)),
                       parallelism=f"{world} independent pools (no collective)",
                       int8_head_choice="seeded",
                       int8_head_list=[h for h in range(w.H) if bits[h] == 8],
                       seq_tokens_per_s=val / w.H),
        "step_sample": f"one sequence (all {w.H} heads) for one period of P={w.P} tokens per step",
        "extrapolated_from_heads": w.H,
        "full_pool_ms_per_period_at_this_rate": 1000.0 * w.B * w.H * w.P / val,
        "cpu_baseline": dict(base, value=val),
        "e2e": {"value": val, "unit": "head-tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


L2_BYTES = 126 * 1024 * 1024


def state_bytes_of(w, bits):
    """Bytes of the pool's state region (records of codes + FP16 scales, each
    padded to 16 bytes), by the layout include/pace.h documents."""
    groups = w.d_k if w.axis == "col" else w.d_v
    rec = [(w.d_v * w.d_k * b // 8 + 2 * groups + 15) // 16 * 16 for b in bits]
    return w.B * ((sum(rec) + 15) // 16 * 16)


def workload_config(w, bits, state_bytes=None):
    n8 = sum(1 for b in bits if b == 8)
    if state_bytes is None or state_bytes >= 4 * L2_BYTES:
        l2 = "state pool larger than L2 (no flush needed)"
    else:
        l2 = (f"state pool {state_bytes / 2**20:.0f} MiB, within 4x of the 126 MB L2: no flush, "
              "so part of the traffic is served from L2")
    return {"workload": f"{w.name}: B={w.B} H={w.H} d_k={w.d_k} d_v={w.d_v} P={w.P} "
                        f"{n8}/{w.H} INT8 heads, {w.axis} scales, {w.io_dtype} io",
            "B": w.B, "H": w.H, "d_k": w.d_k, "d_v": w.d_v, "P": w.P, "int8_heads": n8,
            "scale_axis": w.axis, "io_dtype": w.io_dtype, "state_dtype": "int4/int8 codes + fp16 scales",
            "l2": l2, "prefill_tokens": w.warmup}


class Staggered:
    """Continuous-batching phases: the slots form P groups, group g running
    one token ahead of group g - 1, so that every decode step one group's
    buffers are full.  Each step the full group is committed and decoded on
    stream b while the other groups decode on stream a; with both launches
    held to part of every SM (blocks_per_sm) the commit's arithmetic overlaps
    the other slots' memory-bound decode.  Over P steps every slot decodes P
    tokens and commits once, the same work as P lockstep steps + 1 commit."""

    def __init__(self, pace, pool, w, dec_bps: int, com_bps: int):
        import torch
        from bit_recurrent_state_pace_b200.ranks import slot_range
        self.pace, self.pool, self.P = pace, pool, w.P
        self.groups = [slot_range(w.B, w.P, g) for g in range(w.P)]
        self.dec_bps, self.com_bps = dec_bps, com_bps
        self.sa, self.sb = torch.cuda.Stream(), torch.cuda.Stream()
        self.t = 0
        self.launches = 0

    def _dec(self, b0, nb, x, o, bps, stream):
        if nb > 0:
            self.pace.pace_decode_step_range(self.pool.handle, b0, nb, bps, x["q"], x["k"], x["v"],
                                             x["alpha"], x["beta"], o, stream.cuda_stream)
            self.launches += 1

    def preroll(self, toks, outs, stream):
        """From all fills 0: group g takes g + 1 tokens (group P-1 ends full)."""
        B = self.groups[-1][0] + self.groups[-1][1]
        for r in range(self.P):
            b0 = self.groups[r][0]
            self._dec(b0, B - b0, toks[r], outs[r], 0, stream)
        self.t = 1

    def step(self, x, o, main):
        import torch
        gf = (-self.t) % self.P
        b0, nb = self.groups[gf]
        B = self.groups[-1][0] + self.groups[-1][1]
        ev = torch.cuda.Event()
        ev.record(main)
        self.sa.wait_event(ev)
        self.sb.wait_event(ev)
        self.pace.pace_commit_period_range(self.pool.handle, b0, nb, self.com_bps, self.sb.cuda_stream)
        self.launches += 1
        self._dec(b0, nb, x, o, self.dec_bps, self.sb)
        self._dec(0, b0, x, o, self.dec_bps, self.sa)
        self._dec(b0 + nb, B - b0 - nb, x, o, self.dec_bps, self.sa)
        main.wait_stream(self.sa)
        main.wait_stream(self.sb)
        self.t += 1


def run_pace(args, rank: int, world: int):
    import torch
    import bit_recurrent_state_pace_b200 as pace
    import pace_synth

    dev = torch.device("cuda", torch.cuda.current_device())
    w = pace_synth.workload(args.workload)
    if args.period:
        w = w.replace(P=args.period)
    if args.prefill is not None:
        w = w.replace(warmup=args.prefill)
    if args.slots is not None:
        w = w.replace(B=args.slots)
    if args.axis is not None:
        w = w.replace(axis=args.axis)
    bits = pace_synth.head_bits(w, args.seed)
    BH, P = w.B * w.H, w.P
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream

    cpu_base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu_base = oracle_sample_rate(w, bits, args.cpu_sample_slots, args.seed)

    # ---- state: unquantised fp32 prefill, then encode into the pool
    io_code = pace.PACE_IO_BF16 if w.io_dtype == "bf16" else pace.PACE_IO_F32
    S = torch.zeros(BH, w.d_v, w.d_k, dtype=torch.float32, device=dev)
    gates = [] if args.bits_from_gates else None
    for t in range(w.warmup):
        inp = pace_synth.token_inputs(w, t, seed=args.seed + rank, device=dev, phase="warmup")
        pace.pace_gdn_step_f32(S, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                               io_code, None, BH, w.d_k, w.d_v)
        if gates is not None:
            gates.append(inp["alpha"])
    if gates:
        rates = pace.pace_decay_rates(torch.stack(gates).contiguous(), w.H, io_code)
        bits = pace.pace_select_head_bits(rates.cpu().tolist(), sum(1 for b in bits if b == 8))
        del gates
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, P, bits, axis=w.axis, io=w.io_dtype, device=dev)
    engine = args.commit_engine
    try:
        pool.set_commit_engine(pace.PACE_COMMIT_TCGEN05 if engine == "tcgen05" else pace.PACE_COMMIT_MMA)
    except pace.PaceError:
        engine = "mma"
        pool.set_commit_engine(pace.PACE_COMMIT_MMA)
    pool.load(S)
    S_bf16 = None if args.no_compare else S.to(torch.bfloat16).view(torch.int16)
    del S
    torch.cuda.synchronize()

    toks = [pace_synth.token_inputs(w, t, seed=args.seed + rank, device=dev) for t in range(P)]
    outs = [torch.empty(w.B, w.H, w.d_v, dtype=torch.float32, device=dev) for _ in range(P)]

    def period(ev=None):
        for n in range(P):
            x = toks[n]
            if ev is not None:
                ev[n][0].record(stream)
            pace.pace_decode_step(pool.handle, x["q"], x["k"], x["v"], x["alpha"], x["beta"], outs[n], sp)
            if ev is not None:
                ev[n][1].record(stream)
        if ev is not None:
            ev[P][0].record(stream)
        pace.pace_commit_period(pool.handle, sp)
        if ev is not None:
            ev[P][1].record(stream)

    for _ in range(args.warmup):
        period()
    assert pool.status() == 0, "device status flags set during warm-up"

    mk = lambda: torch.cuda.Event(enable_timing=True)
    evs = [[(mk(), mk()) for _ in range(P + 1)] for _ in range(args.steps)]
    gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
    if not gpu_uuid.startswith("GPU-"):
        gpu_uuid = "GPU-" + gpu_uuid
    barrier(world)
    torch.cuda.synchronize()
    sampler = ClockSampler(gpu_uuid)
    time.sleep(0.2)
    t_start, t_end = mk(), mk()
    t_start.record(stream)
    for s in range(args.steps):
        period(evs[s])
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier(world)
    elapsed_ms = t_start.elapsed_time(t_end)
    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)
    status = pool.status()

    dec_ms = [[evs[s][n][0].elapsed_time(evs[s][n][1]) for s in range(args.steps)] for n in range(P)]
    com_ms = [evs[s][P][0].elapsed_time(evs[s][P][1]) for s in range(args.steps)]
    dec_bytes = [alg_bytes(w, bits, n + 1)[0] for n in range(P)]
    com_bytes = alg_bytes(w, bits, P)[1]
    dec_avg_ms = statistics.mean(statistics.mean(x) for x in dec_ms)
    dec_avg_bytes = statistics.mean(dec_bytes)
    com_avg_ms = statistics.mean(com_ms)
    hbm, peak_kind = measured_peaks()
    dec_gbs = dec_avg_bytes / (dec_avg_ms * 1e-3) / 1e9
    com_gbs = com_bytes / (com_avg_ms * 1e-3) / 1e9
    digest = {"decode_step": kernel_source_digest("decode_step"),
              "commit": kernel_source_digest("commit", COMMIT_SOURCES[engine])}
    dominant = "decode_step" if dec_avg_ms * P >= com_avg_ms else "commit"
    ach = dec_gbs if dominant == "decode_step" else com_gbs
    traffic = ncu_traffic(dominant, digest[dominant])

    from bit_recurrent_state_pace_b200.ranks import aggregate_rate
    lockstep_value = aggregate_rate(BH * P * args.steps, world, elapsed_ms)
    lockstep_ms = elapsed_ms

    # ---- the same periods replayed from one captured CUDA graph (reported
    #      beside the headline; the per-kernel numbers above come from the
    #      launches themselves)
    graph_rec = None
    if not args.no_graph and args.schedule == "lockstep":
        try:
            graph_rec = time_graph(pace, pool, toks, outs, P, args, stream, world, dev, mk, gpu_uuid)
        except Exception as exc:   # capture refused: the eager timing stands
            graph_rec = {"error": f"{type(exc).__name__}: {exc}"}
            torch.cuda.synchronize()
        status |= pool.status()

    # ---- staggered phases (continuous batching): same work per P steps
    stag = None
    if args.schedule == "staggered":
        dbps, cbps = (int(v) for v in args.stagger_blocks.split(","))
        stag = Staggered(pace, pool, w, dbps, cbps)
        stag.preroll(toks, outs, stream)
        for i in range(args.warmup * P):
            stag.step(toks[stag.t % P], outs[stag.t % P], stream)
        torch.cuda.synchronize()
        assert pool.status() == 0, "device status flags set during the staggered warm-up"
        barrier(world)
        torch.cuda.synchronize()
        sampler = ClockSampler(gpu_uuid)
        time.sleep(0.2)
        stag.launches = 0
        a, b = mk(), mk()
        a.record(stream)
        for i in range(args.steps * P):
            stag.step(toks[stag.t % P], outs[stag.t % P], stream)
        b.record(stream)
        torch.cuda.synchronize()
        clocks = sampler.stop()
        barrier(world)
        elapsed_ms = max_over_ranks(a.elapsed_time(b), world, dev)
        status |= pool.status()
    if stag is None and graph_rec and "value" in graph_rec:
        elapsed_ms = graph_rec["ms_per_step"] * args.steps   # the headline from the graph replays
        clocks = graph_rec["clocks"] or clocks
    value = aggregate_rate(BH * P * args.steps, world, elapsed_ms)

    # ---- bf16-state comparison path (unquantised, same shape)
    compare = None
    if S_bf16 is not None:
        for _ in range(2):
            x = toks[0]
            pace.pace_gdn_step_bf16(S_bf16, x["q"], x["k"], x["v"], x["alpha"], x["beta"], pool.io,
                                    outs[0], BH, w.d_k, w.d_v, sp)
        ntok = 2 * P
        a, b = mk(), mk()
        a.record(stream)
        for t in range(ntok):
            x = toks[t % P]
            pace.pace_gdn_step_bf16(S_bf16, x["q"], x["k"], x["v"], x["alpha"], x["beta"], pool.io,
                                    outs[t % P], BH, w.d_k, w.d_v, sp)
        b.record(stream)
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / ntok
        esz = 2 if w.io_dtype == "bf16" else 4
        bbytes = BH * (2 * w.d_v * w.d_k * 2 + (2 * w.d_k + w.d_v + 2) * esz + 4 * w.d_v)
        compare = {"bf16_state": {"value": BH / (ms * 1e-3), "unit": "head-tokens/s",
                                  "ms_per_token": ms, "achieved_gbs": bbytes / (ms * 1e-3) / 1e9,
                                  "state_bytes": BH * w.d_v * w.d_k * 2},
                   "pace_state_bytes": int(pool.state.numel()),
                   "pace_ms_per_token": elapsed_ms / world / (args.steps * P) if world == 1 else None}
        del S_bf16

    # ---- end to end through the public API with pinned host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, pace, pool, w, toks, outs, stream, world, dev, stag)

    # ---- adaptive period: every token is a decode step and a commit launch for
    #      the heads marked by it; the pool is restored afterwards
    adaptive = None
    if args.commit_threshold is not None and stag is None:
        adaptive = run_adaptive(args, pace, pool, w, toks, outs, stream, world, dev, mk)

    # ---- pure-write window: every token is a window step (the oldest pair of
    #      a full window is merged into the history); the pool is restored
    window = None
    if args.window and stag is None:
        window = run_window(args, pace, pool, w, toks, outs, stream, world, dev, mk)

    # ---- chunked fp32 prefill of T tokens into the whole pool (after the decode
    #      numbers: it rewrites the pool); not part of the headline step
    prefill = None
    if args.prefill_tokens > 0 and stag is None:
        Tp = args.prefill_tokens
        ptoks = [pace_synth.token_inputs(w, 100000 + t, seed=args.seed + rank, device=dev) for t in range(Tp)]
        pin = {key: torch.stack([x[key] for x in ptoks]).contiguous() for key in ptoks[0]}
        del ptoks
        po = torch.empty(Tp, w.B, w.H, w.d_v, dtype=torch.float32, device=dev)
        pool.prefill(pin["q"], pin["k"], pin["v"], pin["alpha"], pin["beta"], po)   # warm-up call
        torch.cuda.synchronize()
        barrier(world)
        a, b = mk(), mk()
        a.record(stream)
        pool.prefill(pin["q"], pin["k"], pin["v"], pin["alpha"], pin["beta"], po)
        b.record(stream)
        torch.cuda.synchronize()
        pms = max_over_ranks(a.elapsed_time(b), world, dev)
        esz = 2 if w.io_dtype == "bf16" else 4
        pbytes = (Tp * BH * ((2 * w.d_k + w.d_v + 2) * esz + 4 * w.d_v) + 2 * int(pool.state.numel()))
        from bit_recurrent_state_pace_b200.ranks import aggregate_rate
        # flops: per head-token S k, S q and the rank-one write, 2 d_k d_v each
        pflops = 6.0 * w.d_k * w.d_v * BH * Tp
        tpk, tpk_kind = tensor_peak()
        ach_tf = pflops / (pms * 1e-3) / 1e12
        prefill = {"tokens": Tp, "value": aggregate_rate(BH * Tp, world, pms), "unit": "head-tokens/s",
                   "ms": pms, "alg_bytes": pbytes, "achieved_gbs": pbytes / (pms * 1e-3) / 1e9,
                   "frac_of_peak": pbytes / (pms * 1e-3) / 1e9 / measured_peaks()[0],
                   "roofline_flops": {"bound": "tensor", "achieved": ach_tf, "peak": tpk, "unit": "TFLOP/s",
                                      "frac": ach_tf / tpk, "flops_per_head_token": 6 * w.d_k * w.d_v,
                                      "peak_source": f"{tpk_kind} bf16_tflops_sustained (f16 operands, same rate)"},
                   "status": pool.status()}
        del pin, po

    # ---- period sweep on its own workload (one GPU only: it has no collective
    #      and would only lengthen a multi-rank run)
    sweep = None
    if world == 1 and not args.no_period_sweep and stag is None:
        del toks, outs
        sweep = run_period_sweep(args, pace, dev, mk)

    if rank == 0:
        line = {
            "metric": "decode head-tokens/s (B x H heads, 4-bit state, P=%d)" % P,
            "value": value, "unit": "head-tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": dict(workload_config(w, bits, int(pool.state.numel())),
                           parallelism=f"{world} independent pools (no collective)",
                           int8_head_choice=("slowest mean decay over the prefill gates"
                                             if args.bits_from_gates else "seeded"),
                           int8_head_list=[h for h in range(w.H) if bits[h] == 8],
                           seq_tokens_per_s=value / w.H),
            "buffer_bytes": int(pool.buffer.numel()),
            "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s",
                         "frac": ach / hbm, "traffic": traffic, "kernel": dominant,
                         "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)" if peak_kind == "measured" else "fallback 6.65 TB/s"},
            "kernels": {
                "decode_step": {"avg_ms": dec_avg_ms, "alg_bytes_per_launch": dec_avg_bytes,
                                "achieved_gbs": dec_gbs, "frac_of_peak": dec_gbs / hbm,
                                "ms_by_fill": [statistics.mean(x) for x in dec_ms]},
                "commit": {"avg_ms": com_avg_ms, "alg_bytes_per_launch": com_bytes,
                           "achieved_gbs": com_gbs, "frac_of_peak": com_gbs / hbm},
                "source_digest": digest,
                "commit_engine": engine,
            },
            "clocks": clocks,
            "e2e": e2e,
            "gpu_launches": stag.launches if stag is not None else args.steps * (P + 1),
            "schedule": ("staggered: %d slot groups one token apart; each step the full group's "
                         "commit and decode (stream b) overlap the other groups' decode (stream a), "
                         "%s blocks per SM" % (P, args.stagger_blocks)) if stag is not None
                        else ("lockstep: every slot at the same phase; "
                              + ("periods replayed from one captured CUDA graph (eager launches under "
                                 "'lockstep')" if graph_rec and "value" in graph_rec else "eager launches")),
            "lockstep": {"value": lockstep_value, "ms_per_step": lockstep_ms / args.steps},
            "cuda_graph": graph_rec,
            "device_status": status,
            "comparison": compare,
            "prefill": prefill,
            "adaptive": adaptive,
            "window": window,
            "period_sweep": sweep,
            "cpu_baseline": cpu_base,
        }
        print(json.dumps(line), flush=True)


def time_graph(pace, pool, toks, outs, P, args, stream, world, dev, mk, gpu_uuid):
    """K periods replayed from one captured CUDA graph of a period (P decode
    launches + the commit, the same calls and buffers as the eager loop)."""
    import torch
    from bit_recurrent_state_pace_b200.ranks import aggregate_rate
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for n in range(P):
            x = toks[n]
            pace.pace_decode_step(pool.handle, x["q"], x["k"], x["v"], x["alpha"], x["beta"], outs[n],
                                  side.cuda_stream)
        pace.pace_commit_period(pool.handle, side.cuda_stream)
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        g.replay()
    barrier(world)
    torch.cuda.synchronize()
    sampler = ClockSampler(gpu_uuid)
    time.sleep(0.2)
    a, b = mk(), mk()
    a.record(stream)
    for _ in range(args.steps):
        g.replay()
    b.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier(world)
    gms = max_over_ranks(a.elapsed_time(b), world, dev)
    BH = pool.B * pool.H
    return {"value": aggregate_rate(BH * P * args.steps, world, gms), "unit": "head-tokens/s",
            "ms_per_step": gms / args.steps, "launches_per_step": P + 1, "clocks": clocks,
            "note": "one period (P decode launches + the commit) captured once, replayed K times"}


def run_period_sweep(args, pace, dev, mk):
    """The period-sweep workload (B=512, H=32, d=128, all INT4, outlier value
    channels, bf16 io) for each P in {1, 2, 4, 8, 16}: throughput, per-kernel
    HBM GB/s, and the drift of the outputs from an unquantised fp32 trajectory
    run on the same tokens.

    Every P starts from the same pool: the 512-token fp32 warm-up state,
    encoded.  The fp32 trajectory (pace_gdn_step_f32) starts from that
    encoded state, dequantised, so that what it measures is the rounding
    during decode, not the one initial encode they share.  Drift of head
    (b, h) at token t: ||o - o_fp32||_inf / ||o_fp32||_inf; mean and max over
    the B x H heads at a few horizons."""
    import torch
    import pace_synth

    w0 = pace_synth.workload("period_sweep")
    T = args.sweep_tokens
    bits = pace_synth.head_bits(w0, args.seed)
    BH = w0.B * w0.H
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    io_code = pace.PACE_IO_BF16 if w0.io_dtype == "bf16" else pace.PACE_IO_F32
    horizons = [t for t in (8, 16, 64, 256, 1024, 4096) if t <= T]
    if T not in horizons:
        horizons.append(T)

    S = torch.zeros(BH, w0.d_v, w0.d_k, dtype=torch.float32, device=dev)
    for t in range(w0.warmup):
        inp = pace_synth.token_inputs(w0, t, seed=args.seed, device=dev, phase="warmup")
        pace.pace_gdn_step_f32(S, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                               io_code, None, BH, w0.d_k, w0.d_v)
    toks = [pace_synth.token_inputs(w0, t, seed=args.seed, device=dev) for t in range(T)]

    # the unquantised trajectory from the encoded start, for each scale axis run
    o = torch.empty(w0.B, w0.H, w0.d_v, dtype=torch.float32, device=dev)
    refs = {}
    for axis in ("col", "row"):
        pool = pace.PacePool(w0.B, w0.H, w0.d_k, w0.d_v, 1, bits, axis=axis, io=w0.io_dtype, device=dev)
        pool.load(S)
        S_ref = pool.export().view(BH, w0.d_v, w0.d_k).contiguous()
        del pool
        ref = {}
        for t in range(T):
            x = toks[t]
            pace.pace_gdn_step_f32(S_ref, x["q"], x["k"], x["v"], x["alpha"], x["beta"], io_code, o,
                                   BH, w0.d_k, w0.d_v)
            if t + 1 in horizons:
                ref[t + 1] = o.clone()
        refs[axis] = ref
        del S_ref
    hbm = measured_peaks()[0]

    def drift(out, r):
        num = (out - r).abs().amax(-1)
        den = r.abs().amax(-1).clamp_min(1e-30)
        e = (num / den).flatten()
        return {"mean": float(e.mean()), "max": float(e.max())}

    rows = []
    # the workload's column scales at every P, and row scales (one scale per
    # value channel, the group that holds the outlier channels) at P = 8
    runs = [(P, "col") for P in pace_synth.PERIOD_SWEEP] + [(8, "row")]
    for P, axis in runs:
        w = w0.replace(P=P, axis=axis)
        ref = refs[axis]
        pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, P, bits, axis=w.axis, io=w.io_dtype, device=dev)
        pool.load(S)
        dev_ev = [(mk(), mk()) for _ in range(T)]
        com_ev = [(mk(), mk()) for _ in range(T // P)]
        got = {}
        torch.cuda.synchronize()
        a, b = mk(), mk()
        a.record(stream)
        for t in range(T):
            x = toks[t]
            dev_ev[t][0].record(stream)
            pace.pace_decode_step(pool.handle, x["q"], x["k"], x["v"], x["alpha"], x["beta"], o, sp)
            dev_ev[t][1].record(stream)
            if t + 1 in horizons:
                got[t + 1] = o.clone()
            if (t + 1) % P == 0:
                c = com_ev[(t + 1) // P - 1]
                c[0].record(stream)
                pace.pace_commit_period(pool.handle, sp)
                c[1].record(stream)
        b.record(stream)
        torch.cuda.synchronize()
        status = pool.status()
        dec_ms = [e0.elapsed_time(e1) for e0, e1 in dev_ev]
        com_ms = [e0.elapsed_time(e1) for e0, e1 in com_ev]
        dec_bytes = [alg_bytes(w, bits, t % P + 1)[0] for t in range(T)]
        com_bytes = alg_bytes(w, bits, P)[1]
        kern_ms = sum(dec_ms) + sum(com_ms)
        dec_gbs = sum(dec_bytes) / (sum(dec_ms) * 1e-3) / 1e9
        com_gbs = com_bytes * len(com_ms) / (sum(com_ms) * 1e-3) / 1e9 if com_ms else None
        rows.append({
            "P": P, "axis": axis, "commit_engine": "tcgen05" if axis == "col" else "mma", "tokens": T,
            "value": BH * T / (kern_ms * 1e-3), "unit": "head-tokens/s",
            "ms_per_token": kern_ms / T,
            "wall_ms": a.elapsed_time(b),
            "decode": {"avg_ms": sum(dec_ms) / T, "achieved_gbs": dec_gbs, "frac_of_peak": dec_gbs / hbm},
            "commit": {"launches": len(com_ms), "avg_ms": sum(com_ms) / max(1, len(com_ms)),
                       "achieved_gbs": com_gbs, "frac_of_peak": com_gbs / hbm if com_gbs else None},
            "hbm_gbs_per_token": (sum(dec_bytes) + com_bytes * len(com_ms)) / (kern_ms * 1e-3) / 1e9,
            "drift": {str(h): drift(got[h], ref[h]) for h in horizons},
            "device_status": status,
        })
        del pool, got
    del toks, S, refs
    torch.cuda.synchronize()
    return {
        "workload": f"period_sweep: B={w0.B} H={w0.H} d_k={w0.d_k} d_v={w0.d_v}, all INT4, "
                    f"{w0.axis} scales at P in {list(pace_synth.PERIOD_SWEEP)} and row scales at P = 8, "
                    f"{w0.io_dtype} io, {w0.warmup}-token fp32 warm-up, {T} decode tokens",
        "state_bytes": state_bytes_of(w0, bits),
        "l2": "state pool 138 MB, near the 126 MB L2: no flush; part of the traffic is served from L2",
        "drift_metric": "per head ||o - o_fp32||_inf / ||o_fp32||_inf at token t (mean, max over heads); "
                        "o_fp32 from pace_gdn_step_f32 started at the encoded warm state (same scale axis), "
                        "dequantised",
        "time": "sum of per-launch CUDA-event durations (value); wall_ms includes the output copies "
                "taken at the horizons",
        "rows": rows,
    }


def gram_norm2(pool, w):
    """The accumulated-update norms^2 the tracking decode keeps in each head's
    factor block (float P*P + P of block [b][h] of the buffer's G region)."""
    import torch
    ru = lambda x, a: (x + a - 1) // a * a
    esz = 2 if w.io_dtype == "bf16" else 4
    BH, P = w.B * w.H, w.P
    ab_off = ru(BH * P * (w.d_k + w.d_v) * esz, 256)
    g_off = ru(ab_off + BH * ru(2 * P * esz, 16), 256)
    g_stride = ru(4 * (P * (P + 1) + 2), 16)
    g = pool.buffer[g_off:g_off + BH * g_stride].view(BH, g_stride).view(torch.float32)
    return g[:, P * P + P]


def run_adaptive(args, pace, pool, w, toks, outs, stream, world, dev, mk):
    import torch
    from bit_recurrent_state_pace_b200.ranks import aggregate_rate
    P, BH = w.P, w.B * w.H
    sp = stream.cuda_stream
    saved = pool.state.clone()
    torch.cuda.synchronize()
    assert int(pool.fill().count_nonzero()) == 0

    def restore():
        pool.state.copy_(saved)
        pool.fill().zero_()
        torch.cuda.synchronize()

    if args.commit_threshold == "auto":
        pool.set_commit_threshold(1e30)   # track, never mark
        for n in range(3):
            x = toks[n]
            pace.pace_decode_step(pool.handle, x["q"], x["k"], x["v"], x["alpha"], x["beta"], outs[n], sp)
        tau = float(torch.sqrt(torch.median(gram_norm2(pool, w))))
        rule = "median accumulated-update norm after 3 tokens"
        restore()
    else:
        tau, rule = float(args.commit_threshold), "given"
    pool.set_commit_threshold(tau)

    def token(n, ev=None):
        x = toks[n % P]
        if ev is not None:
            ev[0].record(stream)
        pace.pace_decode_step(pool.handle, x["q"], x["k"], x["v"], x["alpha"], x["beta"], outs[n % P], sp)
        if ev is not None:
            ev[1].record(stream)
        pace.pace_commit_period(pool.handle, sp)
        if ev is not None:
            ev[2].record(stream)

    for n in range(args.warmup * P):
        token(n)
    torch.cuda.synchronize()
    ntok = args.steps * P
    evs = [(mk(), mk(), mk()) for _ in range(ntok)]
    barrier(world)
    torch.cuda.synchronize()
    a, b = mk(), mk()
    a.record(stream)
    for n in range(ntok):
        token(n, evs[n])
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), world, dev)
    dec_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    com_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    # commits per head-token, counted outside the timed region
    commits = 0
    for n in range(2 * P):
        x = toks[n % P]
        pace.pace_decode_step(pool.handle, x["q"], x["k"], x["v"], x["alpha"], x["beta"], outs[n % P], sp)
        f = pool.fill()
        commits += int(((f & pace.PACE_FILL_COMMIT) != 0).sum() + (f == P).sum())
        pace.pace_commit_period(pool.handle, sp)
    status = pool.status()
    pool.set_commit_threshold(float("inf"))
    restore()
    return {"tau": tau, "tau_rule": rule, "value": aggregate_rate(BH * ntok, world, ms),
            "unit": "head-tokens/s", "ms_per_token": ms / ntok, "decode_ms": dec_ms,
            "commit_ms_per_launch": com_ms, "mean_tokens_per_commit": BH * 2 * P / max(commits, 1),
            "gpu_launches": 2 * ntok, "status": status}


def run_window(args, pace, pool, w, toks, outs, stream, world, dev, mk):
    """The pure-write window on a pool of its own whose buffer keeps the pairs
    as E4M3 bytes, starting from the main pool's stored state."""
    import torch
    from bit_recurrent_state_pace_b200.ranks import aggregate_rate
    P, BH = w.P, w.B * w.H
    win = pace.PacePool(w.B, w.H, w.d_k, w.d_v, P, pool.head_bits, axis=w.axis, io=w.io_dtype,
                        device=dev, buffer_e4m3=True)
    win.state.copy_(pool.state)
    torch.cuda.synchronize()

    def token(n):
        x = toks[n % P]
        win.window_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], outs[n % P], stream)

    for n in range(max(args.warmup, 1) * P):   # the window is full from here on
        token(n)
    torch.cuda.synchronize()
    ntok = args.steps * P
    barrier(world)
    torch.cuda.synchronize()
    a, b = mk(), mk()
    a.record(stream)
    for n in range(ntok):
        token(n)
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), world, dev)
    status = win.status()
    buffer_bytes = int(win.buffer.numel())
    del win
    return {"window": P, "value": aggregate_rate(BH * ntok, world, ms), "unit": "head-tokens/s",
            "ms_per_token": ms / ntok, "gpu_launches": 4 * ntok, "status": status,
            "buffer_bytes": buffer_bytes,
            "note": "pairs as E4M3 bytes; every token: the decode step, and the merge of each "
                    "head's oldest pair (one-token commit of every head, then the window shift)"}


def run_e2e(args, pace, pool, w, toks, outs, stream, world, dev, stag=None):
    """Same metric through the public API: every step copies its P tokens'
    inputs host->device from pinned memory and reads every output back.  In
    lockstep this is one pace_decode_host call per period (copies of token
    t+1 in and t-1 out overlap token t's kernels); the staggered schedule
    copies and computes token by token on one stream."""
    import torch
    P = w.P
    host_out = torch.empty((P,) + tuple(outs[0].shape), dtype=outs[0].dtype).pin_memory()
    if stag is None:
        host_in = {k: torch.stack([t[k].cpu() for t in toks]).contiguous().pin_memory() for k in toks[0]}
        h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    else:
        host_in = [{k: v.cpu().pin_memory() for k, v in t.items()} for t in toks]
        h2d = sum(v.numel() * v.element_size() for t in host_in for v in t.values())
    d2h = host_out.numel() * host_out.element_size()

    def step():
        if stag is None:
            pool.decode_host(host_in["q"], host_in["k"], host_in["v"], host_in["alpha"],
                             host_in["beta"], host_out, stream)
            return
        for n in range(P):
            for k, v in host_in[n].items():
                toks[n][k].copy_(v, non_blocking=True)
            stag.step(toks[n], outs[n], stream)
            host_out[n].copy_(outs[n], non_blocking=True)

    step()
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.e2e_steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), world, dev)
    from bit_recurrent_state_pace_b200.ranks import aggregate_rate
    return {"value": aggregate_rate(w.B * w.H * P * args.e2e_steps, world, ms),
            "unit": "head-tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
            # host-buffer decode is bound by the host link: the rates it reached
            "h2d_gbs": h2d * args.e2e_steps / ms / 1e6, "d2h_gbs": d2h * args.e2e_steps / ms / 1e6}


# ----------------------------------------------------------------------------- distributed plumbing

def barrier(world):
    from bit_recurrent_state_pace_b200.ranks import barrier as _barrier
    _barrier(world)


def max_over_ranks(x: float, world: int, dev):
    from bit_recurrent_state_pace_b200.ranks import max_over_ranks as _max
    return _max(x, world, dev)


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, rank, world)
        return
    import torch
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    try:
        run_pace(args, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
