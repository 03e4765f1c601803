#!/usr/bin/env python
"""Causal linear-attention forward throughput on B200 (Lightning Attention-2).

One step = one causal forward pass O = ((Q K^T) ⊙ M) V over one batch of the
workload (default: the long-context case B=1, H=8, N=524288, d=dv=128,
block 128, bf16 in/out, fp32 accumulation and state), through libla2's C ABI.
Prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--impl reference] [--sweep]

--sweep adds one line per other workload: B=4 H=16 N=2048, the sequence-length
sweep, the non-causal form, forward + backward and the decode step.

N > 1 is launched with torch.distributed.run: every rank runs the same
workload on its own GPU (independent (b, h) sequences, no data-path
collective; weak scaling) and rank 0 reports the aggregate.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 1024 * 1024
CLOCK_RAMP_S = 0.2
METRIC = "causal linear-attn fwd tokens/s (B·H·N/s), TFLOP/s, % of roofline, 1 B200"
FWDBWD_METRIC = "causal linear-attn fwd+bwd tokens/s (B·H·N/s), TFLOP/s, % of roofline, 1 B200"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="bf16_long_512k")
    ap.add_argument("--block", type=int, default=0, help="override the workload's block size")
    ap.add_argument("--N", type=int, default=0, help="override the sequence length")
    ap.add_argument("--causal", type=int, default=1, choices=[0, 1],
                    help="0: the non-causal form O = Q (K^T V) of the same workload")
    ap.add_argument("--impl", default="la2", choices=["la2", "reference"])
    ap.add_argument("--sweep", action="store_true",
                    help="also print one line per sequence-length sweep point, B4 H16 N2K, the 512K "
                         "case, fwd+bwd, the grouped-head and decayed workloads, the non-causal form "
                         "and the decode step")
    ap.add_argument("--decode", action="store_true",
                    help="also print the decode-step line (one RNN-mode token per sequence)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-every", type=int, default=10,
                    help="bracket the launches of every n-th timed step with per-kernel CUDA "
                         "events (1 = every step); the step time is measured over all steps "
                         "(an event pair between launches breaks their programmatic overlap: "
                         "every 4th step added ~5 %% to a 35 us step, every 10th ~1.5 %%)")
    ap.add_argument("--no-clocks", action="store_true",
                    help="skip nvidia-smi clock sampling (and its extra steps), e.g. under a profiler")
    return ap.parse_args()


# ------------------------------------------------------------------ helpers


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "linear_attention_la2_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    e = rec.get(f"{kernel}/{workload}")
    if not e or e.get("source_hash") != source_hash():
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def stop(self, t0=None, t1=None):
        """Stop sampling; summarise the samples taken between host times t0 and t1."""
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.t:
            self.t.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for t, ln in self.lines:
            if (t0 is not None and t < t0) or (t1 is not None and t > t1):
                continue
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def workload_from_args(args):
    from linear_attention_la2_b200 import inputs as I

    if args.workload in I.WORKLOADS:
        w = I.WORKLOADS[args.workload]
    elif args.workload in I.EXTRA_WORKLOADS:
        w = I.EXTRA_WORKLOADS[args.workload]
    elif args.workload.startswith("bf16_sweep_n"):
        n, b = args.workload[len("bf16_sweep_n"):].split("_b")
        w = I.sweep_workload(int(n), int(b))
    else:
        raise SystemExit(f"unknown workload {args.workload}")
    if args.block or args.N:
        from dataclasses import replace

        w = replace(w, block=args.block or w.block, N=args.N or w.N,
                    name=f"{w.name}_N{args.N or w.N}_b{args.block or w.block}")
    return w


def flops_per_token(w, causal=True):
    """Dense-tile flops per token·head of one step (the N^2 work LA2 avoids is
    not counted). Forward: S = Q K^T and P V inside a block (2 Bk d + 2 Bk dv),
    Q KV and the state update (2 d dv each); non-causal: K^T V and Q KV only.
    A forward + backward step adds the backward's 2 Bk (3d + 2dv) + 10 d dv
    (dP and S inside a block, the dQ, dK, dV products, two state updates)."""
    if not causal:
        f = 4 * w.d * w.dv
    else:
        f = 2 * w.block * (w.d + w.dv) + 4 * w.d * w.dv
    if w.backward:
        f += 2 * w.block * (3 * w.d + 2 * w.dv) + 10 * w.d * w.dv
    return f


def bytes_per_token(w):
    """HBM bytes per token·head each step must move at least: the forward reads
    Q, K, V and writes O; the backward reads Q, K, V, dO and writes dQ, dK, dV.
    With grouped K/V heads (G query heads a K/V head) the K/V side counts once
    per K/V head: 1/G per query token·head."""
    es = 2 if w.dtype == "bf16" else 4
    g = w.H // w.extra.get("Hkv", w.H)
    b = (w.d + w.dv) * es + (w.d + w.dv) * es / g
    if w.backward:
        b += (w.d + w.dv + w.d) * es + 2 * (w.d + w.dv) * es / g
    return b


# -------------------------------------------------------------- CPU oracle


# Sequences longer than this are timed in the oracle's RNN form over a prefix
# of one sequence (its left product is O(N^2) per sequence), plus the left
# product at sampled rows.
LEFT_PRODUCT_MAX_N = 16384
RNN_SAMPLE_TOKENS = 16384
ROW_SAMPLE = 64


def _oracle_cores():
    try:
        from threadpoolctl import threadpool_info

        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        return os.cpu_count() or 1


def oracle_sample_plan(w, causal=True):
    """What one bounded oracle sample of workload ``w`` computes: (form, tokens
    per sample, text). Whole (b, h) sequences with the float64 left product
    (and the closed-form backward for a forward + backward step) when one
    sequence costs about a second or less; else the float64 RNN form over the
    first RNN_SAMPLE_TOKENS tokens of a sequence."""
    if w.N <= LEFT_PRODUCT_MAX_N or not causal:
        what = "left product O=((QK^T)⊙M)V" if causal else "left product O=(QK^T)V"
        if w.backward:
            what += " + closed-form dQ, dK, dV"
        return "left", w.N, f"one whole (b,h) sequence of N={w.N}, float64 {what}"
    n = min(w.N, RNN_SAMPLE_TOKENS)
    return "rnn", n, (f"the first {n} tokens of one (b,h) sequence of N={w.N}, float64 RNN form "
                      "KV_t = KV_(t-1) + k_t^T v_t, o_t = q_t KV_t (the left product is "
                      "O(N^2) per sequence at this length)")


def oracle_sample(w, i, causal=True):
    """Run one bounded oracle sample (the ``i``-th; inputs drawn with the
    workload's recipe and seed ``w.seed + i``, outside the timing). Returns
    (tokens, seconds)."""
    import oracle
    from linear_attention_la2_b200 import inputs as I

    form, n, _ = oracle_sample_plan(w, causal)
    ins = I.make_custom(1, 1, n, w.d, w.dv, w.dtype, seed=w.seed + i, with_grad_out=w.backward)
    t0 = time.perf_counter()
    if form == "left":
        oracle.forward(ins["q"], ins["k"], ins["v"], causal)
        if w.backward:
            oracle.backward(ins["q"], ins["k"], ins["v"], ins["do"], causal)
    else:
        oracle.recurrent_forward(ins["q"], ins["k"], ins["v"])
    return n, time.perf_counter() - t0


def oracle_rows_rate(w, rows=ROW_SAMPLE):
    """Left product at ``rows`` sampled rows of one sequence of full length N
    (float64): output rows per second. The O(N^2) definition itself, where a
    whole sequence is out of reach."""
    import oracle
    from linear_attention_la2_b200 import inputs as I

    ins = I.make_custom(1, 1, w.N, w.d, w.dv, w.dtype, seed=w.seed)
    rr = I.sample_rows(w.N, w.block, w.seed, count=rows, max_blocks=2)[-rows:]
    t0 = time.perf_counter()
    oracle.forward_rows(ins["q"], ins["k"], ins["v"], rr, True)
    return len(rr) / (time.perf_counter() - t0), len(rr)


def cpu_oracle_rate(w, budget_s=10.0, causal=True):
    """The oracle as it stands, timed on the host cores: one untimed warm-up
    sample, then samples (oracle_sample) until about ``budget_s`` seconds.
    The reference arm times the same samples, one per step."""
    _, _, text = oracle_sample_plan(w, causal)
    oracle_sample(w, 0, causal)
    tokens, elapsed, k = 0, 0.0, 0
    while k == 0 or (elapsed < budget_s and k < 64):
        n, t = oracle_sample(w, k + 1, causal)
        tokens += n
        elapsed += t
        k += 1
    rec = {"value": tokens / elapsed, "unit": "tokens/s", "cores": _oracle_cores(), "kind": "oracle",
           "sample": f"{k} samples, each {text}; {elapsed:.1f} s"}
    if oracle_sample_plan(w, causal)[0] == "rnn":
        rate, nrows = oracle_rows_rate(w)
        rec["left_product_rows_per_s"] = rate
        rec["left_product_sample"] = (f"{nrows} sampled rows of one sequence of N={w.N}, float64 "
                                      "left product (output rows/s; a full sequence needs N rows)")
    return rec


def run_reference(args):
    """--impl reference: the oracle on the host cores, same metric and config;
    each step is one bounded sample of the workload (oracle_sample)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = workload_from_args(args)
    causal = bool(args.causal)
    _, _, text = oracle_sample_plan(w, causal)
    total, tokens = 0.0, 0
    for i in range(args.warmup + args.steps):
        n, t = oracle_sample(w, i, causal)
        if i >= args.warmup:
            total += t
            tokens += n
    value = tokens / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, causal),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": _oracle_cores(),
                         "kind": "oracle", "sample": f"each step: {text}, on host cores"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    if w.backward:
        line["metric"] = FWDBWD_METRIC
    print(json.dumps(line))
    return 0


def config_of(w, causal=True):
    kind = "causal" if causal else "non-causal"
    if "decay" in w.extra:
        kind = f"decayed causal (lambda={w.extra['decay']} every head)"
    heads = f"H={w.H} Hkv={w.extra['Hkv']}" if "Hkv" in w.extra else f"H={w.H}"
    c = {"workload": f"{w.name}: {kind} forward B={w.B} {heads} "
                     f"N={w.N} d={w.d} dv={w.dv} block={w.block} {w.dtype}", "B": w.B, "H": w.H,
         "N": w.N, "d": w.d, "dv": w.dv, "block": w.block, "causal": causal}
    c.update(w.extra)
    return c


# ------------------------------------------------------------------- GPU


def run_gpu(args):
    import torch
    import torch.distributed as dist

    from linear_attention_la2_b200 import inputs as I

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    from linear_attention_la2_b200 import la2

    w = workload_from_args(args)
    hbm, tf_burst, tf_sust, peak_kind = peaks()

    line = bench_workload(args, w, dev, la2, world, rank, local, hbm, peak_kind, main=True,
                          causal=bool(args.causal))
    if rank == 0:
        print(json.dumps(line), flush=True)
    if args.sweep:
        others = [I.WORKLOADS["bf16_b4h16_n2k"]]
        others += [I.sweep_workload(N, b) for N in I.SWEEP_N for b in I.SWEEP_BLOCKS]
        others += [I.WORKLOADS["bf16_long_512k"], I.WORKLOADS["bf16_fwdbwd_b2h32_n8k"]]
        others += list(I.EXTRA_WORKLOADS.values())
        for sw in others:
            if sw.name == w.name:
                continue
            ln = bench_workload(args, sw, dev, la2, world, rank, local, hbm, peak_kind, main=False)
            if rank == 0:
                print(json.dumps(ln), flush=True)
        nc = I.WORKLOADS["bf16_b4h16_n2k"]
        ln = bench_workload(args, nc, dev, la2, world, rank, local, hbm, peak_kind, main=False,
                            causal=False)
        if rank == 0:
            print(json.dumps(ln), flush=True)
    if args.sweep or args.decode:
        ln = bench_decode(args, dev, la2, world, hbm, peak_kind)
        if rank == 0:
            print(json.dumps(ln), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def whole_job_rate(units_per_rank, steps, world, ms_max):
    """Units all ranks processed per second, timed by the slowest rank."""
    return units_per_rank * steps * world / (ms_max / 1e3)


def _max_over_ranks(x, world, dev):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def bench_workload(args, w, dev, la2, world, rank, local, hbm, peak_kind, main, causal=True):
    import torch

    from linear_attention_la2_b200 import inputs as I

    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    Hkv = w.extra.get("Hkv", w.H)
    decay = w.extra.get("decay")
    rates = torch.full((w.H,), float(decay), dtype=torch.float32, device=dev) if decay is not None else None
    set_bytes = w.tokens * bytes_per_token(w)
    nsets = max(1, math.ceil(3 * L2_BYTES / set_bytes)) if set_bytes < 3 * L2_BYTES else 1
    nsets = min(nsets, 8)
    base = I.make_inputs(w, device="cpu")
    sets = []
    for s in range(nsets):
        q = base["q"].to(dev)
        k = base["k"].to(dev)
        v = base["v"].to(dev)
        if s > 0:  # distinct buffers, same values
            pass
        o = torch.empty((w.B, w.H, w.N, w.dv), dtype=w.torch_dtype, device=dev)
        if Hkv < w.H:  # grouped K/V heads: the first Hkv heads of the draw
            k, v = k[:, :Hkv].contiguous(), v[:, :Hkv].contiguous()
        sets.append((q, k, v, o))
    dt = la2.LA2_BF16 if w.dtype == "bf16" else la2.LA2_F32

    def ws_size(bwd):
        if decay is not None:
            return la2.workspace_bytes_decay(w.B, w.H, w.N, w.d, w.dv, w.block, dt, bwd)
        return la2.workspace_bytes_gqa(w.B, w.H, Hkv, w.N, w.d, w.dv, causal, w.block, dt, bwd)

    ws_bytes = ws_size(False)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    st = la2._stream_handle(stream)

    if w.backward:  # one step = forward + backward of the same batch
        dO = I.make_inputs(w, with_grad_out=True)["do"].to(dev)
        grads = (torch.empty_like(sets[0][0]), torch.empty_like(sets[0][1]), torch.empty_like(sets[0][2]))
        wsb_bytes = ws_size(True)
        wsb = torch.empty(max(wsb_bytes, 1), dtype=torch.uint8, device=dev)

    def step(i):
        q, k, v, o = sets[i % nsets]
        if decay is not None:
            rc = la2.la2_forward_decay(la2._ptr(q), la2._ptr(k), la2._ptr(v), la2._ptr(o),
                                       la2._ptr(rates), w.B, w.H, w.N, w.d, w.dv, w.block, dt,
                                       la2._ptr(ws), ws_bytes, st)
        else:
            rc = la2.la2_forward_gqa(la2._ptr(q), la2._ptr(k), la2._ptr(v), la2._ptr(o), w.B, w.H,
                                     Hkv, w.N, w.d, w.dv, int(causal), w.block, dt, la2._ptr(ws),
                                     ws_bytes, st)
        if rc != 0:
            raise la2.La2Error(rc)
        if w.backward:
            g = (la2._ptr(grads[0]), la2._ptr(grads[1]), la2._ptr(grads[2]))
            if decay is not None:
                rc = la2.la2_backward_decay(la2._ptr(q), la2._ptr(k), la2._ptr(v), la2._ptr(dO), *g,
                                            la2._ptr(rates), w.B, w.H, w.N, w.d, w.dv, w.block, dt,
                                            la2._ptr(wsb), wsb_bytes, st)
            else:
                rc = la2.la2_backward_gqa(la2._ptr(q), la2._ptr(k), la2._ptr(v), la2._ptr(dO), *g,
                                          w.B, w.H, Hkv, w.N, w.d, w.dv, 1, w.block, dt,
                                          la2._ptr(wsb), wsb_bytes, st)
            if rc != 0:
                raise la2.La2Error(rc)

    for i in range(args.warmup):
        step(i)
    la2.check(stream)

    sampler = ClockSampler(local) if main and not args.no_clocks else None
    every = max(1, args.profile_every)
    if sampler:
        sampler.start()
    # Clock ramp: after the requested warm-up, keep the same workload running
    # (untimed) for CLOCK_RAMP_S so the timed region does not start at the
    # clocks of an idle GPU (input preparation leaves it idle for seconds).
    ramp_steps = 0
    tr0 = time.monotonic()
    while time.monotonic() - tr0 < CLOCK_RAMP_S:
        step(args.warmup + ramp_steps)
        ramp_steps += 1
    _barrier(world)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    th0 = time.monotonic()
    la2.la2_profile_enable(1)  # clear the records ...
    la2.la2_profile_enable(0)  # ... and record only the sampled steps
    e0.record(stream)
    profiled_steps = 0
    for i in range(args.steps):
        # per-kernel events around the launches of every `every`-th step only:
        # an event pair per launch also costs device time between kernels
        prof = i % every == 0
        if prof:
            la2.la2_profile_enable(2)
            profiled_steps += 1
        step(i)
        if prof:
            la2.la2_profile_enable(0)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    th1 = time.monotonic()
    la2.la2_profile_enable(0)
    clocks = None
    if sampler:
        if th1 - th0 >= 1.0:
            clocks = sampler.stop(th0, th1)
            if clocks:
                clocks["window"] = "timed region"
        else:
            # nvidia-smi samples every 100 ms: keep the same workload running
            # (unprofiled, untimed) for about a second and sample there.
            tw0 = time.monotonic()
            n = 0
            while time.monotonic() - tw0 < 1.2:
                step(args.steps + n)
                n += 1
            torch.cuda.synchronize(dev)
            tw1 = time.monotonic()
            clocks = sampler.stop(tw0 + 0.1, tw1)
            if clocks:
                clocks["window"] = (f"{n} further steps of the same workload right after the timed "
                                    f"region ({tw1 - tw0:.1f} s; the timed region lasted "
                                    f"{1e3 * (th1 - th0):.1f} ms)")
    _barrier(world)
    la2.check(stream)
    ms = e0.elapsed_time(e1)
    ms_max = _max_over_ranks(ms, world, dev)

    per_kernel = {}
    launches = 0
    for kid in range(la2.la2_profile_num_kernels()):
        n, kms = la2.la2_profile_collect(kid)
        if n:
            per_kernel[la2.la2_profile_kernel_name(kid)] = {"launches": n, "ms": kms}
            launches += n
    # every step launches the same kernels: scale the timed sample to all steps
    launches = launches * args.steps // max(1, profiled_steps)
    value = whole_job_rate(w.tokens, args.steps, world, ms_max)
    tflops = flops_per_token(w, causal) * value / 1e12
    roofline = op_roofline(w, per_kernel, profiled_steps, hbm, peak_kind, causal)
    step_frac = (w.tokens * bytes_per_token(w) * args.steps * world / (ms_max / 1e3) / 1e9) / (hbm * world)

    line = {
        "metric": METRIC if causal else METRIC.replace("causal", "non-causal", 1), "value": value,
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic", "config": dict(config_of(w, causal), l2=(
            f"{nsets} rotating input sets of {set_bytes / 1e6:.0f} MB (> L2 126 MB)" if nsets > 1
            else f"inputs {set_bytes / 1e6:.0f} MB > L2"), parallelism=f"dp{world} (independent "
            "(b,h) sequences per rank)"),
        "tflops": tflops, "step_roofline_frac": step_frac, "roofline": roofline,
        "gpu_launches": launches, "kernels": per_kernel,
        "kernel_timing": (f"CUDA events around each launch of {profiled_steps} of the "
                          f"{args.steps} timed steps (every {every}th step)"),
        "clock_ramp": f"{ramp_steps} untimed steps ({CLOCK_RAMP_S} s) after the {args.warmup} "
                      "warm-up steps",
    }
    if clocks:
        line["clocks"] = clocks
    if w.backward:
        line["metric"] = FWDBWD_METRIC
        line["config"]["workload"] += " (+ backward)"
    # (the e2e leg and the CPU oracle time the plain op: not for the follow-on workloads)
    if main and not args.no_e2e and not w.backward and not w.extra:
        line["e2e"] = e2e_measure(args, w, dev, la2, world, base, ws, ws_bytes, dt, causal)
    if main and rank == 0 and world == 1 and not args.no_cpu_baseline and not w.extra:
        line["cpu_baseline"] = cpu_oracle_rate(w, budget_s=10.0, causal=causal)
    return line


def op_roofline(w, per_kernel, profiled_steps, hbm, peak_kind, causal=True):
    """Roofline of the whole op: the algorithmic bytes of one step over the
    summed device time of every launch of that step (CUDA events around each
    launch on the launching stream). Per kernel: launches and time per step,
    and its share of the step's kernel time. ``traffic`` is the summed DRAM
    bytes (ncu) of one step's launches when every kernel of the step has a
    capture taken on the current sources, else None."""
    if not per_kernel or profiled_steps < 1:
        return None
    step_ms = sum(v["ms"] for v in per_kernel.values()) / profiled_steps
    alg_bytes = w.tokens * bytes_per_token(w)
    achieved = alg_bytes / (step_ms / 1e3) / 1e9
    kernels, traffic = {}, 0
    tag = w.name if causal else w.name + "_noncausal"
    for name, v in per_kernel.items():
        launches = v["launches"] / profiled_steps
        kernels[name] = {"launches_per_step": launches, "ms_per_step": v["ms"] / profiled_steps,
                         "share": v["ms"] / profiled_steps / step_ms}
        rec = recorded_traffic(name, tag)
        traffic = None if (traffic is None or rec is None) else traffic + rec * launches
    dom = max(kernels, key=lambda k: kernels[k]["ms_per_step"])
    return {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
            "traffic": traffic, "alg_bytes_per_step": alg_bytes, "scope": "op",
            "kernel": dom, "kernels": kernels,
            "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)" if peak_kind == "measured"
            else "fallback 6.65 TB/s"}


DECODE = dict(name="bf16_decode_b64h32", B=64, H=32, d=128, dv=128, seed=5)


def bench_decode(args, dev, la2, world, hbm, peak_kind):
    """One step = one new token for each of the B*H sequences through
    la2_decode_step (state += k^T v, o = q state) on a [B,H,d,dv] fp32 state that
    is larger than L2; q, k, v rotate over 8 sets."""
    import torch

    c = DECODE
    B, H, d, dv = c["B"], c["H"], c["d"], c["dv"]
    g = torch.Generator().manual_seed(c["seed"])
    sets = [tuple((torch.randn((B, H, n), generator=g) / math.sqrt(d)).to(torch.bfloat16).to(dev)
                  for n in (d, d, dv)) for _ in range(8)]
    state = (torch.randn((B, H, d, dv), generator=g) * 0.01).to(dev)
    o = torch.empty((B, H, dv), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    st = la2._stream_handle(stream)

    def step(i):
        q, k, v = sets[i % len(sets)]
        rc = la2.la2_decode_step(la2._ptr(q), la2._ptr(k), la2._ptr(v), la2._ptr(o),
                                 la2._ptr(state), B, H, d, dv, la2.LA2_BF16, st)
        if rc != 0:
            raise la2.La2Error(rc)

    for i in range(args.warmup):
        step(i)
    la2.check(stream)
    every = max(1, args.profile_every)
    _barrier(world)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    la2.la2_profile_enable(1)
    la2.la2_profile_enable(0)
    e0.record(stream)
    profiled_steps = 0
    for i in range(args.steps):
        prof = i % every == 0
        if prof:
            la2.la2_profile_enable(2)
            profiled_steps += 1
        step(i)
        if prof:
            la2.la2_profile_enable(0)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    la2.la2_profile_enable(0)
    _barrier(world)
    la2.check(stream)
    ms_max = _max_over_ranks(e0.elapsed_time(e1), world, dev)
    per_kernel = {}
    for kid in range(la2.la2_profile_num_kernels()):
        n, kms = la2.la2_profile_collect(kid)
        if n:
            per_kernel[la2.la2_profile_kernel_name(kid)] = {"launches": n, "ms": kms}
    k_ms = per_kernel["la2_decode_step"]["ms"] / per_kernel["la2_decode_step"]["launches"]
    bytes_step = B * H * (2 * d * dv * 4 + (2 * d + 2 * dv) * 2)
    achieved = bytes_step / (k_ms / 1e3) / 1e9
    return {
        "metric": "decode tokens/s (one RNN-mode token per (b,h) sequence), 1 B200",
        "value": whole_job_rate(B * H, args.steps, world, ms_max), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{c['name']}: decode step B={B} H={H} d={d} dv={dv} bf16 q/k/v/o, "
                               "fp32 state", "B": B, "H": H, "d": d, "dv": dv,
                   "l2": f"state {B * H * d * dv * 4 / 1e6:.0f} MB > L2"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": recorded_traffic("la2_decode_step", c["name"]),
                     "kernel": "la2_decode_step",
                     "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)"},
        "gpu_launches": sum(v["launches"] for v in per_kernel.values()) * args.steps
        // max(1, profiled_steps), "kernels": per_kernel,
        "kernel_timing": (f"CUDA events around each launch of {profiled_steps} of the "
                          f"{args.steps} timed steps (every {every}th step)"),
    }


def e2e_measure(args, w, dev, la2, world, base, ws, ws_bytes, dt, causal=True):
    """Same metric through the public binding with host buffers: every step copies
    Q, K, V from pinned host memory, runs the forward and reads O back."""
    import torch

    stream = torch.cuda.current_stream(dev)
    hq, hk, hv = (base[n].pin_memory() for n in "qkv")
    ho = torch.empty((w.B, w.H, w.N, w.dv), dtype=w.torch_dtype).pin_memory()
    dq = torch.empty_like(hq, device=dev)
    dk = torch.empty_like(hk, device=dev)
    dvv = torch.empty_like(hv, device=dev)
    do = torch.empty_like(ho, device=dev)

    def step():
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dvv.copy_(hv, non_blocking=True)
        la2.forward(dq, dk, dvv, causal=causal, block=w.block, out=do, workspace=ws if ws_bytes else None)
        ho.copy_(do, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        step()
    _barrier(world)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = _max_over_ranks(e0.elapsed_time(e1), world, dev)
    h2d = (hq.numel() + hk.numel() + hv.numel()) * hq.element_size()
    d2h = ho.numel() * ho.element_size()
    return {"value": whole_job_rate(w.tokens, args.steps, world, ms), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
