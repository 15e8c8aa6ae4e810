#!/usr/bin/env python
"""Benchmark of the SFA operator: prefill + decode tokens/s on B200.

One step is one pass of the whole hot path over one batch of synthetic
input; a token is one sequence position through all layers.  Three kinds of
step, chosen by the workload:

  * decode only (batched_decode, the default, and the k x gamma_far x alpha
    sweep points): the prompt is prefilled once, untimed; a step is the
    workload's decode steps over all layers and sequences (each decode call
    moves more than the L2, so nothing is flushed).
  * prefill only (long_prefill): state reset and one prefill of the batch;
    L2 is flushed (256 MB write) before every timed step, outside its events.
  * prefill + decode (tiny, qwen05b, qwen7b_decode): state reset, prefill of
    the prompt, then the decode steps, every layer and sequence; L2 flushed
    as for prefill.

Default line: the batched decode of the Qwen2.5-7B attention shape (28
layers, 28 query / 4 KV heads, head_dim 128, 256 sequences, k = 16, 1,024
prefilled tokens, 512 timed decode steps, Student-t inputs in bf16) is the
headline; the same run adds one object each for the long prefill (4 x 65,536
tokens of one 7B-shaped layer), the Qwen2.5-0.5B step (512 + 128 tokens, 24
layers, batch 1) and the decode time after 1K / 4K / 8K-token prompts
(context flatness), each with its own roofline fraction.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload NAME] [--context N] [--no-extras]

N > 1 runs under torch.distributed.run as independent replicas (the
operator has no cross-stream exchange), timed per rank and reduced with MAX.
``--impl reference`` times the fp64 oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import contextlib
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "SFA prefill & decode tokens/s on 1 B200; achieved HBM GB/s vs ~8 TB/s peak"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_HBM_GBS = 6650.0
HEADLINE = "batched_decode"  # default workload of the bench line
EXTRAS = ("long_prefill", "qwen05b")  # timed in the same run, each in its own object
CONTEXTS = (1024, 4096, 8192)  # context-flatness object: decode after these prompt lengths


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=HEADLINE)
    ap.add_argument("--no-extras", action="store_true",
                    help="time the headline workload only (no long_prefill, qwen05b and "
                         "context-flatness objects)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--context", type=int, default=0,
                    help="prompt length (default: the workload's first prefill length)")
    ap.add_argument("--report", choices=["context", "enhancement"], default=None,
                    help="instead of the bench line: state footprint and decode time against "
                         "the context, or the enhancement share and its angle to x")
    ap.add_argument("--max-context", type=int, default=65536)
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (smaller cases for profiling)")
    ap.add_argument("--layers", type=int, default=0,
                    help="override the workload's layer count (smaller cases for profiling)")
    return ap.parse_args()


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


@contextlib.contextmanager
def nvtx_range(name: str):
    """NVTX range around a phase of the bench, for Nsight timelines; a no-op
    where NVTX is unavailable."""
    pushed = False
    try:
        import torch
        torch.cuda.nvtx.range_push(name)
        pushed = True
    except Exception:
        pass
    try:
        yield
    finally:
        if pushed:
            try:
                torch.cuda.nvtx.range_pop()
            except Exception:
                pass


def max_over_ranks(values, world, device):
    """Per-rank times (ms) reduced with MAX over the ranks, so the slowest
    replica sets the job's time; every rank receives the result."""
    import torch
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_rate(world, units_per_rank, ms):
    """Whole-job throughput: the units all `world` replicas processed (each
    the same amount) over the max-over-ranks time in ms."""
    return world * units_per_rank / (ms / 1e3)


def step_medians(pre_ms, dec_ms):
    """Median over the timed steps of this rank's per-step times (ms): the
    whole step, its prefill part and its decode part."""
    tot = [a + b for a, b in zip(pre_ms, dec_ms)]
    return {"step_ms": statistics.median(tot), "prefill_ms": statistics.median(pre_ms),
            "decode_ms": statistics.median(dec_ms), "steps": len(tot)}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernels_per_call(w, n_pre, n_sm):
    """(prefill, decode) kernels the library launches per call for workload
    w, following its routing: decode calls of 64 or more sequences (at most
    8 query heads per KV head, hidden a multiple of 64) launch the near-field
    and pool kernels, smaller ones the batch-1 kernel; a prefill launches the
    two far-field kernels and the output kernel, plus the fused kernel (bf16,
    k <= 16, at least 4 tiles per SM) or a near-field and a pool kernel."""
    G = w.n_q_heads // w.n_kv_heads
    tiled = w.batch >= 64 and w.window_k <= 256 and G <= 8 and w.hidden % 64 == 0
    tiles = w.n_layers * w.batch * ((max(n_pre, 1) + 63) // 64)
    fused = w.in_dtype == "bf16" and w.window_k <= 16 and tiles >= 4 * n_sm
    return (4 if fused else 5), (2 if tiled else 1)


def workload_bytes(w, n_pre=None):
    """Algorithmic bytes (what the method must move; no re-reads).

    decode launch: per (layer, sequence) q (e*H), out (4H), ring slot read +
    write (8H), ring sum r/w (8H), field r/w (8H), new K/V read and window
    write (4e*nkv*d), window read (2k*e*nkv*d), S r/w (8*nkv*d); per layer the
    64 x H fp32 slots (256H).
    prefill call of n tokens: per token-layer q, k, v read and out write
    (e*H + 2e*nkv*d + 4H); per stream the final state write; per layer slots.
    """
    e = 4 if w.in_dtype == "f32" else 2
    H, S, k = w.hidden, w.n_kv_heads * w.head_dim, w.window_k
    per_seq_layer = (28 + e) * H + (4 * e + 8 + 2 * k * e) * S
    decode = w.n_layers * (w.batch * per_seq_layer + 256 * H)
    n = w.prefill_n[0] if n_pre is None else n_pre
    state_write = 2 * k * S * e + 4 * S + 72 * H
    prefill = (w.n_layers * w.batch * (n * (e * H + 2 * e * S + 4 * H) + state_write)
               + w.n_layers * 256 * H)
    return decode, prefill


class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_index_for(device) -> str:
    import torch
    try:
        uuid = str(torch.cuda.get_device_properties(device).uuid)
        out = subprocess.run(["nvidia-smi", "--query-gpu=index,uuid", "--format=csv,noheader"],
                             capture_output=True, text=True, timeout=20).stdout
        for line in out.splitlines():
            idx, u = [s.strip() for s in line.split(",")]
            if uuid in u or u.endswith(uuid):
                return idx
    except Exception:
        pass
    return os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[0] or "0"


def kernel_traffic(kernel_src: str, name: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, only if it was
    taken on the current kernel source (matching sha256) and workload."""
    path = os.path.join(ROOT, "profiles", f"{name}_traffic_{workload}.json")
    try:
        with open(path) as f:
            d = json.load(f)
        sha = hashlib.sha256(open(kernel_src, "rb").read()).hexdigest()
        if d.get("kernel_sha256") == sha:
            return float(d["dram_bytes_per_launch"]), d.get("workload")
    except Exception:
        pass
    return None, None


# ------------------------------------------------------------------ oracle


def sample_streams(w):
    """The (layer, sequence) streams the oracle times: first, middle and last
    layer and sequence (for the batched-decode sweep: layers 0, 14, 27 x
    sequences 0, 128, 255)."""
    pick = lambda n: sorted({0, n // 2, n - 1})
    return pick(w.n_layers), pick(w.batch)


def oracle_inputs(w, layers, seqs, n_tokens, dev):
    """q, k, v of the chosen streams for positions 0 .. n_tokens-1, float32
    numpy [len(layers), len(seqs), n, heads, d].  Drawn with the workload's
    own generator on `dev` (the bench's GPU when there is one, so the oracle
    sees exactly the values the GPU arm uses) one token block at a time, and
    only the chosen streams are copied to the host."""
    import torch
    from workloads import TOKEN_BLOCK, TokenSource
    src = TokenSource(w, dev)
    li = torch.tensor(layers, device=dev)
    si = torch.tensor(seqs, device=dev)
    parts = ([], [], [])
    for t0 in range(0, n_tokens, TOKEN_BLOCK):
        blk = src.get(t0, min(n_tokens, t0 + TOKEN_BLOCK))
        for i, x in enumerate(blk):
            parts[i].append(x.index_select(0, li).index_select(1, si).float().cpu())
        del blk
    return tuple(torch.cat(p, dim=2).numpy() for p in parts)


def oracle_tokens_per_s(w, layers, seqs, qn, kn, vn, slots_np):
    """Times the fp64 oracle from position 0 on the streams layers x seqs
    (inputs from oracle_inputs); returns (tokens/s as positions through all
    layers, threads used, seconds)."""
    import numpy as np
    import oracle
    f = lambda x: float(np.float32(x))
    v = w.values
    p = oracle.OracleParams(w.n_q_heads, w.n_kv_heads, w.head_dim, w.window_k,
                            gamma_far=f(v.gamma_far), alpha_far=f(v.alpha_far))
    pairs = [(a, b) for a in range(len(layers)) for b in range(len(seqs))]
    n = qn.shape[2]
    alpha = [oracle.alpha_layer(f(v.alpha_base), f(v.cross_decay), layers[a], w.n_layers)
             for a, _ in pairs]
    sl = np.stack([slots_np[layers[a]] for a, _ in pairs]).astype(np.float32)
    qq = np.stack([qn[a, b] for a, b in pairs])
    kk = np.stack([kn[a, b] for a, b in pairs])
    vv = np.stack([vn[a, b] for a, b in pairs])
    st = oracle.OracleState(p, len(pairs))
    t0 = time.perf_counter()
    _, used = oracle.run_streams(p, alpha, sl, qq, kk, vv, st)
    dt = time.perf_counter() - t0
    tokens = len(pairs) * n / w.n_layers  # positions through all layers
    return tokens / dt, used, dt


def input_device():
    """Where inputs for the oracle are drawn: the GPU when present."""
    import torch
    return torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")


def run_reference(args, w, n_pre):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from workloads import make_slots
    dev = input_device()
    slots_np = make_slots(w, dev).cpu().numpy()
    n_tok = 64  # bounded sample per step: one layer, a few sequences, 64 positions
    seqs = list(range(min(w.batch, 4)))
    steps = [s % w.n_layers for s in range(args.steps)]
    inputs = {l: oracle_inputs(w, [l], seqs, n_tok, dev) for l in sorted(set(steps) | {0})}
    for _ in range(args.warmup):
        oracle_tokens_per_s(w, [0], seqs, *inputs[0], slots_np)
    times, used = [], 1
    for l in steps:
        _, used, dt = oracle_tokens_per_s(w, [l], seqs, *inputs[l], slots_np)
        times.append(dt)
    total = sum(times)
    tokens = args.steps * len(seqs) * n_tok / w.n_layers
    value = tokens / total
    sample = (f"per step: 1 layer x {len(seqs)} seq x {n_tok} positions of the {w.name} "
              f"workload, scaled to positions through all {w.n_layers} layers")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, n_pre),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": used, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def step_kind(w) -> str:
    if w.decode_steps == 0:
        return "prefill"
    if w.batch >= 64:
        return "decode"
    return "step"


def workload_config(w, n_pre=None):
    n_pre = w.prefill_n[0] if n_pre is None else n_pre
    kind = step_kind(w)
    if kind == "decode":
        what = (f"prefill {n_pre} (untimed) then {w.decode_steps} decode steps")
        l2 = "not flushed: every decode call moves more bytes than the 126 MB L2"
    elif kind == "prefill":
        what = f"prefill {n_pre}"
        l2 = "flushed before every timed step (256 MB write); inputs exceed L2"
    else:
        what = f"prefill {n_pre} + {w.decode_steps} decode steps"
        l2 = "flushed before every timed step (256 MB write)"
    return {
        "workload": (f"{w.name}: {w.n_layers} layers, {w.n_q_heads}q/{w.n_kv_heads}kv heads, "
                     f"head_dim {w.head_dim}, batch {w.batch}, {what}, k={w.window_k}"),
        "global_batch": w.batch, "seq_len": n_pre + w.decode_steps,
        "in_dtype": w.in_dtype, "window_k": w.window_k, "step": kind,
        "l2": l2, "parallelism": "replicas",
    }


def sfa_config_for(sfa, w):
    v = w.values
    return sfa.SfaConfig(n_layers=w.n_layers, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                         head_dim=w.head_dim, window_k=w.window_k, gamma_far=v.gamma_far,
                         alpha_far=v.alpha_far, ema_gamma=v.ema_gamma, temperature=v.temperature,
                         clip_eps=v.clip_eps, alpha_base=v.alpha_base, cross_decay=v.cross_decay,
                         in_dtype=sfa.SFA_F32 if w.in_dtype == "f32" else sfa.SFA_BF16)


# ------------------------------------------------------------------ ours


DECODE_RING = 64  # distinct decode inputs cycled by the decode-only step


class Run:
    """One workload's operator, inputs and captured CUDA graphs.

    ``one_step(ev)`` replays one step (prefill part a, decode part b); with
    ``ev`` it records three events around the parts."""

    def __init__(self, w, n_pre, dev, rank, sfa):
        import torch
        from workloads import TokenSource, make_slots
        self.w, self.n_pre = w, n_pre
        self.kind = kind = step_kind(w)
        n_dec = w.decode_steps
        L, B, H = w.n_layers, w.batch, w.hidden
        src = TokenSource(w, dev, salt=rank)
        slots = make_slots(w, dev)
        chunk = 128 if kind == "decode" else n_pre
        op = sfa.SfaOperator(sfa_config_for(sfa, w), slots, B, max_prefill=chunk, device=dev)
        self.op = op
        # Every decode input is complete before its call: the timed steps
        # replay inputs written before the timed region, and the e2e steps copy
        # them in with cudaMemcpyAsync ordered by events.  So the decode kernel
        # may fetch them before the previous kernel on the stream ends.
        sfa.sfa_set_decode_input_prefetch(op.handle, True)
        self.flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.qp = self.kp = self.vp = None
        if kind == "decode":
            # untimed prompt, in chunks; then a ring of distinct decode inputs
            n_ring = min(DECODE_RING, n_dec)
            out_c = torch.empty((L, B, chunk, H), dtype=torch.float32, device=dev)
            for t0 in range(0, n_pre, chunk):
                q, k, v = src.get(t0, min(n_pre, t0 + chunk))
                op.prefill(q, k, v, out=out_c[:, :, :q.shape[2]])
                del q, k, v
            del out_c
            qa, ka, va = src.get(n_pre, n_pre + n_ring)
            qd = [qa[:, :, t].contiguous() for t in range(n_ring)]
            kd = [ka[:, :, t].contiguous() for t in range(n_ring)]
            vd = [va[:, :, t].contiguous() for t in range(n_ring)]
            del qa, ka, va
            out_d = torch.empty((n_ring, L, B, H), dtype=torch.float32, device=dev)
            self.replays = max(1, n_dec // n_ring)
            self.n_dec = self.replays * n_ring

            def part_a():
                pass

            def part_b():
                for t in range(n_ring):
                    op.decode(qd[t], kd[t], vd[t], out=out_d[t])
        else:
            qp, kp, vp = src.get(0, n_pre)
            self.qp, self.kp, self.vp = qp, kp, vp
            qa, ka, va = src.get(n_pre, n_pre + n_dec)
            qd = [qa[:, :, t].contiguous() for t in range(n_dec)]
            kd = [ka[:, :, t].contiguous() for t in range(n_dec)]
            vd = [va[:, :, t].contiguous() for t in range(n_dec)]
            del qa, ka, va
            out_p = torch.empty((L, B, n_pre, H), dtype=torch.float32, device=dev)
            out_d = torch.empty((n_dec, L, B, H), dtype=torch.float32, device=dev)
            self.replays = 1
            self.n_dec = n_dec

            def part_a():
                op.reset()
                op.prefill(qp, kp, vp, out=out_p)

            def part_b():
                for t in range(n_dec):
                    op.decode(qd[t], kd[t], vd[t], out=out_d[t])
        self.qd, self.kd, self.vd = qd, kd, vd
        del src

        # eager warm-up, then capture both halves as CUDA graphs
        part_a()
        part_b()
        torch.cuda.synchronize()
        rc = op.check()
        if rc != 0:
            raise SystemExit(f"{w.name}: device error during warm-up: {sfa.sfa_status_string(rc)}")
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        self.g_a, self.g_b = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        self.has_a, self.has_b = kind != "decode", kind != "prefill"
        with torch.cuda.stream(side):
            if self.has_a:
                with torch.cuda.graph(self.g_a, stream=side):
                    part_a()
            if self.has_b:
                with torch.cuda.graph(self.g_b, stream=side):
                    part_b()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        self.flush_each = kind != "decode"
        pre_k, dec_k = kernels_per_call(w, n_pre, torch.cuda.get_device_properties(dev).multi_processor_count)
        # our kernels per step: the state header write and the prefill's
        # kernels; the decode kernels of every call
        self.launches_per_step = (1 + pre_k if self.has_a else 0) + (dec_k * self.n_dec if self.has_b else 0)

    def one_step(self, ev=None):
        if self.flush_each:
            self.flush.zero_()
        if ev:
            ev[0].record()
        if self.has_a:
            self.g_a.replay()
        if ev:
            ev[1].record()
        for _ in range(self.replays if self.has_b else 0):
            self.g_b.replay()
        if ev:
            ev[2].record()

    def tokens_per_step(self):
        return self.w.batch * ((self.n_pre if self.has_a else 0) + (self.n_dec if self.has_b else 0))

    def release(self):
        import torch
        for name in ("g_a", "g_b", "op", "flush", "qd", "kd", "vd", "qp", "kp", "vp"):
            if hasattr(self, name):
                delattr(self, name)
        torch.cuda.synchronize()
        torch.cuda.empty_cache()


def time_run(run, sfa, steps, warmup, world, dev, sampler=None):
    """W untimed steps, then exactly K steps between barriers and device
    synchronisations; per-step CUDA-event times of the prefill and decode
    parts (ms) and the clock record of the timed region."""
    import torch
    import torch.distributed as dist
    with nvtx_range(f"sfa {run.w.name} warm-up"):
        for _ in range(warmup):
            run.one_step()
        torch.cuda.synchronize()
    if run.op.check() != 0:
        raise SystemExit(f"{run.w.name}: device error during warm-up")
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.1)
    with nvtx_range(f"sfa {run.w.name} timed steps"):
        for s in range(steps):
            run.one_step(ev[s])
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    pre_ms = [e[0].elapsed_time(e[1]) for e in ev]
    dec_ms = [e[1].elapsed_time(e[2]) for e in ev]
    rc = run.op.check()
    if rc != 0:
        raise SystemExit(f"{run.w.name}: device error in the timed region: "
                         f"{sfa.sfa_status_string(rc)}")
    return pre_ms, dec_ms, clocks


def roofline_sections(run, pre_tot, dec_tot, steps, world, peak):
    """Per part (prefill, decode): tokens/s, time, algorithmic bytes per
    launch, achieved GB/s and the fraction of the HBM peak."""
    w, B = run.w, run.w.batch
    dec_bytes, pre_bytes = workload_bytes(w, run.n_pre)
    section = {}
    if run.has_a:
        pre_ms_avg = pre_tot / steps
        pre_gbs = pre_bytes / (pre_ms_avg / 1e3) / 1e9
        section["prefill"] = {"tokens_per_s": job_rate(world, B * run.n_pre * steps, pre_tot),
                              "ms": pre_ms_avg, "algorithmic_bytes": pre_bytes,
                              "achieved_gbs": pre_gbs, "frac": pre_gbs / peak}
    if run.has_b:
        dec_launch_ms = dec_tot / (steps * run.n_dec)
        dec_gbs = dec_bytes / (dec_launch_ms / 1e3) / 1e9
        section["decode"] = {"tokens_per_s": job_rate(world, B * run.n_dec * steps, dec_tot),
                             "us_per_step": 1e3 * dec_launch_ms, "algorithmic_bytes": dec_bytes,
                             "achieved_gbs": dec_gbs, "frac": dec_gbs / peak}
    return section


def dominant_kernel(run):
    """(part, kernel label, source file, traffic-file key) of the launch unit
    that dominates a step: one decode call or one prefill call."""
    if run.has_b and (not run.has_a or run.kind == "decode"):
        if run.w.batch >= 64 and run.w.window_k <= 256:  # the library's batch-tiled rule
            return ("decode", "decode_near_mma_kernel + decode_pool_kernel", "sfa_decode_tile.cu",
                    "decode_tile")
        return "decode", "decode_kernel", "sfa_decode.cu", "decode"
    return "prefill", "prefill", "sfa_prefill.cu", "prefill"


def roofline_for(run, section, peak, peak_src):
    part, kernel, src, key = dominant_kernel(run)
    if part not in section:  # a prefill-and-decode step whose prefill dominates
        part = "prefill" if "prefill" in section else "decode"
    dom = section[part]
    traffic, traffic_wl = kernel_traffic(
        os.path.join(ROOT, "kv_cache_compression_sfa_b200", "csrc", src), key, run.w.name)
    return {"bound": "hbm", "kernel": kernel, "part": part, "achieved": dom["achieved_gbs"],
            "peak": peak, "unit": "GB/s", "frac": dom["achieved_gbs"] / peak,
            "peak_source": peak_src, "traffic": traffic,
            "traffic_source": traffic_wl}


def extra_object(args, name, sfa, world, dev, rank, peak, peak_src):
    """A further workload timed in the same run: its own tokens/s, bytes,
    GB/s and roofline fraction (steps and warm-up bounded to keep the run
    short)."""
    from workloads import get_workload
    w = get_workload(name)
    n_pre = w.prefill_n[0]
    run = Run(w, n_pre, dev, rank, sfa)
    steps = max(3, min(args.steps, 10))
    pre_ms, dec_ms, _ = time_run(run, sfa, steps, max(3, args.warmup), world, dev)
    total, pre_tot, dec_tot = max_over_ranks(
        [sum(pre_ms) + sum(dec_ms), sum(pre_ms), sum(dec_ms)], world, dev)
    section = roofline_sections(run, pre_tot, dec_tot, steps, world, peak)
    obj = {"workload": workload_config(w, n_pre)["workload"],
           "value": job_rate(world, run.tokens_per_step() * steps, total), "unit": UNIT,
           "steps": steps, "ms_per_step": total / steps,
           "median": step_medians(pre_ms, dec_ms), **section,
           "roofline": roofline_for(run, section, peak, peak_src),
           "gpu_launches": steps * run.launches_per_step,
           "l2": workload_config(w, n_pre)["l2"]}
    run.release()
    return obj


def context_rows(w, sfa, dev, contexts, n_dec=64, reps=4):
    """Decode time per step after prompts of each length, with the SFA state
    per sequence against a full K/V cache [P1 §2.2, §3.3, §3.4]: the prompt is
    prefilled in 4,096-token calls, then n_dec decode steps are captured in a
    CUDA graph and replayed `reps` times."""
    import torch
    from workloads import TokenSource, make_slots
    src = TokenSource(w, dev)
    op = sfa.SfaOperator(sfa_config_for(sfa, w), make_slots(w, dev), w.batch,
                         max_prefill=4096, device=dev)
    lay = op.layout()
    state_per_seq = lay.stream_stride * w.n_layers
    rows = []
    for ctx in contexts:
        op.reset()
        for t0 in range(0, ctx, 4096):
            q, k, v = src.get(t0, min(ctx, t0 + 4096))
            op.prefill(q, k, v)
            del q, k, v
        qa, ka, va = src.get(ctx, ctx + n_dec)
        qd = [qa[:, :, t].contiguous() for t in range(n_dec)]
        kd = [ka[:, :, t].contiguous() for t in range(n_dec)]
        vd = [va[:, :, t].contiguous() for t in range(n_dec)]
        out_d = torch.empty((n_dec, w.n_layers, w.batch, w.hidden), dtype=torch.float32,
                            device=dev)
        for t in range(n_dec):  # warm-up (advances the state; cost is flat in t)
            op.decode(qd[t], kd[t], vd[t], out=out_d[t])
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                for t in range(n_dec):
                    op.decode(qd[t], kd[t], vd[t], out=out_d[t])
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        if op.check() != 0:
            raise SystemExit("device error in the context report")
        us = 1e3 * e0.elapsed_time(e1) / (reps * n_dec)
        rows.append({"context": ctx, "decode_us_per_step": us,
                     "sfa_state_bytes_per_seq": state_per_seq,
                     "full_kv_bytes_per_seq": full_kv_bytes(w, ctx),
                     "compression": full_kv_bytes(w, ctx) / state_per_seq})
        del g, qd, kd, vd, out_d, qa, ka, va
    del op
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rows


def flatness_object(sfa, dev):
    from workloads import get_workload
    w = get_workload("qwen7b_decode")
    rows = context_rows(w, sfa, dev, CONTEXTS)
    us = [r["decode_us_per_step"] for r in rows]
    return {"workload": (f"{w.name}: {w.n_layers} layers, {w.n_q_heads}q/{w.n_kv_heads}kv heads, "
                         f"head_dim {w.head_dim}, batch {w.batch}, k={w.window_k}; 64 decode "
                         f"steps after each prompt"),
            "rows": rows, "decode_us_spread": (max(us) - min(us)) / min(us)}


def main():
    args = parse()
    from workloads import get_workload
    if args.report:
        run_report(args)
        return
    headline_default = args.workload == HEADLINE and not args.batch and not args.layers
    w = get_workload(args.workload)
    if args.batch:
        w = w.replace(batch=args.batch)
    if args.layers:
        w = w.replace(n_layers=args.layers)
    n_pre = args.context or w.prefill_n[0]
    if args.impl == "reference":
        run_reference(args, w, n_pre)
        return

    import torch
    import torch.distributed as dist
    import kv_cache_compression_sfa_b200 as sfa
    from kv_cache_compression_sfa_b200 import build as sfa_build

    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    sfa_build.build()

    run = Run(w, n_pre, dev, rank, sfa)
    sampler = ClockSampler(gpu_index_for(dev)) if rank == 0 else None
    pre_ms, dec_ms, clocks = time_run(run, sfa, args.steps, args.warmup, world, dev, sampler)
    medians = step_medians(pre_ms, dec_ms)
    total_ms, pre_tot, dec_tot = max_over_ranks(
        [sum(pre_ms) + sum(dec_ms), sum(pre_ms), sum(dec_ms)], world, dev)
    value = job_rate(world, run.tokens_per_step() * args.steps, total_ms)
    ms_per_step = total_ms / args.steps

    peak, peak_kind = measured_peaks()
    peak_src = (f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                if peak_kind == "measured" else "fallback 6.65 TB/s")
    section = roofline_sections(run, pre_tot, dec_tot, args.steps, world, peak)
    roofline = roofline_for(run, section, peak, peak_src)

    # ---- e2e through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        with nvtx_range("sfa e2e"):
            if run.kind == "decode":
                e2e = measure_e2e_decode(args, w, run.op, run.qd, run.kd, run.vd, run.n_dec,
                                         world, dev)
            else:
                e2e = measure_e2e(args, w, run.op, run.qp, run.kp, run.vp, run.qd, run.kd,
                                  run.vd, n_pre, run.n_dec, world, dev)
    launches = args.steps * run.launches_per_step
    run.release()

    # ---- further workloads in the same run (one GPU only: every replica of
    # a multi-GPU run would repeat them)
    extras = {}
    if headline_default and not args.no_extras and world == 1:
        for name in EXTRAS:
            with nvtx_range(f"sfa extra {name}"):
                extras[name] = extra_object(args, name, sfa, world, dev, rank, peak, peak_src)
        with nvtx_range("sfa context flatness"):
            extras["context_flatness"] = flatness_object(sfa, dev)

    # ---- oracle on the host cores (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, n_pre, dev)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "median": medians,
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {**workload_config(w, n_pre),
                   "decode_inputs": "prefetched: complete before each call "
                                    "(sfa_set_decode_input_prefetch)"},
        **section,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
        **extras,
    }
    print(json.dumps(line), flush=True)


def measure_e2e(args, w, op, qp, kp, vp, qd, kd, vd, n_pre, n_dec, world, dev):
    """Same metric through SfaOperator with pinned host inputs and outputs:
    every step copies its q/k/v host->device, runs reset + prefill + decode
    steps, and reads all outputs back.  As a serving loop would, the copies
    run on their own streams and overlap the neighbouring steps' compute:
    step i+1's inputs go in and step i's outputs come out (the prefill's as
    soon as the prefill ends) while the compute stream works.  Device
    buffers are double-buffered and ordered by events; the timed region runs
    from before the first input copy to the end of the last output copy."""
    import torch
    import torch.distributed as dist
    L, B, H = w.n_layers, w.batch, w.hidden
    # decode inputs step-major ([step, L, B, heads, d]) so each step's slice
    # is contiguous on the device
    dec = [torch.stack(x) if x else None for x in (qd, kd, vd)]
    host_in = [x.cpu().pin_memory() for x in (qp, kp, vp, *dec) if x is not None]
    dev_in = [[torch.empty_like(x, device=dev) for x in host_in] for _ in range(2)]
    h_out_p = torch.empty((L, B, n_pre, H), dtype=torch.float32).pin_memory()
    h_out_d = torch.empty((n_dec, L, B, H), dtype=torch.float32).pin_memory()
    d_out_p = [torch.empty((L, B, n_pre, H), dtype=torch.float32, device=dev) for _ in range(2)]
    d_out_d = [torch.empty((n_dec, L, B, H), dtype=torch.float32, device=dev) for _ in range(2)]
    h2d = sum(x.numel() * x.element_size() for x in host_in)
    d2h = (h_out_p.numel() + h_out_d.numel()) * 4
    steps = max(3, min(args.steps, 200))
    comp = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    # Per-call views of each buffer set, made once: a serving loop keeps its
    # buffers, and slicing inside the loop would time tensor indexing.
    dec_views = [[(dev_in[b][3][t], dev_in[b][4][t], dev_in[b][5][t], d_out_d[b][t])
                  for t in range(n_dec)] if n_dec else [] for b in range(2)]

    def run(n):
        ev = lambda: torch.cuda.Event()
        in_done = [ev() for _ in range(n)]
        pre_done = [ev() for _ in range(n)]
        comp_done = [ev() for _ in range(n)]
        out_done = [ev() for _ in range(n)]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(comp)
        s_in.wait_event(e0)

        def copy_in(i):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:  # buffer b's inputs were read by step i-2
                    s_in.wait_event(comp_done[i - 2])
                for h, d in zip(host_in, dev_in[b]):
                    d.copy_(h, non_blocking=True)
                in_done[i].record(s_in)

        copy_in(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                copy_in(i + 1)
            comp.wait_event(in_done[i])
            if i >= 2:  # buffer b's outputs were read back by step i-2's copies
                comp.wait_event(out_done[i - 2])
            x = dev_in[b]
            op.reset()
            op.prefill(x[0], x[1], x[2], out=d_out_p[b])
            pre_done[i].record(comp)
            for qv, kv, vv, ov in dec_views[b]:
                op.decode(qv, kv, vv, out=ov)
            comp_done[i].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(pre_done[i])
                h_out_p.copy_(d_out_p[b], non_blocking=True)
                if n_dec:
                    s_out.wait_event(comp_done[i])
                    h_out_d.copy_(d_out_d[b], non_blocking=True)
                out_done[i].record(s_out)
        comp.wait_event(out_done[n - 1])
        e1.record(comp)
        return e0, e1

    run(3)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = run(steps)
    torch.cuda.synchronize()
    ms = max_over_ranks([e0.elapsed_time(e1)], world, dev)[0]
    # Host time to issue one step into empty queues (outside the timed run):
    # when it is close to the step time, the e2e figure is bound by the host.
    h0 = time.perf_counter()
    run(1)
    host_ms = 1e3 * (time.perf_counter() - h0)
    torch.cuda.synchronize()
    value = job_rate(world, B * (n_pre + n_dec) * steps, ms)
    return {"value": value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": steps, "ms_per_step": ms / steps, "host_issue_ms_per_step": host_ms,
            "l2": "not flushed (host copies between steps)",
            "overlap": "copies on two streams overlap the neighbouring steps' compute"}


def measure_e2e_decode(args, w, op, qd, kd, vd, n_dec, world, dev):
    """Decode-only step through SfaOperator: every decode call copies its
    q/k/v from pinned host memory and its result back.  As a serving loop
    would, the copies run on their own streams and overlap the neighbouring
    calls' compute: call i+1's inputs go in and call i's result comes out
    while call i runs.  Device buffers are double-buffered and ordered by
    events; the timed region runs from before the first input copy to the
    end of the last output copy."""
    import torch
    import torch.distributed as dist
    L, B, H = w.n_layers, w.batch, w.hidden
    n_ring = len(qd)
    host = [[x.cpu().pin_memory() for x in xs] for xs in (qd, kd, vd)]
    dev_in = [[torch.empty_like(xs[0], device=dev) for xs in (qd, kd, vd)] for _ in range(2)]
    d_out = [torch.empty((L, B, H), dtype=torch.float32, device=dev) for _ in range(2)]
    h_out = torch.empty((n_dec, L, B, H), dtype=torch.float32).pin_memory()
    per = sum(x[0].numel() * x[0].element_size() for x in host)
    steps = max(3, min(args.steps, 5))
    h_views = [h_out[t] for t in range(n_dec)]  # made once, outside the timed calls
    comp = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def run(n_steps):
        n = n_steps * n_dec
        ev = lambda: torch.cuda.Event()
        in_done = [ev() for _ in range(n)]
        comp_done = [ev() for _ in range(n)]
        out_done = [ev() for _ in range(n)]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(comp)
        s_in.wait_event(e0)

        def copy_in(i):
            b, r = i % 2, (i % n_dec) % n_ring
            with torch.cuda.stream(s_in):
                if i >= 2:  # buffer b's inputs were read by call i-2
                    s_in.wait_event(comp_done[i - 2])
                for src, dst in zip((host[0][r], host[1][r], host[2][r]), dev_in[b]):
                    dst.copy_(src, non_blocking=True)
                in_done[i].record(s_in)

        copy_in(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                copy_in(i + 1)
            comp.wait_event(in_done[i])
            if i >= 2:  # buffer b's result was read back by call i-2's copy
                comp.wait_event(out_done[i - 2])
            op.decode(dev_in[b][0], dev_in[b][1], dev_in[b][2], out=d_out[b])
            comp_done[i].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[i])
                h_views[i % n_dec].copy_(d_out[b], non_blocking=True)
                out_done[i].record(s_out)
        comp.wait_event(out_done[n - 1])
        e1.record(comp)
        return e0, e1

    run(3)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = run(steps)
    torch.cuda.synchronize()
    ms = max_over_ranks([e0.elapsed_time(e1)], world, dev)[0]
    value = job_rate(world, B * n_dec * steps, ms)
    return {"value": value, "unit": UNIT, "h2d_bytes_per_step": per * n_dec,
            "d2h_bytes_per_step": n_dec * L * B * H * 4, "steps": steps,
            "l2": "not flushed",
            "overlap": "copies on two streams overlap the neighbouring calls' compute"}


def cpu_baseline(w, n_pre, dev):
    """The fp64 oracle on the host cores, from position 0 over the workload's
    prompt and decode steps, on the streams of sample_streams(w); the token
    count is capped so one pass stays near 15 s, and the pass is repeated
    (from a fresh state) until about 10 s of work."""
    from workloads import make_slots
    slots_np = make_slots(w, dev).cpu().numpy()
    layers, seqs = sample_streams(w)
    n_full = n_pre + w.decode_steps
    q, k, v = oracle_inputs(w, layers, seqs, min(64, n_full), dev)
    _, _, dt64 = oracle_tokens_per_s(w, layers, seqs, q, k, v, slots_np)
    n_tok = max(64, min(n_full, int(64 * 15.0 / max(dt64, 1e-3))))
    q, k, v = oracle_inputs(w, layers, seqs, n_tok, dev)
    total_tok, total_dt, reps, used = 0.0, 0.0, 0, 1
    while reps < 1 or (total_dt < 10.0 and reps < 100):
        rate, used, dt = oracle_tokens_per_s(w, layers, seqs, q, k, v, slots_np)
        total_tok += rate * dt
        total_dt += dt
        reps += 1
    return {"value": total_tok / total_dt, "unit": UNIT, "cores": used, "kind": "oracle",
            "sample": (f"layers {layers} x sequences {seqs} of {w.name} ({w.n_layers} layers x "
                       f"{w.batch} seq), positions 0..{n_tok - 1} of {n_full}, repeated {reps} "
                       f"times ({total_dt:.1f} s); tokens scaled to positions through all "
                       f"layers")}


# ------------------------------------------------------------------ reports


def full_kv_bytes(w, n: int) -> int:
    """Bytes of a full K/V cache for one sequence at context n, all layers."""
    e = 4 if w.in_dtype == "f32" else 2
    return 2 * n * w.n_kv_heads * w.head_dim * e * w.n_layers


def enhancement_stats(x, out):
    """Per (layer, sequence, token): cos(enh, x) and |enh| / |out| with
    enh = out - x; returns medians and 90th percentiles over all rows."""
    import numpy as np
    x = np.asarray(x, np.float64).reshape(-1, np.shape(x)[-1])
    out = np.asarray(out, np.float64).reshape(-1, np.shape(out)[-1])
    enh = out - x
    ne = np.linalg.norm(enh, axis=1)
    nx = np.linalg.norm(x, axis=1)
    no = np.linalg.norm(out, axis=1)
    ok = (ne > 0) & (nx > 0)
    cos = (enh * x).sum(axis=1)[ok] / (ne[ok] * nx[ok])
    share = ne[no > 0] / no[no > 0]
    q = lambda a, p: float(np.percentile(a, p)) if a.size else 0.0
    return {"cos_median": q(cos, 50), "abs_cos_p90": q(np.abs(cos), 90),
            "share_median": q(share, 50), "share_p90": q(share, 90), "rows": int(x.shape[0])}


def run_report(args):
    import dataclasses
    import numpy as np
    import torch
    import kv_cache_compression_sfa_b200 as sfa
    from kv_cache_compression_sfa_b200 import build as sfa_build
    from workloads import ALPHA_PRESETS, TokenSource, get_workload, make_slots
    if not torch.cuda.is_available():
        raise SystemExit("bench.py --report needs a CUDA device")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    sfa_build.build()

    if args.report == "context":
        # state bytes per sequence vs a full K/V cache, and decode time per
        # step after prompts of growing length [P1 §2.2, §3.4]
        w = get_workload(args.workload if args.workload != HEADLINE else "qwen7b_decode")
        ctxs, ctx = [], 1024
        while ctx <= args.max_context:
            ctxs.append(ctx)
            ctx *= 2
        rows = context_rows(w, sfa, dev, ctxs)
        print(json.dumps({"report": "context", "workload": w.name, "n_layers": w.n_layers,
                          "window_k": w.window_k, "rows": rows}), flush=True)
        return

    # enhancement share and its angle to x against alpha_base [P2 calibration]
    w = get_workload(args.workload if args.workload != HEADLINE else "qwen05b")
    n = args.context or w.prefill_n[0]
    src = TokenSource(w, dev)
    slots = make_slots(w, dev)
    q, k, v = src.get(0, n)
    res = []
    presets = [(0.0, 0.8)] + [(0.1, 0.8)] + list(ALPHA_PRESETS)
    outs = {}
    for ab, dec in presets:
        wv = w.replace(values=dataclasses.replace(w.values, alpha_base=ab, cross_decay=dec))
        op = sfa.SfaOperator(sfa_config_for(sfa, wv), slots, w.batch, max_prefill=n, device=dev)
        outs[(ab, dec)] = op.prefill(q, k, v).cpu().numpy()
        if op.check() != 0:
            raise SystemExit("device error in the enhancement report")
    x = outs[(0.0, 0.8)]  # alpha_base = 0: out == x exactly
    for ab, dec in presets[1:]:
        st = enhancement_stats(x, outs[(ab, dec)])
        per_layer = [enhancement_stats(x[l], outs[(ab, dec)][l])["share_median"]
                     for l in (0, w.n_layers // 2, w.n_layers - 1)]
        res.append({"alpha_base": ab, "cross_decay": dec, **st,
                    "share_median_layers_first_mid_last": per_layer})
    print(json.dumps({"report": "enhancement", "workload": w.name, "tokens": n,
                      "data": "synthetic N(0,1) activations; not comparable with trained models",
                      "rows": res}), flush=True)


if __name__ == "__main__":
    main()
