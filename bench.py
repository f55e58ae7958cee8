"""Decode benchmark: Qwen3-8B-shaped greedy decode, batch 1, through the
persistent megakernel (one launch for all timed decode iterations).

Workload (MPK blog excerpt, Figure 1): a 39-token prompt followed by 512
greedy tokens, no speculative decoding.  Weights are seeded synthetic bf16
N(0, 0.02) draws of the Qwen3-8B shape.  A step is one decode iteration (one
token for the request): W warm-up iterations after the prompt, then the state
is rewound to the end of the prompt and exactly K iterations (K <= 512) are
timed inside ONE persistent launch with CUDA events on the launching stream.
Every iteration streams all 15.1 GB of weights, far more than the 126 MB L2,
so no L2 flush is needed between iterations.

Multi-GPU: the path does not shard (replicas only); with --gpus N every rank
decodes its own request on its own GPU, the time is the maximum over ranks and
the value counts the tokens of all ranks.

--impl reference times the CPU oracle (the reference arm of this build) on
the host cores with the same metric.

--workload batch8 measures the batched configuration instead: 8 concurrent
requests in tokens[8, 1024], prompt lengths uniform in [32, 512], 256 greedy
tokens each.  The prompts are ingested first (untimed, one decode iteration
per prompt token), then 256 lock-step iterations (every request one token per
iteration, each at its own position) run in ONE timed launch; a step is one
such iteration, reported in ms/step.  The projections run on the tensor cores.
--requests R (2..16) runs the same workload with R requests (9..16: every
contraction 16 requests wide).

--workload long measures one request over a KV cache pre-filled with 32768
positions (seeded N(0,1) bf16): 128 greedy iterations in one timed launch.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

PROMPT = 39
GENERATED = 512
METRIC = "decode ms/token (Qwen3-8B-shape, batch 1) and HBM GB/s vs ~8 TB/s peak"
UNIT = "ms/token"
A100_MPK_MS = 12.5  # the pages' MPK figure on one A100 40GB for this workload (context)

BATCH, BATCH_SEQ, BATCH_PROMPT, BATCH_GENERATED = 8, 1024, (32, 512), 256
METRIC_BATCH = "decode ms/step (Qwen3-8B-shape, 8 requests) and HBM GB/s vs ~8 TB/s peak"
UNIT_BATCH = "ms/step"

LONG_CONTEXT, LONG_GENERATED = 32768, 128
PREFILL_TOKENS = 8  # prompt positions per prefill iteration (the tensor-core path's column count)
METRIC_LONG = "decode ms/token (Qwen3-8B-shape, batch 1, 32768 cached positions) and HBM GB/s vs ~8 TB/s peak"


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--workload", choices=["batch1", "batch8", "long"], default="batch1",
                   help="batch1: one request, 39-token prompt + 512 tokens (default); batch8: 8 requests; "
                        "long: one request over 32768 pre-filled positions")
    p.add_argument("--requests", type=int, default=0, help="batch8 workload: requests (2..16, default 8)")
    p.add_argument("--steps", type=int, default=0, help="timed steps (default: 512 for batch1, 256 for batch8)")
    p.add_argument("--warmup", type=int, default=8)
    p.add_argument("--impl", choices=["mpk", "reference"], default="mpk")
    p.add_argument("--shape", default="qwen3-8b", help="qwen3-8b (default), qwen3-0.6b or tiny")
    p.add_argument("--workers", type=int, default=0, help="num_workers (default: SMs - local/4)")
    p.add_argument("--local-schedulers", type=int, default=16)
    p.add_argument("--attn-chunks", type=int, default=0)
    p.add_argument("--lookahead", type=int, default=0)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--op-by-op", action="store_true", help="also time one launch per operation")
    p.add_argument("--profiling", action="store_true", help="record the task timeline of the timed run")
    p.add_argument("--timeline-out", default="")
    p.add_argument("--cpu-budget-s", type=float, default=20.0)
    p.add_argument("--prefetch-kb", type=int, default=0, help="L2 prefetch distance per worker (<=0 off)")
    p.add_argument("--tasks-per-worker", type=int, default=2, help="tasks per worker of the claimed GEMV ops")
    p.add_argument("--claim-tasks", action="store_true",
                   help="GEMV ops hand tasks out through a shared counter instead of the fixed mapping")
    p.add_argument("--attention", choices=["auto", "fused", "split"], default="auto")
    p.add_argument("--layers", type=int, default=0, help="override the layer count (profiling cases)")
    p.add_argument("--vocab", type=int, default=0, help="override the vocabulary (profiling cases)")
    args = p.parse_args(argv)
    if args.requests and not 2 <= args.requests <= 16:
        p.error("--requests must be in 2..16")
    if not args.steps:
        args.steps = {"batch1": GENERATED, "batch8": BATCH_GENERATED, "long": LONG_GENERATED}[args.workload]
    return args


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = tempfile.mktemp(prefix="clocks_", suffix=".csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
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
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def kernel_source_digest() -> str:
    import hashlib
    csrc = os.path.join(ROOT, "persistent_megakernel_decode_02_b200", "csrc")
    h = hashlib.sha256()
    for f in ("mpk_kernel.cu", "mpk_internal.h", "mpk_ptx.cuh", "mpk_batch.cuh"):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_ratio(kernel: str = "mpk_persistent_kernel"):
    """DRAM bytes per algorithmic byte of `kernel` from the committed ncu summary,
    when it was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_dram_traffic.txt")
    if not os.path.exists(path):
        return None
    kv = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
    if kv.get("kernel_source_sha256_16") != kernel_source_digest():
        return None
    return float(kv["dram_bytes_per_algorithmic_byte"])


def algorithmic_bytes(shape, first_pos: int, iters: int) -> int:
    """Bytes one decode iteration must move, summed over iterations at positions
    first_pos .. first_pos+iters-1: every streamed weight byte once, the K/V of
    positions 0..s read and the new position written."""
    per_pos = shape.kv_bytes_per_position()
    total = 0
    for i in range(iters):
        s = first_pos + i
        total += shape.streamed_weight_bytes() + (s + 1) * per_pos + per_pos
    return total


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if args.impl == "mpk" else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
        pg = dist
    return world, rank, local, pg


def max_over_ranks(pg, value: float, device=None) -> float:
    if pg is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def whole_job(ms_max: float, steps: int, world: int):
    """Replicas: each of `world` ranks decodes `steps` tokens of its own request;
    the job took the slowest rank's `ms_max`.  Returns (ms per generated token
    of the whole job, whole-job tokens/s)."""
    tokens = steps * world
    return ms_max / tokens, 1e3 * tokens / ms_max


def barrier(pg, device=None):
    if pg is None:
        return
    import torch
    t = torch.zeros(1, device=device)
    pg.all_reduce(t)


# ----------------------------------------------------------------------------- oracle timing

def time_oracle(shape, w_cpu, tokens_cpu, budget_s: float, max_iters: int = 64, layer_sample=None, kv=None,
                step0: int = 0):
    """Time the CPU oracle on the first iterations of the same workload (from
    position step0, over the pre-filled bf16 caches kv = (K, V) when given).
    Returns (ms per full token, iterations, threads, description)."""
    import numpy as np
    import torch
    import oracle
    from synth import qwen3 as sq

    sub_shape, sub_w, frac = shape, w_cpu, 1.0
    if layer_sample is not None and layer_sample < shape.layers:
        # a bounded sample: the first `layer_sample` layers and the LM head
        sub_shape = sq.Qwen3Shape(shape.name + f"-first{layer_sample}", layer_sample, shape.hidden, shape.q_heads,
                                  shape.kv_heads, shape.head_dim, shape.intermediate, shape.vocab, shape.tied)
        keep = set(sub_shape.weight_shapes())
        sub_w = {k: v for k, v in w_cpu.items() if k in keep}
        frac = sub_shape.streamed_weight_bytes() / shape.streamed_weight_bytes()
    dec = oracle.Decoder(sub_shape, sub_w)
    toks = tokens_cpu.numpy().copy()
    R, S = toks.shape
    if kv is None:
        kc, vc = dec.new_cache(R, S)
    else:
        kc, vc = (np.ascontiguousarray(c[:sub_shape.layers].view(torch.int16).numpy().view(np.uint16)) for c in kv)
    step = np.full(R, step0, np.int32)
    times = []
    t_start = time.perf_counter()
    while len(times) < max_iters:
        t0 = time.perf_counter()
        dec.iteration(kc, vc, step, toks, None, oracle.ROUND_NONE, None, None)
        times.append(time.perf_counter() - t0)
        if time.perf_counter() - t_start > budget_s:
            break
    ms = 1e3 * (sum(times) / len(times)) / frac
    first = step0
    desc = (f"{len(times)} oracle decode iterations at positions {first}..{first + len(times) - 1} of the same request "
            f"({sub_shape.layers} of {shape.layers} layers + LM head, scaled by weight bytes x{1 / frac:.2f})"
            if frac < 1.0 else
            f"{len(times)} full oracle decode iterations at positions {first}..{first + len(times) - 1} of the same "
            f"request")
    return ms, len(times), oracle.num_threads(), desc


def run_reference(args):
    """The reference arm: the CPU oracle, as it stands, on the host cores."""
    world, rank, _, pg = dist_setup(args)
    if rank != 0:
        if pg is not None:
            pg.destroy_process_group()
        return
    import torch
    from synth import qwen3 as sq

    shape = sq.SHAPES[args.shape]
    S = PROMPT + GENERATED
    w_cpu = sq.make_weights(shape, seed=0)
    tokens = sq.make_tokens(shape, 1, S, [PROMPT], seed=0)
    total = args.steps + args.warmup
    # each step is a bounded sample sized so the whole run ends within a few minutes
    per_step_budget = max(0.05, 150.0 / max(total, 1))
    _, _, _, _ = time_oracle(shape, w_cpu, tokens, 0.0, max_iters=1, layer_sample=1)  # load + first touch
    probe_ms, _, _, _ = time_oracle(shape, w_cpu, tokens, 0.0, max_iters=1, layer_sample=1)
    per_layer_s = probe_ms / 1e3 * (sq.Qwen3Shape("x", 1, shape.hidden, shape.q_heads, shape.kv_heads,
                                                  shape.head_dim, shape.intermediate, shape.vocab,
                                                  shape.tied).streamed_weight_bytes()
                                     / shape.streamed_weight_bytes())
    layers = max(1, min(shape.layers, int(per_step_budget / max(per_layer_s, 1e-6))))
    import numpy as np
    import oracle
    sub_shape = sq.Qwen3Shape(shape.name + "-s", layers, shape.hidden, shape.q_heads, shape.kv_heads,
                              shape.head_dim, shape.intermediate, shape.vocab, shape.tied)
    keep = set(sub_shape.weight_shapes())
    dec = oracle.Decoder(sub_shape, {k: v for k, v in w_cpu.items() if k in keep})
    frac = sub_shape.streamed_weight_bytes() / shape.streamed_weight_bytes()
    toks = tokens.numpy().copy()
    kc, vc = dec.new_cache(1, S)
    step = np.zeros(1, np.int32)
    for _ in range(args.warmup):
        dec.iteration(kc, vc, step, toks, None, oracle.ROUND_NONE, None, None)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        dec.iteration(kc, vc, step, toks, None, oracle.ROUND_NONE, None, None)
    el = time.perf_counter() - t0
    ms = 1e3 * el / max(args.steps, 1) / frac
    sample = (f"each step: one oracle decode iteration over the first {layers} of {shape.layers} layers + LM head, "
              f"scaled to a full token by weight bytes (x{1 / frac:.2f})")
    line = {
        "impl": "reference", "metric": METRIC, "value": ms, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": ms / A100_MPK_MS, "dtype": "f64", "data": "synthetic",
        "config": workload_config(shape, args, None),
        "cpu_baseline": {"value": ms, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": ms, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def workload_config(shape, args, dec):
    cfg = {
        "workload": f"{shape.name}-shape greedy decode, batch 1, {PROMPT}-token prompt + {GENERATED} generated tokens",
        "requests": 1, "prompt_tokens": PROMPT, "seq_len": PROMPT + GENERATED, "timed_tokens": args.steps,
        "weights": "seeded synthetic bf16 N(0,0.02), norms 1.0",
        "l2": "no flush: every step streams all weights (>= 1.19 GB), larger than the 126 MB L2",
    }
    if dec is not None:
        cfg.update({"num_workers": dec.kernel.num_workers, "num_local_schedulers": dec.kernel.num_local_schedulers,
                    "parallelism": "replicas"})
    return cfg


# ----------------------------------------------------------------------------- GPU arm

def sized_shape(sq, args):
    """The --shape, with --layers / --vocab overrides (smaller profiling cases)."""
    shape = sq.SHAPES[args.shape]
    if args.layers or args.vocab:
        import dataclasses
        shape = dataclasses.replace(shape, name=f"{shape.name}-L{args.layers or shape.layers}-V{args.vocab or shape.vocab}",
                                    layers=args.layers or shape.layers, vocab=args.vocab or shape.vocab)
    return shape


def batch_algorithmic_bytes(shape, first_pos, iters: int) -> int:
    """Bytes one lock-step iteration of several requests must move, summed over
    iterations: every streamed weight byte once (shared by the batch), and per
    request the K/V of positions 0..s read and position s written."""
    per_pos = shape.kv_bytes_per_position()
    total = 0
    for i in range(iters):
        total += shape.streamed_weight_bytes()
        for p in first_pos:
            total += (int(p) + i + 1) * per_pos + per_pos
    return total


def main_batch(args):
    """The batched configuration: 8 requests, prompts U[32, 512], 256 lock-step
    decode iterations timed in one launch."""
    import torch
    world, rank, local, pg = dist_setup(args)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from synth import qwen3 as sq
    from persistent_megakernel_decode_02_b200 import build_decoder, load

    shape = sized_shape(sq, args)
    R, S, G = args.requests or BATCH, BATCH_SEQ, BATCH_GENERATED
    if not 2 <= R <= 16:
        raise SystemExit("--requests must be in 2..16")
    kname = "mpk_persistent_batch_kernel" if R <= 8 else "mpk_persistent_batch16_kernel"
    steps = args.steps
    if not (1 <= steps <= G and 0 <= args.warmup <= G):
        raise SystemExit(f"--steps must be in 1..{G} and --warmup in 0..{G}")
    t0 = time.time()
    w_cpu = sq.make_weights(shape, seed=0)
    w = {k: v.to(dev) for k, v in w_cpu.items()}
    t_gen = time.time() - t0
    lens = sq.make_prompt_lengths(R, BATCH_PROMPT[0], BATCH_PROMPT[1], seed=0)
    tokens_cpu = sq.make_tokens(shape, R, S, lens, seed=0)
    ls = args.local_schedulers
    W = args.workers or (load().mpk_device_sm_count() - ls // 4)
    dec = build_decoder(shape, w, requests=R, max_seq=S, num_workers=W, num_local_schedulers=ls,
                        attn_chunks=args.attn_chunks or None, sched_lookahead=args.lookahead,
                        profiling=args.profiling)
    # the prompts' graph: PREFILL_TOKENS positions of one request per
    # iteration, the requests one after another, on the decode graph's cache
    pre = build_decoder(shape, w, requests=R, max_seq=S, num_workers=W, num_local_schedulers=ls,
                        prefill_tokens=PREFILL_TOKENS, k_cache=dec.k_cache, v_cache=dec.v_cache)
    stream = torch.cuda.current_stream(dev)
    tok = tokens_cpu.to(dev)
    p_end = (lens - 1).to(torch.int32).to(dev)          # each request has consumed its prompt
    step = torch.zeros(R, dtype=torch.int32, device=dev)
    pre.run(step, tok, p_end)                            # phase A: the prompts
    dec.run(step, tok, p_end + args.warmup)              # warm-up iterations
    torch.cuda.synchronize(dev)
    dec.kernel.check_status()
    tok.copy_(tokens_cpu.to(dev))                        # rewind to the end of the prompts
    step.copy_(p_end)
    stop = p_end + steps
    barrier(pg, dev)
    torch.cuda.synchronize(dev)
    clk = ClockSampler(local)
    clk.start()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    dec.run(step, tok, stop, stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = clk.stop()
    barrier(pg, dev)
    dec.kernel.check_status()
    ms_launch = e0.elapsed_time(e1)
    assert torch.equal(step, stop), "not every request ran its timed steps"
    gen = [tok[r, int(lens[r]):int(lens[r]) + steps].cpu() for r in range(R)]
    assert all(bool((g >= 0).all()) for g in gen), "some timed tokens were not generated"
    ms_max = max_over_ranks(pg, ms_launch, dev)
    ms_per_step = ms_max / steps
    tokens_per_s = 1e3 * R * steps * world / ms_max
    p_host = (lens - 1).tolist()
    bytes_launch = batch_algorithmic_bytes(shape, p_host, steps)
    gbs = bytes_launch / (ms_launch * 1e-3) / 1e9
    peak, peak_kind = measured_peaks()

    timeline_stats = None
    if args.profiling:
        tl = dec.kernel.timeline()
        if args.timeline_out:
            write_chrome_trace(tl, dec, args.timeline_out)
        op_kind.per_layer = (dec.kernel.num_ops() - 2) // shape.layers
        timeline_stats = timeline_summary(tl, shape)

    op_ms = None
    if args.op_by_op:
        # the same timed iterations, one launch per operation
        tok.copy_(tokens_cpu.to(dev))
        step.copy_(p_end)
        torch.cuda.synchronize(dev)
        o0 = torch.cuda.Event(enable_timing=True)
        o1 = torch.cuda.Event(enable_timing=True)
        o0.record(stream)
        dec.run_op_by_op(step, tok, stop, stream)
        o1.record(stream)
        torch.cuda.synchronize(dev)
        dec.kernel.check_status()
        op_ms = o0.elapsed_time(o1) / steps

    # end to end through the public API with host buffers: the prompts are
    # ingested in one launch (timed on its own, through the prefill graph and
    # for comparison as lock-step decode iterations); the decode window is H2D
    # of tokens / step / step_end from pinned memory, the timed lock-step
    # iterations in one launch and D2H of the tokens, reported per step.
    e2e = None
    if not args.no_e2e:
        host_tok = tokens_cpu.clone().pin_memory()
        host_step0 = torch.zeros(R, dtype=torch.int32).pin_memory()
        host_pend = (lens - 1).to(torch.int32).pin_memory()
        host_end = ((lens - 1) + steps).to(torch.int32).pin_memory()
        out_tok = torch.empty_like(host_tok).pin_memory()
        barrier(pg, dev)
        torch.cuda.synchronize(dev)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
        # ev[0..1]: prefill graph, ev[2..3]: lock-step decode (run first), ev[4..5]: decode window
        for graph, (a, b) in ((dec, (2, 3)), (pre, (0, 1))):
            ev[a].record(stream)
            tok.copy_(host_tok, non_blocking=True)
            step.copy_(host_step0, non_blocking=True)
            stop.copy_(host_pend, non_blocking=True)
            graph.run(step, tok, stop, stream)
            ev[b].record(stream)
            torch.cuda.synchronize(dev)
            graph.kernel.check_status()
        barrier(pg, dev)
        ev[4].record(stream)
        tok.copy_(host_tok, non_blocking=True)
        step.copy_(host_pend, non_blocking=True)
        stop.copy_(host_end, non_blocking=True)
        dec.run(step, tok, stop, stream)
        out_tok.copy_(tok, non_blocking=True)
        ev[5].record(stream)
        torch.cuda.synchronize(dev)
        dec.kernel.check_status()
        prompt_ms = max_over_ranks(pg, ev[0].elapsed_time(ev[1]), dev)
        prompt_decode_ms = max_over_ranks(pg, ev[2].elapsed_time(ev[3]), dev)
        e2e_ms = max_over_ranks(pg, ev[4].elapsed_time(ev[5]), dev)
        for r in range(R):
            assert torch.equal(out_tok[r, int(lens[r]):int(lens[r]) + steps], gen[r]), "e2e tokens differ"
        e2e = {"value": e2e_ms / steps, "unit": UNIT_BATCH,
               "h2d_bytes_per_step": (host_tok.numel() * 8 + 8 * R) / steps,
               "d2h_bytes_per_step": out_tok.numel() * 8 / steps,
               "includes": f"H2D of tokens/step/step_end, {steps} lock-step decode iterations in one launch after "
                           f"the prompts, D2H of tokens",
               "prompt_ingestion_ms": prompt_ms,
               "prompt_ingestion": f"H2D of the prompts, their {int((lens - 1).sum())} positions through the "
                                   f"prefill graph ({PREFILL_TOKENS} positions of one request per iteration on the "
                                   f"tensor cores, the requests one after another) in one launch",
               "prompt_ingestion_ms_lock_step_decode": prompt_decode_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ms_cpu, n, cores, desc = time_oracle(shape, w_cpu, tokens_cpu, args.cpu_budget_s, layer_sample=2)
        cpu = {"value": ms_cpu, "unit": UNIT_BATCH, "cores": cores, "kind": "oracle",
               "sample": desc.replace("of the same request", f"of all {R} requests")}

    if rank == 0:
        line = {
            "metric": METRIC_BATCH.replace("8 requests", f"{R} requests"), "value": ms_per_step, "unit": UNIT_BATCH, "n_gpus": world, "steps": steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {
                "workload": f"{shape.name}-shape greedy decode, {R} requests, tokens[{R},{S}], prompt lengths "
                            f"U[{BATCH_PROMPT[0]},{BATCH_PROMPT[1]}] (seed 0), {steps} lock-step tokens each",
                "requests": R, "prompt_tokens": [int(x) for x in lens], "seq_len": S, "timed_steps": steps,
                "weights": "seeded synthetic bf16 N(0,0.02), norms 1.0",
                "projections": "tcgen05 MMA over the batch (bf16 inputs, fp32 accumulate)",
                "l2": "no flush: every step streams all weights (15.1 GB), larger than the 126 MB L2",
                "num_workers": dec.kernel.num_workers, "num_local_schedulers": dec.kernel.num_local_schedulers,
                "parallelism": "replicas"},
            "tokens_per_s": tokens_per_s,
            "hbm_gbs": gbs,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "traffic": (None if traffic_ratio(kname) is None else traffic_ratio(kname) * bytes_launch),
                         "traffic_source": "ncu dram bytes of a 4-layer case scaled by algorithmic bytes",
                         "peak_kind": peak_kind,
                         "algorithmic_bytes_per_launch": bytes_launch, "launch_ms": ms_launch,
                         "kernel": kname},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": 1,
            "clocks": clocks,
            "op_by_op_ms_per_step": op_ms,
            "timeline": timeline_stats,
            "setup_s": {"weights": round(t_gen, 1)},
        }
        print(json.dumps(line), flush=True)
    pre.kernel.close()
    dec.kernel.close()
    if pg is not None:
        pg.destroy_process_group()


def main_long(args):
    """Long-context decode: one request whose KV cache holds 32768 pre-filled
    positions (seeded N(0,1) bf16), 128 greedy iterations timed in one launch."""
    import torch
    world, rank, local, pg = dist_setup(args)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from synth import qwen3 as sq
    from persistent_megakernel_decode_02_b200 import build_decoder, load

    shape = sized_shape(sq, args)
    P, steps = LONG_CONTEXT, args.steps
    if not (1 <= steps <= LONG_GENERATED and 0 <= args.warmup <= LONG_GENERATED):
        raise SystemExit(f"--steps must be in 1..{LONG_GENERATED} and --warmup in 0..{LONG_GENERATED}")
    S = P + LONG_GENERATED + 1
    t0 = time.time()
    w_cpu = sq.make_weights(shape, seed=0)
    w = {k: v.to(dev) for k, v in w_cpu.items()}
    kc_cpu, vc_cpu = sq.make_kv_prefill(shape, 1, S, P, seed=11)
    kc, vc = kc_cpu.to(dev), vc_cpu.to(dev)
    t_gen = time.time() - t0
    tokens_cpu = sq.make_tokens(shape, 1, S, [P + 1], seed=12)
    ls = args.local_schedulers
    W = args.workers or (load().mpk_device_sm_count() - ls // 4)
    dec = build_decoder(shape, w, requests=1, max_seq=S, num_workers=W, num_local_schedulers=ls,
                        attn_chunks=args.attn_chunks or None, k_cache=kc, v_cache=vc, profiling=args.profiling)
    stream = torch.cuda.current_stream(dev)
    tok = tokens_cpu.to(dev)
    step = torch.full((1,), P, dtype=torch.int32, device=dev)
    end = lambda n: torch.full((1,), n, dtype=torch.int32, device=dev)
    dec.run(step, tok, end(P + args.warmup))             # warm-up iterations
    torch.cuda.synchronize(dev)
    dec.kernel.check_status()
    tok.copy_(tokens_cpu.to(dev))                        # rewind (positions >= P are rewritten)
    step.fill_(P)
    stop = end(P + steps)
    barrier(pg, dev)
    torch.cuda.synchronize(dev)
    clk = ClockSampler(local)
    clk.start()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    dec.run(step, tok, stop, stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = clk.stop()
    barrier(pg, dev)
    dec.kernel.check_status()
    ms_launch = e0.elapsed_time(e1)
    assert int(step.item()) == P + steps
    gen = tok[0, P + 1:P + 1 + steps].cpu()
    assert bool((gen >= 0).all()), "some timed tokens were not generated"
    ms_max = max_over_ranks(pg, ms_launch, dev)
    value, tokens_per_s = whole_job(ms_max, steps, world)
    bytes_launch = algorithmic_bytes(shape, P, steps)
    gbs = bytes_launch / (ms_launch * 1e-3) / 1e9
    peak, peak_kind = measured_peaks()
    timeline_stats = None
    if args.profiling:
        tl = dec.kernel.timeline()
        if args.timeline_out:
            write_chrome_trace(tl, dec, args.timeline_out)
        op_kind.per_layer = (dec.kernel.num_ops() - 2) // shape.layers
        timeline_stats = timeline_summary(tl, shape)

    op_ms = None
    if args.op_by_op:
        # the same timed iterations, one launch per operation
        tok.copy_(tokens_cpu.to(dev))
        step.fill_(P)
        torch.cuda.synchronize(dev)
        o0 = torch.cuda.Event(enable_timing=True)
        o1 = torch.cuda.Event(enable_timing=True)
        o0.record(stream)
        dec.run_op_by_op(step, tok, stop, stream)
        o1.record(stream)
        torch.cuda.synchronize(dev)
        dec.kernel.check_status()
        op_ms = o0.elapsed_time(o1) / steps

    # end to end through the public API with host buffers: H2D of tokens / step /
    # step_end from pinned memory, the timed iterations in one launch over the
    # resident pre-filled cache, D2H of the tokens; per generated token
    e2e = None
    if not args.no_e2e:
        host_tok = tokens_cpu.clone().pin_memory()
        host_step = torch.full((1,), P, dtype=torch.int32).pin_memory()
        host_end = torch.full((1,), P + steps, dtype=torch.int32).pin_memory()
        out_tok = torch.empty_like(host_tok).pin_memory()
        barrier(pg, dev)
        torch.cuda.synchronize(dev)
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        tok.copy_(host_tok, non_blocking=True)
        step.copy_(host_step, non_blocking=True)
        stop.copy_(host_end, non_blocking=True)
        dec.run(step, tok, stop, stream)
        out_tok.copy_(tok, non_blocking=True)
        f1.record(stream)
        torch.cuda.synchronize(dev)
        dec.kernel.check_status()
        e2e_ms = max_over_ranks(pg, f0.elapsed_time(f1), dev)
        assert torch.equal(out_tok[0, P + 1:P + 1 + steps], gen), "e2e tokens differ from the timed run"
        e2e = {"value": whole_job(e2e_ms, steps, world)[0], "unit": UNIT,
               "h2d_bytes_per_step": (host_tok.numel() * 8 + 8) / steps,
               "d2h_bytes_per_step": out_tok.numel() * 8 / steps,
               "includes": f"H2D of tokens/step/step_end, {steps} decode iterations over the {P} cached positions "
                           f"in one launch, D2H of tokens"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ms_cpu, n, cores, desc = time_oracle(shape, w_cpu, tokens_cpu, args.cpu_budget_s, kv=(kc_cpu, vc_cpu),
                                             step0=P)
        cpu = {"value": ms_cpu, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": desc + f" over the {P} pre-filled cached positions"}
    if rank == 0:
        line = {
            "metric": METRIC_LONG, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps,
            "warmup": args.warmup, "ms_per_step": ms_max / steps, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{shape.name}-shape greedy decode, batch 1, KV cache pre-filled with {P} "
                                   f"positions of seeded N(0,1) bf16, {steps} greedy tokens",
                       "requests": 1, "cached_positions": P, "seq_len": S, "timed_tokens": steps,
                       "weights": "seeded synthetic bf16 N(0,0.02), norms 1.0",
                       "attention": "split-K operation", "num_workers": dec.kernel.num_workers,
                       "l2": "no flush: every step streams all weights (15.1 GB) and 4.8 GB of KV",
                       "parallelism": "replicas"},
            "tokens_per_s": tokens_per_s, "hbm_gbs": gbs,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "traffic": (None if traffic_ratio("mpk_persistent_split_kernel") is None
                                     else traffic_ratio("mpk_persistent_split_kernel") * bytes_launch),
                         "traffic_source": "ncu dram bytes of a 2-iteration run scaled by algorithmic bytes",
                         "peak_kind": peak_kind, "algorithmic_bytes_per_launch": bytes_launch,
                         "launch_ms": ms_launch, "kernel": "mpk_persistent_split_kernel"},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": 1, "clocks": clocks, "op_by_op_ms_per_token": op_ms,
            "timeline": timeline_stats,
            "setup_s": {"weights_and_kv": round(t_gen, 1)},
        }
        print(json.dumps(line), flush=True)
    dec.kernel.close()
    if pg is not None:
        pg.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "batch8":
        return main_batch(args)
    if args.workload == "long":
        return main_long(args)
    import torch
    world, rank, local, pg = dist_setup(args)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from synth import qwen3 as sq
    from persistent_megakernel_decode_02_b200 import build_decoder, load

    shape = sized_shape(sq, args)
    S = PROMPT + GENERATED
    if not (1 <= args.steps <= GENERATED and 0 <= args.warmup <= GENERATED):
        raise SystemExit(f"--steps must be in 1..{GENERATED} and --warmup in 0..{GENERATED}")
    t0 = time.time()
    w_cpu = sq.make_weights(shape, seed=0)
    w = {k: v.to(dev) for k, v in w_cpu.items()}
    t_gen = time.time() - t0
    tokens_cpu = sq.make_tokens(shape, 1, S, [PROMPT], seed=0)
    ls = args.local_schedulers
    W = args.workers or (load().mpk_device_sm_count() - ls // 4)
    dec = build_decoder(shape, w, requests=1, max_seq=S, num_workers=W, num_local_schedulers=ls,
                        attn_chunks=args.attn_chunks or None, sched_lookahead=args.lookahead,
                        profiling=args.profiling, prefetch_kb=args.prefetch_kb,
                        fused_attention={"auto": None, "fused": True, "split": False}[args.attention],
                        dynamic_tasks=args.claim_tasks, tasks_per_worker=args.tasks_per_worker)
    # the prompt's graph: PREFILL_TOKENS positions per iteration on the tensor
    # cores, sharing the decode graph's weights and KV cache
    pre = build_decoder(shape, w, requests=1, max_seq=S, num_workers=W, num_local_schedulers=ls,
                        prefill_tokens=PREFILL_TOKENS, k_cache=dec.k_cache, v_cache=dec.v_cache)
    stream = torch.cuda.current_stream(dev)
    tok = tokens_cpu.to(dev)
    step = torch.zeros(1, dtype=torch.int32, device=dev)
    end = lambda n: torch.full((1,), n, dtype=torch.int32, device=dev)
    # prompt (prefill), then warm-up iterations
    pre.run(step, tok, end(PROMPT - 1))
    dec.run(step, tok, end(PROMPT - 1 + args.warmup))
    torch.cuda.synchronize(dev)
    dec.kernel.check_status()
    # rewind to the end of the prompt: positions >= PROMPT are regenerated
    tok.copy_(tokens_cpu.to(dev))
    step.fill_(PROMPT - 1)
    stop = end(PROMPT - 1 + args.steps)
    barrier(pg, dev)
    torch.cuda.synchronize(dev)
    clk = ClockSampler(local)
    clk.start()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    dec.run(step, tok, stop, stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = clk.stop()
    barrier(pg, dev)
    dec.kernel.check_status()
    ms_launch = e0.elapsed_time(e1)
    assert int(step.item()) == PROMPT - 1 + args.steps
    gen = tok[0, PROMPT:PROMPT + args.steps].cpu()
    assert bool((gen >= 0).all()), "some timed tokens were not generated"
    ms_max = max_over_ranks(pg, ms_launch, dev)
    value, tokens_per_s = whole_job(ms_max, args.steps, world)
    ms_per_step = ms_max / args.steps
    bytes_launch = algorithmic_bytes(shape, PROMPT - 1, args.steps)
    gbs = bytes_launch / (ms_launch * 1e-3) / 1e9
    peak, peak_kind = measured_peaks()

    timeline_stats = None
    if args.profiling:
        tl = dec.kernel.timeline()
        if args.timeline_out:
            write_chrome_trace(tl, dec, args.timeline_out)
        op_kind.per_layer = (dec.kernel.num_ops() - 2) // shape.layers
        timeline_stats = timeline_summary(tl, shape)

    op_ms = None
    if args.op_by_op:
        tok.copy_(tokens_cpu.to(dev))
        step.fill_(PROMPT - 1)
        torch.cuda.synchronize(dev)
        o0 = torch.cuda.Event(enable_timing=True)
        o1 = torch.cuda.Event(enable_timing=True)
        o0.record(stream)
        dec.run_op_by_op(step, tok, stop, stream)
        o1.record(stream)
        torch.cuda.synchronize(dev)
        op_ms = o0.elapsed_time(o1) / args.steps
        dec.kernel.check_status()

    # end to end through the public API with host buffers.  Prompt ingestion is
    # one launch, timed on its own: H2D of the prompt, its PROMPT - 1 positions
    # through the prefill graph (for comparison also as PROMPT - 1 decode
    # iterations).  The decode window is the headline: H2D of tokens / step /
    # step_end from pinned memory, the K generated tokens in one launch, D2H of
    # the tokens; reported per generated token.
    e2e = None
    if not args.no_e2e:
        host_tok = tokens_cpu.clone().pin_memory()
        host_step0 = torch.zeros(1, dtype=torch.int32).pin_memory()
        host_pend = torch.full((1,), PROMPT - 1, dtype=torch.int32).pin_memory()
        host_step = torch.full((1,), PROMPT - 1, dtype=torch.int32).pin_memory()
        host_end = torch.full((1,), PROMPT - 1 + args.steps, dtype=torch.int32).pin_memory()
        out_tok = torch.empty_like(host_tok).pin_memory()
        barrier(pg, dev)
        torch.cuda.synchronize(dev)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
        for k, graph in enumerate((dec, pre)):  # one position per iteration, then the prefill graph
            ev[2 * k].record(stream)
            tok.copy_(host_tok, non_blocking=True)
            step.copy_(host_step0, non_blocking=True)
            stop.copy_(host_pend, non_blocking=True)
            graph.run(step, tok, stop, stream)
            ev[2 * k + 1].record(stream)
            torch.cuda.synchronize(dev)
            graph.kernel.check_status()
        barrier(pg, dev)
        ev[4].record(stream)
        tok.copy_(host_tok, non_blocking=True)
        step.copy_(host_step, non_blocking=True)
        stop.copy_(host_end, non_blocking=True)
        dec.run(step, tok, stop, stream)
        out_tok.copy_(tok, non_blocking=True)
        ev[5].record(stream)
        torch.cuda.synchronize(dev)
        dec.kernel.check_status()
        prompt_decode_ms = max_over_ranks(pg, ev[0].elapsed_time(ev[1]), dev)
        prompt_ms = max_over_ranks(pg, ev[2].elapsed_time(ev[3]), dev)
        e2e_ms = max_over_ranks(pg, ev[4].elapsed_time(ev[5]), dev)
        assert torch.equal(out_tok[0, PROMPT:PROMPT + args.steps], gen), "e2e tokens differ from the timed run"
        h2d = host_tok.numel() * 8 + 4 + 4
        d2h = out_tok.numel() * 8
        e2e = {"value": whole_job(e2e_ms, args.steps, world)[0], "unit": UNIT,
               "h2d_bytes_per_step": h2d / args.steps, "d2h_bytes_per_step": d2h / args.steps,
               "includes": f"H2D of tokens/step/step_end, {args.steps} decode iterations in one launch after the "
                           f"prompt, D2H of tokens",
               "prompt_ingestion_ms": prompt_ms,
               "prompt_ingestion": f"H2D of the {PROMPT}-token prompt, its {PROMPT - 1} positions through the prefill "
                                   f"graph ({PREFILL_TOKENS} per iteration on the tensor cores) in one launch",
               "prompt_ingestion_ms_one_position_per_iteration": prompt_decode_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ms_cpu, n, cores, desc = time_oracle(shape, w_cpu, tokens_cpu, args.cpu_budget_s)
        cpu = {"value": ms_cpu, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": value / A100_MPK_MS, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(shape, args, dec),
            "tokens_per_s": tokens_per_s,
            "hbm_gbs": gbs,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "traffic": (None if traffic_ratio() is None else traffic_ratio() * bytes_launch),
                         "traffic_source": "ncu dram bytes of a 4-layer case scaled by algorithmic bytes",
                         "peak_kind": peak_kind,
                         "algorithmic_bytes_per_launch": bytes_launch, "launch_ms": ms_launch,
                         "kernel": "mpk_persistent_kernel"},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": 1,
            "clocks": clocks,
            "op_by_op_ms_per_token": op_ms,
            "timeline": timeline_stats,
            "setup_s": {"weights": round(t_gen, 1)},
        }
        print(json.dumps(line), flush=True)
    pre.kernel.close()
    dec.kernel.close()
    if pg is not None:
        pg.destroy_process_group()


def op_kind(op: int, shape) -> str:
    last = 1 + op_kind.per_layer * shape.layers
    if op == 0:
        return "embed"
    if op == last:
        return "lmhead_argmax"
    per = 5 if op_kind.per_layer == 5 else 4
    names = (["rmsnorm_qkv", "attention", "o_proj_resid", "rmsnorm_gateup_silu", "down_resid"] if per == 5 else
             ["rmsnorm_qkv_attention", "o_proj_resid", "rmsnorm_gateup_silu", "down_resid"])
    return names[(op - 1) % per]


op_kind.per_layer = 5


def timeline_summary(tl, shape) -> dict:
    """Per operation kind, means over tasks (us): wait = popped -> dependency met,
    pro = dependency met -> prologue done, data = prologue done -> first weight
    stage ready, lead = first stage issued -> dependency met (how early the
    producer started on the task's weights), work = dependency met -> done,
    stall = time the consumers waited for weight stages, tail = last stage
    ready -> done;
    span = first dependency met -> last task done of the operation, gap = last
    task of the previous operation done -> first dependency met here."""
    import collections
    if tl.shape[0] == 0:
        return {"records": 0}
    recs = tl.tolist()
    by_op = collections.defaultdict(list)
    for rec in recs:
        it, op = (rec[0] >> 32) & 0xFFFFFFFF, (rec[0] >> 16) & 0xFFFF
        by_op[(it, op)].append(rec)
    keys = sorted(by_op)
    first_it = keys[0][0]
    acc = collections.defaultdict(lambda: collections.defaultdict(list))
    prev_end = None
    for it, op in keys:
        rows = by_op[(it, op)]
        k = op_kind(op, shape)
        ready0 = min(r[3] for r in rows)
        end1 = max(r[4] for r in rows)
        a = acc[k]
        for r in rows:
            _, _, tp, tr, te, tpro, tdat, tiss, tstall, tlast, tloop = r
            a["wait"].append((tr - tp) / 1e3)
            a["work"].append((te - tr) / 1e3)
            if tpro:
                a["pro"].append((tpro - tr) / 1e3)
            if tdat and tpro:
                a["data"].append((max(tdat, tpro) - tpro) / 1e3)
            if tiss:
                a["lead"].append((tr - tiss) / 1e3)
            if tlast:
                a["stall"].append(tstall / 1e3)
                a["tail"].append((te - tlast) / 1e3)
        a["span"].append((end1 - ready0) / 1e3)
        if prev_end is not None and it > first_it:
            a["gap"].append((ready0 - prev_end) / 1e3)
        prev_end = end1
    out = {"records": len(recs)}
    for k, a in acc.items():
        out[k] = {m: round(sum(v) / len(v), 2) for m, v in a.items() if v}
    iters = sorted({k[0] for k in keys})
    if len(iters) > 2:
        t_it = [min(r[3] for (i2, o), rs in by_op.items() if i2 == it for r in rs) for it in iters]
        out["iteration_us"] = round((t_it[-1] - t_it[1]) / (len(iters) - 2) / 1e3, 2)
    return out


def write_chrome_trace(tl, dec, path):
    """Per-task timeline as Chrome-trace JSON (one row per worker)."""
    ev = []
    if tl.shape[0] == 0:
        return
    t0 = int(tl[:, 2].min())
    for rec in tl.tolist():
        entry, worker, ts, tr, te = rec[:5]
        it, op, task = (entry >> 32) & 0xFFFFFFFF, (entry >> 16) & 0xFFFF, entry & 0xFFFF
        ev.append({"name": f"op{op}", "ph": "X", "pid": 0, "tid": int(worker), "ts": (ts - t0) / 1e3,
                   "dur": max(te - ts, 0) / 1e3,
                   "args": {"iter": it, "task": task, "wait_us": (tr - ts) / 1e3,
                            "pro_us": (rec[5] - tr) / 1e3 if rec[5] else 0.0, "stall_us": rec[8] / 1e3,
                            "tail_us": (te - rec[9]) / 1e3 if rec[9] else 0.0,
                            "rows_done_us": (rec[10] - tr) / 1e3 if rec[10] else 0.0}})
    with open(path, "w") as f:
        json.dump({"traceEvents": ev}, f)


if __name__ == "__main__":
    main()
