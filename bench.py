"""Benchmark of the layer-streamed LoRA training step (forward + backward) on B200 GPUs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one call of the library's step through its C ABI: embedding, every decoder layer copied
from the pinned host arena through the two-buffer device pool (2L layer reads), forward, LM head +
cross-entropy, recompute + backward of every layer, LoRA gradients. Inputs are seeded synthetic
weights / tokens of the workload's shape (no dataset, no trained weights).

Prints ONE JSON line (rank 0). For N > 1 (torchrun, one process per GPU) every rank runs its own
replica of the workload on its own GPU and PCIe link and the LoRA gradients are all-reduced over
NCCL after each step (data parallel); the time is the max over ranks.

--impl reference times the CPU oracle (tests' reference implementation) on this host's cores, on
a bounded sample of the same workload, and reports the same metric.
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

METRIC = "streamed LoRA fwd+bwd tokens/sec on 1 B200; % of PCIe/HBM/tensor roofline"
UNIT = "tokens/s"


# ---------------------------------------------------------------------------------------- setup
def workload(name: str):
    import synthetic as syn
    return syn.WORKLOADS[name]


def describe(wl) -> str:
    base = "NF4 (double-quant) base" if wl.base_format == "nf4" else "bf16 base"
    head = f", vocab {wl.vocab} head + CE" if wl.vocab else ", no head (loss = sum(x_L * G))"
    return (f"{wl.name}: {wl.n_layers} x decoder layer d{wl.d_model} h{wl.n_heads}/{wl.n_kv_heads} "
            f"hd{wl.head_dim} ffn{wl.ffn}, {base} streamed from pinned host, LoRA r{wl.lora_rank} "
            f"a{int(wl.lora_alpha)} on 7 projections{head}, batch {wl.batch} x seq {wl.seq}")


# DRAM traffic of the GEMMs of one llama8b step, from small ncu captures: for each GEMM shape of
# the step, one launch of `kernel_cases.py <shape>` (dram__bytes_read.sum + dram__bytes_write.sum),
# times the launches of that shape in a step (kernel_cases.GEMM_LAUNCHES_PER_STEP). The figures
# belong to the GEMM sources whose hashes are recorded with them; with other sources bench.py
# reports the traffic as null. Commands and values: profiles/gemm_traffic_llama8b_shapes.md.
GEMM_TRAFFIC = {"workload": "llama8b",
                "bytes_per_launch": {"gemm_qkv": 74810624, "gemm_o": 92734208, "gemm_gu": 356411136,
                                     "gemm_down": 298519808, "gemm_dx_down": 217685504, "gemm_dx_gu": 509340416,
                                     "gemm_dx_o": 52140032, "gemm_dx_qkv": 92449536, "gemm_head": 2111525120,
                                     "gemm_dx_head": 2577441536},
                "sources": {"gemm.cu": "25fb8f9c5e07d9da", "gemm.cuh": "bfa9880e2fabba28",
                            "common.cuh": "704b7549d8511a32", "pdl.cuh": "9d27364b6fccf4eb"}}


def gemm_traffic(wl_name: str):
    """(average DRAM bytes per GEMM launch, bytes per step) of the recorded per-shape captures, or
    (None, None) when the workload differs, nothing is recorded or the GEMM sources changed."""
    import hashlib
    from kernel_cases import GEMM_LAUNCHES_PER_STEP
    rec = GEMM_TRAFFIC
    if wl_name != rec["workload"] or not rec["bytes_per_launch"] or not rec["sources"]:
        return None, None
    csrc = os.path.join(ROOT, "layer_streamed_qlora_streaming_b200", "csrc")
    for f, h in rec["sources"].items():
        with open(os.path.join(csrc, f), "rb") as fh:
            if hashlib.sha256(fh.read()).hexdigest()[:16] != h:
                return None, None
    per_step = sum(rec["bytes_per_launch"][c] * n for c, n in GEMM_LAUNCHES_PER_STEP.items())
    return per_step / sum(GEMM_LAUNCHES_PER_STEP.values()), per_step


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def h2d_peak_gbs(torch) -> float:
    """Pinned host -> device copy bandwidth of this GPU's link (1 GiB, best of 5, CUDA events)."""
    n = 1 << 30
    h = torch.empty(n, dtype=torch.uint8).pin_memory()
    d = torch.empty(n, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    best = 0.0
    for i in range(7):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(s):
            e0.record(s)
            d.copy_(h, non_blocking=True)
            e1.record(s)
        s.synchronize()
        if i >= 2:
            best = max(best, n / (e0.elapsed_time(e1) * 1e-3) / 1e9)
    del h, d
    return best


def build_context(wl, torch, stream, seed: int = 1234, streamed: bool = True):
    """Library context with every layer registered from device-resident synthetic weights."""
    import layer_streamed_qlora_streaming_b200 as lst
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    dev = "cuda"

    def normal(shape, std):
        return torch.randn(shape, generator=g, device=dev, dtype=torch.float32) * std

    def uniform(shape, b):
        return (torch.rand(shape, generator=g, device=dev, dtype=torch.float32) * 2 - 1) * b

    cfg = lst.make_config(wl, streamed=streamed)
    if wl.vocab:
        E = normal((wl.vocab, wl.d_model), 0.02)
        H = normal((wl.vocab, wl.d_model), 0.02)
        gf = torch.ones(wl.d_model, device=dev)
        ctx = lst.Context(cfg, E, gf, H, stream=stream)
        del E, H
    else:
        ctx = lst.Context(cfg, stream=stream)
    ones = torch.ones(wl.d_model, device=dev)
    for i in range(wl.n_layers):
        W, A, B = {}, {}, {}
        for p in lst.PROJ:
            out, inp = wl.proj_shape(p)
            W[p] = normal((out, inp), 0.02)
            A[p] = uniform((wl.lora_rank, inp), 1.0 / math.sqrt(inp))
            B[p] = normal((out, wl.lora_rank), 0.01)
        bias = None
        if wl.qkv_bias:
            bias = {p: normal((wl.proj_shape(p)[0],), 0.02) for p in ("q", "k", "v")}
        ctx.register_layer(i, W, A, B, ones, ones, bias)
        del W, A, B, bias
    torch.cuda.synchronize()
    return ctx


def timeline_summary(tl) -> dict:
    """Copy / compute overlap of one profiled step, from the library's per-read timeline: per read
    kind, mean copy, dequant and compute durations; how much of each read's copy ran while the
    compute stream was busy with an earlier read; and the compute stream's idle time waiting for
    copies inside the step."""
    out = {}
    for kind in ("forward", "backward"):
        rows = [r for r in tl if r["kind"] == kind]
        if not rows:
            continue
        def mean(xs):
            xs = [x for x in xs if x is not None]
            return sum(xs) / len(xs) if xs else None
        cp = [r["copy"][1] - r["copy"][0] for r in rows if r["copy"][0] is not None]
        dq = [r["dequant"][1] - r["dequant"][0] for r in rows if r["dequant"][0] is not None]
        cm = [r["compute"][1] - r["compute"][0] for r in rows]
        out[kind] = {"reads": len(rows), "copy_ms": mean(cp), "dequant_ms": mean(dq), "compute_ms": mean(cm)}
    # hidden copy time: the part of each copy interval covered by the compute intervals of the reads
    comp = sorted(r["compute"] for r in tl)
    hidden = total = 0.0
    for r in tl:
        c0, c1 = r["copy"]
        if c0 is None:
            continue
        total += c1 - c0
        for k0, k1 in comp:
            hidden += max(0.0, min(c1, k1) - max(c0, k0))
    # compute-stream gaps between consecutive reads (waiting for a copy or dequant, or the head)
    gaps = [max(0.0, tl[n]["compute"][0] - tl[n - 1]["compute"][1]) for n in range(1, len(tl))]
    out["copy_hidden_frac"] = hidden / total if total else None
    out["compute_gap_ms_total"] = sum(gaps)
    out["first_compute_start_ms"] = tl[0]["compute"][0]
    out["last_compute_end_ms"] = tl[-1]["compute"][1]
    return out


def time_steps(torch, stream, step, steps: int, warmup: int) -> float:
    """ms of `steps` back-to-back calls of step() after `warmup` untimed ones (CUDA events on the
    library's stream, synchronised on both sides)."""
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def sub_workload(name: str, torch, stream, link_gbs: float, steps: int, warmup: int, modes=("streamed",)):
    """tokens/s of one more workload on this GPU in the given modes ("streamed": base in pinned host
    memory, 2L layer copies per step; "resident": base kept on the GPU), the streamed mode's PCIe
    floor and the copy / compute overlap of one profiled step. AdamW inside every step, as the
    main line."""
    import synthetic as syn
    wl = syn.WORKLOADS[name]
    T = wl.tokens
    out = {"workload": describe(wl)}
    for streamed in (m == "streamed" for m in modes):
        ctx = build_context(wl, torch, stream, seed=4321, streamed=streamed)
        ctx.set_optimizer(lr=2e-4)
        g = torch.Generator(device="cpu")
        g.manual_seed(7)
        if wl.vocab:
            toks = torch.randint(0, wl.vocab, (T,), generator=g, dtype=torch.int32).cuda()
            tgts = torch.randint(0, wl.vocab, (T,), generator=g, dtype=torch.int32).cuda()
            step = lambda: ctx.step(toks, tgts, wl.batch, wl.seq)
        else:
            x = torch.randn(T, wl.d_model, generator=g).to(torch.bfloat16).cuda().view(torch.int16)
            gg = torch.randn(T, wl.d_model, generator=g).to(torch.bfloat16).cuda().view(torch.int16)
            step = lambda: ctx.step_hidden(x, gg, wl.batch, wl.seq)
        ms = time_steps(torch, stream, step, steps, warmup) / steps
        st = ctx.stats()
        entry = {"value": T / (ms * 1e-3), "unit": UNIT, "ms_per_step": ms, "steps": steps, "warmup": warmup,
                 "layer_reads_per_step": st["layer_reads_last_step"], "h2d_bytes_per_step": st["h2d_bytes_last_step"],
                 "layer_blob_bytes": st["blob_bytes"], "base_bytes": st["arena_bytes"]}
        if streamed:
            floor = st["h2d_bytes_last_step"] / (link_gbs * 1e9) * 1e3
            entry.update({"pinned_host_bytes": st["arena_bytes"], "min_ms": floor, "frac": floor / ms})
            ctx.set_profiling(True)
            step()
            torch.cuda.synchronize()
            entry["overlap"] = timeline_summary(ctx.read_timeline())
            ctx.set_profiling(False)
        out["streamed" if streamed else "resident"] = entry
        ctx.close()
        del ctx
        torch.cuda.empty_cache()
    return out


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.p = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.p is not None:
            self.p.terminate()
            try:
                self.out, _ = self.p.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.p.kill()
                self.out, _ = self.p.communicate()

    def summary(self) -> dict:
        rows = []
        for line in (self.out or "").strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), f[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------------------- CPU oracle
def oracle_sample(wl, seq: int = 512):
    """Time the CPU oracle on a bounded sample of the workload: one decoder layer (forward,
    recompute, backward; streamed schedule) and the head at batch 1 x seq tokens. Returns
    (tokens/s extrapolated to the whole workload, seconds of CPU work, description)."""
    import numpy as np
    from oracle import model as M

    rng = np.random.default_rng(7)
    T = seq
    lw = wl.with_(n_layers=1, vocab=0, batch=1, seq=seq)
    raw = [{"W": {p: (rng.standard_normal(lw.proj_shape(p), dtype=np.float32) * 0.02) for p in M.PROJ},
            "A": {p: rng.uniform(-1, 1, (lw.lora_rank, lw.proj_shape(p)[1])).astype(np.float32) /
                  math.sqrt(lw.proj_shape(p)[1]) for p in M.PROJ},
            "B": {p: (rng.standard_normal((lw.proj_shape(p)[0], lw.lora_rank), dtype=np.float32) * 0.01)
                  for p in M.PROJ},
            "attn_norm": np.ones(lw.d_model, np.float32), "mlp_norm": np.ones(lw.d_model, np.float32),
            "bias": ({p: rng.standard_normal(lw.proj_shape(p)[0], dtype=np.float32) * 0.02
                      for p in ("q", "k", "v")} if lw.qkv_bias else None)}]
    x = rng.standard_normal((T, lw.d_model), dtype=np.float32)
    G = rng.standard_normal((T, lw.d_model), dtype=np.float32)
    t0 = time.perf_counter()
    M.step(lw, raw_layers=raw, x_in=x, G=G, schedule="streamed")
    t_layer = time.perf_counter() - t0
    t_head = 0.0
    if wl.vocab:
        H = rng.standard_normal((wl.vocab, wl.d_model), dtype=np.float32) * 0.02
        y = rng.integers(0, wl.vocab, T)
        t0 = time.perf_counter()
        loss, logits, hc = M.head_fwd(x.astype(np.float64), np.ones(wl.d_model), H.astype(np.float64), y,
                                      wl.rms_eps)
        M.head_bwd(hc, logits, np.ones(wl.d_model), H.astype(np.float64), y)
        t_head = time.perf_counter() - t0
    step_s = wl.n_layers * t_layer + t_head
    desc = (f"oracle (numpy fp64) on batch 1 x seq {seq}: one decoder layer fwd+recompute+bwd "
            f"({t_layer:.2f} s) x {wl.n_layers} layers" + (f" + head and CE ({t_head:.2f} s)" if wl.vocab else "")
            + "; tokens/s = tokens / extrapolated step time")
    return T / step_s, t_layer + t_head, desc


def oracle_sample_threads(wl, seq: int, threads: int):
    """oracle_sample with the BLAS thread pool limited to `threads` (None: as configured)."""
    if threads is None:
        return oracle_sample(wl, seq=seq)
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=threads):
        return oracle_sample(wl, seq=seq)


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = max((i.get("num_threads", 0) for i in info), default=0)
        if n:
            return int(n)
    except Exception:
        pass
    return os.cpu_count() or 1


# ---------------------------------------------------------------------------------------- ranks
def max_over_ranks(ms: float, dist, device) -> float:
    """The slowest rank's time (every rank calls this at the same point)."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def allreduce_grads(grads, dist) -> None:
    """Data-parallel exchange: average the LoRA gradients of all replicas (NCCL on GPUs), so every
    replica applies the same update. The sum runs in a fixed order (rank 0, 1, ..., N-1), whatever
    algorithm the collective library picks, so every replica and every run gets the same bytes:
    rank q gathers shard q of every replica's gradient (all-to-all), adds the N copies in rank
    order, and the reduced shards are then gathered by everyone (all-gather)."""
    if dist is None:
        return
    import torch
    N = dist.get_world_size()
    n = grads.numel()
    shard = -(-n // N)
    g = torch.nn.functional.pad(grads, (0, shard * N - n)) if shard * N != n else grads
    parts = torch.empty_like(g)
    dist.all_to_all_single(parts, g)              # parts[q] = replica q's copy of my shard
    parts = parts.view(N, shard)
    acc = parts[0].clone()
    for q in range(1, N):
        acc += parts[q]
    acc /= N
    out = torch.empty(N * shard, dtype=grads.dtype, device=grads.device)
    dist.all_gather_into_tensor(out, acc)
    grads.copy_(out[:n])


def job_throughput(world: int, tokens_per_step: int, steps: int, ms: float) -> float:
    """Whole-job tokens/s: every rank processes its own batch each step."""
    return world * tokens_per_step * steps / (ms * 1e-3)


# ---------------------------------------------------------------------------------------- arms
def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    for _ in range(args.warmup):
        oracle_sample(wl, seq=args.ref_seq)
    vals, secs, desc = [], [], ""
    for _ in range(args.steps):
        v, sec, desc = oracle_sample(wl, seq=args.ref_seq)
        vals.append(v)
        secs.append(sec)
    value = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            # each step is a bounded sample of the workload, timed as it ran; the metric is the
            # whole workload's tokens over the step time extrapolated from the sample
            "ms_per_step": statistics.median(secs) * 1e3, "extrapolated": True,
            "extrapolated_ms_per_step": wl.tokens / value * 1e3,
            "sample_shape": {"layers": 1, "batch": 1, "seq": args.ref_seq, "head": bool(wl.vocab)},
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": describe(wl), "batch": wl.batch, "seq": wl.seq},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_gpu(args, wl):
    import torch
    import layer_streamed_qlora_streaming_b200 as lst

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    # above the library's prep stream, so the next read's dequant only takes SM slots this leaves free
    stream = torch.cuda.Stream(priority=-1)
    link_gbs = h2d_peak_gbs(torch)
    ctx = build_context(wl, torch, stream, seed=1234 + rank)
    split = world > 1 and args.split_copy
    if split:
        # every rank copies 1/N of each layer blob over its own link; NCCL all-gathers the rest
        uid = [lst.nccl_unique_id() if rank == 0 else b""]
        dist.broadcast_object_list(uid, src=0)
        ctx.set_split_copy(rank, world, uid[0])
    if not args.no_optimizer:
        # one process: the step applies AdamW itself; replicas: after the gradient average
        ctx.set_optimizer(lr=2e-4, deferred=world > 1)
    n_grad = ctx.lora_numel()
    lora0 = torch.empty(n_grad, dtype=torch.float32, device="cuda")
    ctx.get_lora(lora0)              # initial adapters, restored before the DPO measurement
    grads = torch.zeros(n_grad, dtype=torch.float32, device="cuda")
    g = torch.Generator(device="cpu")
    g.manual_seed(99 + rank)
    T = wl.tokens
    if wl.vocab:
        toks = torch.randint(0, wl.vocab, (T,), generator=g, dtype=torch.int32)
        tgts = torch.randint(0, wl.vocab, (T,), generator=g, dtype=torch.int32)
        toks_d, tgts_d = toks.cuda(), tgts.cuda()

        def step(gr):
            return ctx.step(toks_d, tgts_d, wl.batch, wl.seq, gr)
    else:
        xg = (torch.randn(T, wl.d_model, generator=g)).to(torch.bfloat16)
        gg = (torch.randn(T, wl.d_model, generator=g)).to(torch.bfloat16)
        x_d, g_d = xg.cuda().view(torch.int16), gg.cuda().view(torch.int16)

        def step(gr):
            return ctx.step_hidden(x_d, g_d, wl.batch, wl.seq, gr)

    def exchange_and_update():
        if dist is None:
            return
        with torch.cuda.stream(stream):
            allreduce_grads(grads, dist)
        if not args.no_optimizer:
            ctx.apply_optimizer(grads)   # the replicas' mean gradient, on the context's stream

    def one_step():
        loss = step(grads)
        exchange_and_update()
        return loss

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    # timed region: K steps bracketed by barrier + synchronize, CUDA events on the step stream
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            loss = one_step()
        e1.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), dist, "cuda")
    # per-class device times: K more steps with CUDA events around every launch of a class
    ctx.set_profiling(True)
    agg = {k: 0.0 for k in ("gemm_ms", "attention_ms", "dequant_ms", "lora_ms", "copy_ms", "gemm_flops",
                            "gemm_launches", "launches_last_step", "h2d_bytes_last_step", "step_ms")}
    for _ in range(args.steps):
        one_step()
        st = ctx.stats()
        for k in agg:
            agg[k] += st[k]
    torch.cuda.synchronize()
    overlap = timeline_summary(ctx.read_timeline())
    ctx.set_profiling(False)
    value = job_throughput(world, T, args.steps, ms)

    # end to end: host tokens in (pinned), host loss and gradients out, inside the timed region
    hg = torch.zeros(n_grad, dtype=torch.float32).pin_memory()
    if wl.vocab:
        ht, hy = toks.pin_memory(), tgts.pin_memory()
        host_step = lambda: ctx.step(ht, hy, wl.batch, wl.seq, hg)
        h2d = 2 * T * 4
    else:
        hx, hgg = xg.view(torch.int16).pin_memory(), gg.view(torch.int16).pin_memory()
        host_step = lambda: ctx.step_hidden(hx, hgg, wl.batch, wl.seq, hg)
        h2d = 2 * T * wl.d_model * 2
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    f0.record(stream)
    for _ in range(args.steps):
        host_step()
    f1.record(stream)
    torch.cuda.synchronize()
    ems = max_over_ranks(f0.elapsed_time(f1), dist, "cuda")
    e2e = {"value": job_throughput(world, T, args.steps, ems), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": n_grad * 4 + 4,
           "path": "lst_step with pinned host inputs and host gradient buffer (copies inside the call)"}

    # the reuse schedule (layers still in the pool are not copied again): same results, fewer bytes
    ctx.set_reuse(True)
    for _ in range(2):
        one_step()
    torch.cuda.synchronize()
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    r0.record(stream)
    for _ in range(args.steps):
        one_step()
    r1.record(stream)
    torch.cuda.synchronize()
    rms = max_over_ranks(r0.elapsed_time(r1), dist, "cuda")
    rst = ctx.stats()
    ctx.set_reuse(False)
    reuse_bytes = rst["h2d_bytes_last_step"]
    reuse = {"value": job_throughput(world, T, args.steps, rms), "unit": UNIT, "ms_per_step": rms / args.steps,
             "layer_reads_per_step": rst["layer_reads_last_step"], "h2d_bytes_per_step": reuse_bytes,
             "min_ms": reuse_bytes / (link_gbs * 1e9) * 1e3,
             "frac": reuse_bytes / (link_gbs * 1e9) * 1e3 / (rms / args.steps),
             "note": "steady state: the two layers at the forward/backward turn and layers 0, 1 from the "
                     "previous step are not copied again (2L - 4 reads)"}

    # the same 2L copies without copying the next step's first read ahead (A/B of that overlap)
    ctx.set_prefetch(False)
    for _ in range(2):
        one_step()
    torch.cuda.synchronize()
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    p0.record(stream)
    for _ in range(args.steps):
        one_step()
    p1.record(stream)
    torch.cuda.synchronize()
    pms = max_over_ranks(p0.elapsed_time(p1), dist, "cuda")
    pst = ctx.stats()
    ctx.set_prefetch(True)
    no_prefetch = {"value": job_throughput(world, T, args.steps, pms), "unit": UNIT, "ms_per_step": pms / args.steps,
                   "layer_reads_per_step": pst["layer_reads_last_step"],
                   "frac": pst["h2d_bytes_last_step"] / (link_gbs * 1e9) * 1e3 / (pms / args.steps),
                   "note": "every step copies its own first read at its start instead of the step before copying "
                           "it during its last layer and the optimizer"}

    dpo = None
    if wl.vocab and wl.batch % 2 == 0:
        # DPO step on the same model: reference forward with the adapters off + policy step (3L reads)
        dmask = torch.zeros(wl.batch, wl.seq, dtype=torch.int32)
        dmask[:, wl.seq // 2:] = 1                       # response half counts, prompt half does not
        dtoks, dtgts = toks.clone().view(wl.batch, wl.seq), tgts.clone().view(wl.batch, wl.seq)
        P = wl.batch // 2
        dtoks[P:, :wl.seq // 2] = dtoks[:P, :wl.seq // 2]  # pair p shares its prompt
        dtgts[P:, :wl.seq // 2] = dtgts[:P, :wl.seq // 2]
        dt, dy, dm = dtoks.reshape(-1).cuda(), dtgts.reshape(-1).cuda(), dmask.reshape(-1).cuda()
        # start from the initial adapters (the SFT steps above trained on the same tokens)
        for (l, pname), ((oa, sa), (ob, sb)) in ctx.grad_slices().items():
            ctx.set_lora(l, lst.PROJ.index(pname), lora0[oa:oa + sa[0] * sa[1]], lora0[ob:ob + sb[0] * sb[1]])
        if not args.no_optimizer:
            ctx.set_optimizer(lr=2e-4, deferred=world > 1)

        def dpo_step():
            loss = ctx.step_dpo(dt, dy, dm, P, wl.seq, 0.1, grads)
            exchange_and_update()
            return loss
        dloss_first = dpo_step()
        dpo_step()
        torch.cuda.synchronize()
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        d0.record(stream)
        for _ in range(args.steps):
            dloss = dpo_step()
        d1.record(stream)
        torch.cuda.synchronize()
        dms = max_over_ranks(d0.elapsed_time(d1), dist, "cuda")
        dst = ctx.stats()
        dbytes = dst["h2d_bytes_last_step"]
        dpo = {"value": job_throughput(world, T, args.steps, dms), "unit": UNIT, "ms_per_step": dms / args.steps,
               "layer_reads_per_step": dst["layer_reads_last_step"], "h2d_bytes_per_step": dbytes,
               "min_ms": dbytes / (link_gbs * 1e9) * 1e3, "frac": dbytes / (link_gbs * 1e9) * 1e3 / (dms / args.steps),
               "pairs": P, "beta": 0.1, "loss_first": dloss_first, "loss_last": dloss,
               "note": "DPO: reference forward with the adapters off, then the policy forward, head and backward "
                       "(3L reads); tokens/s counts the 2P sequences once; starts from the initial adapters, "
                       "whose B != 0 already separates policy and reference; the same pairs every step, so "
                       "the loss falls fast under AdamW"}

    st = ctx.stats()
    peaks = measured_peaks()
    traffic_launch, traffic_step = gemm_traffic(args.workload)
    K = args.steps
    gemm_ms = agg["gemm_ms"] / K
    gemm_tflops = agg["gemm_flops"] / K / (gemm_ms * 1e-3) / 1e12 if gemm_ms > 0 else 0.0
    peak_t = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    step_ms = ms / K
    h2d_bytes = agg["h2d_bytes_last_step"] / K
    pcie_ms = h2d_bytes / (link_gbs * 1e9) * 1e3
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded torch.randn weights / uniform tokens)",
        "config": {"workload": describe(wl), "batch": wl.batch, "seq": wl.seq, "layers": wl.n_layers,
                   "parallelism": f"dp{world}" if world > 1 else "single GPU",
                   "layer_copies": ("each rank copies 1/N of every layer blob, NCCL all-gathers the blob over "
                                    "NVLink" if split else "every rank copies whole layer blobs over its own link"),
                   "optimizer": "none" if args.no_optimizer else (
                       "AdamW lr 2e-4 on every adapter, inside the step" if world == 1 else
                       "AdamW lr 2e-4 on every adapter with the replicas' mean gradient (NCCL all-reduce)"),
                   "l2": "not flushed: every step streams all layer blobs (GBs) through HBM, far above the 126 MB L2",
                   "loss_last": loss},
        "roofline": {"bound": "tensor", "kernel": "tcgen05 bf16 GEMM (all projection + LM-head GEMMs)",
                     "achieved": gemm_tflops, "peak": peak_t, "unit": "TFLOP/s",
                     "frac": gemm_tflops / peak_t if peak_t else None, "traffic": traffic_launch,
                     "traffic_per_step": traffic_step,
                     "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch of each "
                                       "GEMM shape, times its launches per step (average per launch); null when "
                                       "the GEMM sources differ from those captured",
                     "peak_source": f"{peaks['source']} bf16_tflops_sustained (kernel timed inside a long step)",
                     "gemm_ms_per_step": gemm_ms, "gemm_launches_per_step": agg["gemm_launches"] / K},
        "step_roofline": {"bound": "pcie", "h2d_bytes_per_step": h2d_bytes, "link_gbs": link_gbs,
                          "link_source": "measured in this run: pinned 1 GiB host->device copy",
                          "min_ms": pcie_ms, "frac": pcie_ms / step_ms,
                          "achieved_h2d_gbs": h2d_bytes / (step_ms * 1e-3) / 1e9,
                          "copy_ms_per_step": agg["copy_ms"] / K,
                          "attention_ms_per_step": agg["attention_ms"] / K,
                          "dequant_ms_per_step": agg["dequant_ms"] / K, "lora_ms_per_step": agg["lora_ms"] / K,
                          "profiled_step_ms": agg["step_ms"] / K, "overlap": overlap,
                          "note": "class times from K extra steps with CUDA events around each launch; "
                                  "overlap from the per-read timeline of the last of them"},
        "gpu_launches": int(agg["launches_last_step"] / K * K),
        "memory": {"library_device_bytes": int(st["device_bytes"]), "pinned_host_bytes": int(st["arena_bytes"]),
                   "layer_blob_bytes": int(st["blob_bytes"])},
        "clocks": clk.summary(),
    }
    line["e2e"] = e2e
    line["reuse_schedule"] = reuse
    line["no_prefetch"] = no_prefetch
    if dpo is not None:
        line["dpo"] = dpo
    ctx.close()
    del ctx
    torch.cuda.empty_cache()
    if world == 1 and not args.no_extra and args.workload == "llama8b":
        # the other configurations of the method, each its own context on this GPU in turn
        Ke, We = min(args.steps, 5), 2
        extra = {"note": f"{Ke} timed steps after {We} warm-up each; AdamW inside every step"}
        extra["llama8b_resident"] = sub_workload("llama8b", torch, stream, link_gbs, Ke, We, modes=("resident",))
        r = extra["llama8b_resident"]["resident"]
        r["streamed_over_resident_time"] = step_ms / r["ms_per_step"]
        extra["llama8b_layer"] = sub_workload("llama8b_layer", torch, stream, link_gbs, Ke, We,
                                              modes=("streamed", "resident"))
        e = extra["llama8b_layer"]
        e["streamed_over_resident_time"] = e["streamed"]["ms_per_step"] / e["resident"]["ms_per_step"]
        extra["qwen3b_bf16"] = sub_workload("qwen3b_bf16", torch, stream, link_gbs, Ke, We)
        extra["qwen32b"] = sub_workload("qwen32b", torch, stream, link_gbs, Ke, We)
        line["workloads"] = extra
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, secs, desc = oracle_sample_threads(wl, args.ref_seq, None)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                                "sample": desc, "cpu_seconds": secs}
        v1, secs1, desc1 = oracle_sample_threads(wl, 64, 1)
        line["cpu_baseline"]["one_core"] = {"value": v1, "unit": UNIT, "cores": 1, "sample": desc1,
                                            "cpu_seconds": secs1}
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="llama8b")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-seq", type=int, default=128)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-optimizer", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="time only the main workload")
    ap.add_argument("--split-copy", action="store_true",
                    help="N > 1: each rank copies 1/N of every layer blob, NCCL all-gathers it over NVLink")
    args = ap.parse_args()
    wl = workload(args.workload)
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_gpu(args, wl)


if __name__ == "__main__":
    main()
