"""Benchmark: SeerAttention prefill layer on B200.

One step = the inference hot path of one attention layer on one batch of
synthetic input: AttnGate scores -> per-row TopK mask -> block-sparse causal
attention (GQA).  Default workload: Llama-3.1-8B-shaped layer (32 q-heads,
8 kv-heads, head dim 128) at 32k tokens, TopK density 0.1 (first and diagonal
blocks kept).  Reported value: active-block TFLOP/s of the whole step
(4*64*64*d flops per active (head, query block, key block)), summed over ranks
over the max time across ranks.  With N ranks, either every rank runs its own
layer (--split replicas, weak scaling) or the ranks split one layer by KV-head
group (--split heads, strong scaling; no collective on the data path).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--split heads]

Prints ONE JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse prefill ms/layer & active-block TFLOP/s (% bf16 peak) vs density, 32k"
UNIT = "TFLOP/s"
BLOCK = 64
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def attn_flops(mask_sum: int, d: int) -> float:
    return 4.0 * BLOCK * BLOCK * d * float(mask_sum)


def profile_traffic(kernel_src: str, summary: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current source of the kernel (sha256 recorded in the summary)."""
    path = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(path):
        return None
    sha = hashlib.sha256(open(os.path.join(ROOT, kernel_src), "rb").read()).hexdigest()[:16]
    tb, src = None, None
    for line in open(path):
        if line.startswith("traffic_bytes_per_launch:"):
            tb = float(line.split(":", 1)[1])
        if line.startswith("kernel_source_sha256_16:"):
            src = line.split(":", 1)[1].strip()
    return tb if (tb is not None and src == sha) else None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        # nvidia-smi numbers GPUs physically; identify ours by UUID.
        self.gpu = str(gpu_index)
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(gpu_index).uuid)
            self.gpu = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            pass
        self.proc = None
        self.path = os.path.join("/tmp", f"seer_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# --------------------------------------------------------------------------- GPU arm
def run_gpu(args, world, rank, local):
    import numpy as np
    import torch

    import long_context_prefill_attngate_b200 as seer
    from long_context_prefill_attngate_b200 import build as seer_build
    from long_context_prefill_attngate_b200 import synthetic as syn

    from long_context_prefill_attngate_b200 import partition

    seer_build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w_full = syn.WORKLOADS[args.workload]
    if args.split == "heads" and world > 1:
        # One layer split by KV-head group: every rank draws the same layer and keeps its heads.
        x = partition.slice_layer(syn.make_inputs(w_full), w_full.Hq, w_full.Hkv, world, rank)
        q0, q1, k0, k1 = partition.head_range(w_full.Hq, w_full.Hkv, world, rank)
        w = dataclasses.replace(w_full, Hq=q1 - q0, Hkv=k1 - k0)
    else:
        x = syn.make_inputs(w_full, seed=w_full.seed + 1000 * rank)
        w = w_full
    pk, pk_kind = peaks()
    stream = torch.cuda.current_stream()

    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    wq, wk = x["wq"].to(dev), x["wk"].to(dev)
    nb = w.nb
    sh = seer.shape_of(q, k)
    scores = torch.empty((w.B, w.Hq, nb, nb), dtype=torch.float32, device=dev)
    mask = torch.empty((w.B, w.Hq, nb, nb), dtype=torch.uint8, device=dev)
    o = torch.empty_like(q)
    gws = torch.empty(seer.seer_workspace_bytes(seer.SEER_CALL_GATE_SCORES, sh), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # > 126 MB L2

    def gate_mask(density):
        seer.seer_gate_scores(q, k, wq, wk, rope_theta=w.rope_theta, scores=scores, workspace=gws)
        seer.seer_block_mask(scores, "topk", density=density, mask=mask, Hkv=w.Hkv, d=w.d)

    def attention():
        seer.seer_block_sparse_prefill(q, k, v, mask, o=o)

    def timed_steps(density, steps, warmup, settle_s=0.0):
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
        for _ in range(warmup):
            gate_mask(density)
            attention()
        # Untimed steps until the power-capped clock has settled, so the timed steps
        # measure the steady state rather than the first fraction of a second.
        t_settle = time.time() + settle_s
        while time.time() < t_settle:
            for _ in range(4):
                flush.zero_()
                gate_mask(density)
                attention()
            torch.cuda.synchronize()
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        for s in range(steps):
            flush.zero_()
            e = ev[s]
            e[0].record(stream)
            seer.seer_gate_scores(q, k, wq, wk, rope_theta=w.rope_theta, scores=scores, workspace=gws)
            e[1].record(stream)
            seer.seer_block_mask(scores, "topk", density=density, mask=mask, Hkv=w.Hkv, d=w.d)
            e[2].record(stream)
            attention()
            e[3].record(stream)
        torch.cuda.synchronize()
        barrier(world)
        seer.seer_check_status()
        gate = [e[0].elapsed_time(e[1]) for e in ev]
        msk = [e[1].elapsed_time(e[2]) for e in ev]
        att = [e[2].elapsed_time(e[3]) for e in ev]
        step = [e[0].elapsed_time(e[3]) for e in ev]
        return dict(gate=gate, mask=msk, attn=att, step=step)

    # ---------------- headline: density from args (default 0.1), timed K steps.
    # The clock sampler runs through the headline steps and a repeat of them
    # (same work) so that the sub-second timed region still gets several samples.
    with ClockSampler(local) as clk:
        t_wall0 = time.time()
        res = timed_steps(args.density, args.steps, args.warmup, args.settle_s)
        t_wall = time.time() - t_wall0
        t_end = time.time() + 1.5
        while time.time() < t_end:
            timed_steps(args.density, args.steps, 0)
    clocks = clk.summary()
    mask_sum = int(mask.sum(dtype=torch.int64).item())
    flops = attn_flops(mask_sum, w.d)
    flops_all = sum_over_ranks(flops, world)          # work of all ranks (replicas or head slices)
    density_meas = mask_sum / (w.B * w.Hq * nb * (nb + 1) / 2)
    ms_step = statistics.mean(res["step"])
    ms_attn = statistics.mean(res["attn"])
    ms_gate = statistics.mean(res["gate"])
    ms_mask = statistics.mean(res["mask"])
    ms_step_max = max_over_ranks(ms_step, world)
    value = flops_all / (ms_step_max * 1e-3) / 1e12
    attn_tflops = flops / (ms_attn * 1e-3) / 1e12

    # ---------------- steady state: the same step back to back for about a second
    # (L2 flushed before every step, outside its events), with its own clock record,
    # so the headline can be read against a power-capped steady state.
    steady = None
    if args.steady_steps > 0:
        with ClockSampler(local) as clk2:
            t0 = time.time()
            r2 = timed_steps(args.density, args.steady_steps, 0)
            wall2 = time.time() - t0
        a2 = statistics.mean(r2["attn"])
        st2 = max_over_ranks(statistics.mean(r2["step"]), world)
        steady = {"steps": args.steady_steps, "wall_s": round(wall2, 3), "ms_per_step": round(st2, 4),
                  "value": round(flops_all / (st2 * 1e-3) / 1e12, 2), "ms_layer_attention": round(a2, 4),
                  "attention_active_tflops": round(flops / (a2 * 1e-3) / 1e12, 1),
                  "frac_of_bf16_peak": round(flops / (a2 * 1e-3) / 1e12 / pk["bf16_tflops"], 4),
                  "clocks": clk2.summary()}

    # ---------------- density sweep (attention only; 1.0 is the dense causal point)
    sweep = []
    if not args.no_sweep:
        for dens in w.densities or (1.0, 0.5, 0.3, 0.2, 0.1):
            r = timed_steps(dens, max(3, args.steps // 2), 2)
            ms = statistics.median(r["attn"])
            msum = int(mask.sum(dtype=torch.int64).item())
            fl = attn_flops(msum, w.d)
            ent = {"density_target": dens,
                   "density": round(msum / (w.B * w.Hq * nb * (nb + 1) / 2), 4),
                   "attn_ms": round(ms, 4), "step_ms": round(statistics.median(r["step"]), 4),
                   "active_tflops": round(fl / (ms * 1e-3) / 1e12, 1),
                   "frac_of_bf16_peak": round(fl / (ms * 1e-3) / 1e12 / pk["bf16_tflops"], 4)}
            if dens == 1.0:
                fa = 4.0 * w.S * w.S * w.d * w.Hq * w.B / 2
                ent["fa_convention_tflops"] = round(fa / (ms * 1e-3) / 1e12, 1)
            sweep.append(ent)
        # restore the headline mask for the e2e leg
        gate_mask(args.density)

    # ---------------- pooled-map companion pass (Figure 8) on the same layer
    pooled = None
    if not args.no_map:
        A = torch.empty((w.B, w.Hq, nb, nb), dtype=torch.float32, device=dev)
        mws = torch.empty(seer.seer_workspace_bytes(seer.SEER_CALL_ATTN_POOLED_MAP, sh), dtype=torch.uint8,
                          device=dev)
        om = torch.empty_like(q)
        for _ in range(2):
            seer.seer_attn_pooled_map(q, k, v, o=om, A=A, workspace=mws)
        ts = []
        for _ in range(3):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            seer.seer_attn_pooled_map(q, k, v, o=om, A=A, workspace=mws)
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        seer.seer_check_status()
        fl = attn_flops(w.B * w.Hq * nb * (nb + 1) // 2, w.d)
        ms = statistics.median(ts)
        pooled = {"ms": round(ms, 3), "active_tflops": round(fl / (ms * 1e-3) / 1e12, 1),
                  "frac_of_bf16_peak": round(fl / (ms * 1e-3) / 1e12 / pk["bf16_tflops"], 4)}
        # Distillation loss on the same layer: gate scores vs the row-normalised map.
        seer.seer_gate_scores(q, k, wq, wk, rope_theta=w.rope_theta, scores=scores, workspace=gws)
        for _ in range(3):
            seer.seer_distill_loss(scores, A, Hkv=w.Hkv, d=w.d)
        ts = []
        for _ in range(5):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            seer.seer_distill_loss(scores, A, Hkv=w.Hkv, d=w.d)
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        seer.seer_check_status()
        ms = statistics.median(ts)
        byt = 2 * 4 * w.B * w.Hq * nb * nb + 4 * w.B * w.Hq * nb
        pooled["distill_loss"] = {"ms": round(ms, 4), "gbs": round(byt / (ms * 1e-3) / 1e9, 1),
                                  "frac_of_hbm_peak": round(byt / (ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4)}
        del A, mws, om

    # ---------------- decode step of the last token on the same cache (SeerAttention-R form)
    decode = None
    if not args.no_decode:
        q_tok = q[:, :, -1].contiguous()
        dws = torch.empty(seer.seer_workspace_bytes(seer.SEER_CALL_DECODE_GATE_SCORES, sh), dtype=torch.uint8,
                          device=dev)
        aws = torch.empty(seer.seer_workspace_bytes(seer.SEER_CALL_BLOCK_SPARSE_DECODE, sh), dtype=torch.uint8,
                          device=dev)
        ds = seer.seer_decode_gate_scores(q_tok, k, wq, wk, rope_theta=w.rope_theta, workspace=dws)
        dm = seer.seer_decode_block_mask(ds, "topk", density=args.density)
        do = seer.seer_block_sparse_decode(q_tok, k, v, dm, workspace=aws)
        tg, tm, ta = [], [], []
        for _ in range(10):
            flush.zero_()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            ev[0].record(stream)
            seer.seer_decode_gate_scores(q_tok, k, wq, wk, rope_theta=w.rope_theta, scores=ds, workspace=dws)
            ev[1].record(stream)
            seer.seer_decode_block_mask(ds, "topk", density=args.density, mask=dm)
            ev[2].record(stream)
            seer.seer_block_sparse_decode(q_tok, k, v, dm, o=do, workspace=aws)
            ev[3].record(stream)
            torch.cuda.synchronize()
            tg.append(ev[0].elapsed_time(ev[1]))
            tm.append(ev[1].elapsed_time(ev[2]))
            ta.append(ev[2].elapsed_time(ev[3]))
        seer.seer_check_status()
        # steady state of a decoder: key rows cached, only the last (partial) block's row refreshed
        kt = seer.seer_gate_key_cache(k, wk, rope_theta=w.rope_theta)
        cws = torch.empty(seer.seer_workspace_bytes(seer.SEER_CALL_DECODE_GATE_CACHED, sh), dtype=torch.uint8,
                          device=dev)
        kws = torch.empty(seer.seer_workspace_bytes(seer.SEER_CALL_GATE_KEY_CACHE, sh), dtype=torch.uint8,
                          device=dev)
        tstep = []
        for _ in range(10):
            flush.zero_()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            ev[0].record(stream)
            seer.seer_gate_key_cache(k, wk, kt=kt, first_block=nb - 1, rope_theta=w.rope_theta, workspace=kws)
            seer.seer_decode_gate_scores_cached(q_tok, kt, wq, w.S, w.Hkv, rope_theta=w.rope_theta, scores=ds,
                                               workspace=cws)
            seer.seer_decode_block_mask(ds, "topk", density=args.density, mask=dm)
            seer.seer_block_sparse_decode(q_tok, k, v, dm, o=do, workspace=aws)
            ev[1].record(stream)
            torch.cuda.synchronize()
            tstep.append(ev[0].elapsed_time(ev[1]))
        seer.seer_check_status()
        # the same step replayed from a CUDA graph (how a decoder issues it: no host work per kernel)
        tgraph = None
        try:
            def dstep():
                seer.seer_gate_key_cache(k, wk, kt=kt, first_block=nb - 1, rope_theta=w.rope_theta, workspace=kws)
                seer.seer_decode_gate_scores_cached(q_tok, kt, wq, w.S, w.Hkv, rope_theta=w.rope_theta, scores=ds,
                                                   workspace=cws)
                seer.seer_decode_block_mask(ds, "topk", density=args.density, mask=dm)
                seer.seer_block_sparse_decode(q_tok, k, v, dm, o=do, workspace=aws)
            side = torch.cuda.Stream(device=dev)
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                for _ in range(3):
                    dstep()
            stream.wait_stream(side)
            torch.cuda.synchronize()
            want = do.clone()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, capture_error_mode="relaxed"):
                dstep()
            torch.cuda.synchronize()
            do.zero_()
            graph.replay()
            torch.cuda.synchronize()
            if torch.equal(do, want):
                tg2 = []
                for _ in range(10):
                    flush.zero_()
                    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
                    ev[0].record(stream)
                    graph.replay()
                    ev[1].record(stream)
                    torch.cuda.synchronize()
                    tg2.append(ev[0].elapsed_time(ev[1]))
                tgraph = statistics.median(tg2)
            del graph
        except Exception as exc:   # graph capture is a reporting extra; the eager step above stands
            print(f"decode graph capture skipped: {exc!r}", file=sys.stderr)
        seer.seer_check_status()
        g = w.Hq // w.Hkv
        union = int(dm.view(w.B, w.Hkv, g, nb).amax(2).sum().item())      # (KV head, block) pairs read
        kv_bytes = union * 64 * w.d * 2 * 2
        ms_a = statistics.median(ta)
        decode = {"cache_tokens": w.S, "batch": w.B, "density": round(float(dm.float().mean().item()), 4),
                  "gate_us": round(statistics.median(tg) * 1e3, 1), "mask_us": round(statistics.median(tm) * 1e3, 1),
                  "attention_us": round(ms_a * 1e3, 1), "kv_bytes": kv_bytes,
                  "step_us_cached_keys": round(statistics.median(tstep) * 1e3, 1),
                  "step_us_cached_keys_graph": None if tgraph is None else round(tgraph * 1e3, 1),
                  "attention_gbs": round(kv_bytes / (ms_a * 1e-3) / 1e9, 1),
                  "frac_of_hbm_peak": round(kv_bytes / (ms_a * 1e-3) / 1e9 / pk["hbm_gbs"], 4)}
        del dws, aws, cws, kws, kt

    # ---------------- e2e: pinned host inputs -> C ABI -> host output, per step
    hq, hk, hv = (x[n].pin_memory() for n in ("q", "k", "v"))
    hwq, hwk = x["wq"].pin_memory(), x["wk"].pin_memory()
    ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hwq, hwk))
    d2h = ho.numel() * ho.element_size()
    e2e_steps = max(3, args.steps // 2)

    # The library's host-memory entry (long_context_prefill_attngate_b200.HostPrefill): per KV-head
    # group, H2D of its Q/K/V, gate -> TopK mask -> sparse attention, D2H of its O, on three streams
    # so that the PCIe copies overlap the kernels.
    e2e_ms = e2e_value = None
    if not args.no_e2e:
        hp = seer.HostPrefill(w.B, w.Hq, w.Hkv, w.S, w.d, w.d_gate, device=dev)

        def e2e_step():
            hp.run(hq, hk, hv, hwq, hwk, ho, density=args.density, rope_theta=w.rope_theta)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        seer.seer_check_status()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)
        e2e_value = flops_all / (e2e_ms * 1e-3) / 1e12

    # ---------------- host link: pinned 256 MiB copies each way (what bounds the e2e leg)
    host_link = None
    if not args.no_e2e:
        host_link = measure_host_link(dev, stream)

    # ---------------- CPU baseline: the oracle on a bounded sample (rank 0, N=1).  It runs in
    # a child process that regenerates the same inputs, so this GPU process never loads the oracle.
    cpu_baseline = None
    mask_np = mask.cpu().numpy() if (rank == 0 and world == 1 and not args.no_cpu) else None

    launches_per_step, launches_src = count_step_launches(lambda: (gate_mask(args.density), attention()))

    # ---------------- the other workloads of the benchmark spec, timed in the same run (N=1 only)
    configs = None
    if world == 1 and not args.no_configs:
        del q, k, v, wq, wk, scores, mask, o, gws, x
        torch.cuda.empty_cache()
        configs = run_configs(args, dev, stream, flush, pk)

    if mask_np is not None:
        cpu_baseline = oracle_sample_subprocess(args, mask_np)

    traffic = profile_traffic("long_context_prefill_attngate_b200/csrc/seer_sparse.cu",
                              "attn_sparse_llama8b_32k_d0.1.md")
    # Algorithmic bytes: gate reads Q and K once and writes the scores; the
    # mask reads the causal scores and writes the mask.
    gate_bytes = 2 * (w.B * w.Hq * w.S * w.d + w.B * w.Hkv * w.S * w.d) + 4 * w.B * w.Hq * nb * nb
    mask_bytes = 4 * w.B * w.Hq * nb * (nb + 1) // 2 + w.B * w.Hq * nb * nb
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "settle_s": args.settle_s, "ms_per_step": round(ms_step_max, 4), "higher_is_better": True,
        "scaling": "strong" if (args.split == "heads" and world > 1) else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w_full.name, "B": w_full.B, "Hq": w_full.Hq, "Hkv": w_full.Hkv, "S": w_full.S,
                   "d": w_full.d, "mask": "gate-topk", "density_target": args.density,
                   "density": round(density_meas, 4), "d_gate": w_full.d_gate, "rope_theta": w_full.rope_theta,
                   "l2": "flushed between timed GPU steps (256 MiB write, outside the step events); the host oracle arm has no GPU cache",
                   "parallelism": ("single" if world == 1 else
                                   f"kv-head split x{world}" if args.split == "heads" else f"replicas x{world}")},
        "ms_layer_attention": round(ms_attn, 4), "ms_gate": round(ms_gate, 4), "ms_mask": round(ms_mask, 4),
        "gate_hbm": {"algorithmic_bytes": gate_bytes, "gbs": round(gate_bytes / (ms_gate * 1e-3) / 1e9, 1),
                     "frac_of_hbm_peak": round(gate_bytes / (ms_gate * 1e-3) / 1e9 / pk["hbm_gbs"], 4)},
        "mask_hbm": {"algorithmic_bytes": mask_bytes, "gbs": round(mask_bytes / (ms_mask * 1e-3) / 1e9, 1),
                     "frac_of_hbm_peak": round(mask_bytes / (ms_mask * 1e-3) / 1e9 / pk["hbm_gbs"], 4)},
        "attention_active_tflops": round(attn_tflops, 1),
        "roofline": {"bound": "tensor", "achieved": round(attn_tflops, 1), "peak": pk["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": round(attn_tflops / pk["bf16_tflops"], 4), "traffic": traffic,
                     "peak_kind": f"{pk_kind} bf16 burst (cuBLAS)",
                     "frac_of_sustained": round(attn_tflops / pk["bf16_tflops_sustained"], 4),
                     "kernel": f"sparse_attn_kernel<{w.d}> (seer_block_sparse_prefill)",
                     "algorithmic_flops_per_launch": flops},
        "steady": steady, "density_sweep": sweep, "pooled_map": pooled, "decode": decode, "configs": configs,
        "e2e": None if e2e_value is None else {"value": round(e2e_value, 2), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 3), "host_link": host_link},
        "gpu_launches": launches_per_step * args.steps,
        "gpu_launches_per_step": {"count": launches_per_step, "source": launches_src},
        "clocks": clocks, "cpu_baseline": cpu_baseline, "wall_s_timed_region": round(t_wall, 3),
    }
    if rank == 0:
        print(json.dumps(out), flush=True)


def measure_host_link(dev, stream):
    """Pinned host <-> device copy rate (256 MiB each way, best of 3), GB/s."""
    import torch
    n = 256 << 20
    h = torch.empty(n, dtype=torch.uint8).pin_memory()
    d = torch.empty(n, dtype=torch.uint8, device=dev)
    out = {}
    for name, (dst, src) in (("h2d_gbs", (d, h)), ("d2h_gbs", (h, d))):
        best = None
        for _ in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            dst.copy_(src, non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
            best = ms if best is None else min(best, ms)
        out[name] = round(n / (best * 1e-3) / 1e9, 1)
    del h, d
    return out


def run_configs(args, dev, stream, flush, pk):
    """Time the other workloads of the task on this GPU: the 8k threshold layer,
    the 128k threshold layer (threshold at the 0.83 quantile of one head's causal
    scores, for about 0.17 density) and the Qwen 64k Figure-8 pass."""
    import torch

    import long_context_prefill_attngate_b200 as seer
    from long_context_prefill_attngate_b200 import synthetic as syn

    def timed(fn, reps):
        fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        seer.seer_check_status()
        return statistics.median(ts)

    out = {}
    for name in ("llama8b_8k", "llama8b_128k", "qwen14b_64k_map"):
        w = syn.WORKLOADS[name]
        x = syn.make_inputs(w)
        q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
        nb = w.nb
        sh = seer.shape_of(q, k)
        o = torch.empty_like(q)
        if w.mask_source == "dense-map":
            A = torch.empty((w.B, w.Hq, nb, nb), dtype=torch.float32, device=dev)
            ws = torch.empty(seer.seer_workspace_bytes(seer.SEER_CALL_ATTN_POOLED_MAP, sh), dtype=torch.uint8,
                             device=dev)
            ms = timed(lambda: seer.seer_attn_pooled_map(q, k, v, o=o, A=A, workspace=ws), 3)
            fl = attn_flops(w.B * w.Hq * nb * (nb + 1) // 2, w.d)
            out[name] = {"pass": "Figure-8 (O and A)", "ms": round(ms, 3), "density": 1.0,
                         "active_tflops": round(fl / (ms * 1e-3) / 1e12, 1),
                         "frac_of_bf16_peak": round(fl / (ms * 1e-3) / 1e12 / pk["bf16_tflops"], 4),
                         "A_bytes": A.numel() * 4}
            del A, ws
        else:
            wq, wk = x["wq"].to(dev), x["wk"].to(dev)
            gws = torch.empty(seer.seer_workspace_bytes(seer.SEER_CALL_GATE_SCORES, sh), dtype=torch.uint8,
                              device=dev)
            scores = torch.empty((w.B, w.Hq, nb, nb), dtype=torch.float32, device=dev)
            mask = torch.empty((w.B, w.Hq, nb, nb), dtype=torch.uint8, device=dev)
            ms_gate = timed(lambda: seer.seer_gate_scores(q, k, wq, wk, rope_theta=w.rope_theta, scores=scores,
                                                           workspace=gws), 3)
            if w.threshold is not None:
                thr, how = w.threshold, "fixed"
            else:
                # the 0.83 quantile of head 0's causal scores, from an evenly strided sample
                tri = torch.tril(torch.ones(nb, nb, dtype=torch.bool, device=dev))
                vals = scores[0, 0][tri]
                vals = vals[:: max(1, vals.numel() >> 20)].float()
                thr, how = float(torch.quantile(vals, 1.0 - w.target_density)), "quantile of head 0"
            ms_mask = timed(lambda: seer.seer_block_mask(scores, "threshold", threshold=thr, mask=mask, Hkv=w.Hkv,
                                                         d=w.d), 3)
            msum = int(mask.sum(dtype=torch.int64).item())
            ms_att = timed(lambda: seer.seer_block_sparse_prefill(q, k, v, mask, o=o), 5)
            fl = attn_flops(msum, w.d)
            out[name] = {"mask": f"gate-threshold {thr:.4g} ({how})", "density_target": w.target_density,
                         "density": round(msum / (w.B * w.Hq * nb * (nb + 1) / 2), 4),
                         "ms_gate": round(ms_gate, 4), "ms_mask": round(ms_mask, 4), "ms_attention": round(ms_att, 4),
                         "ms_layer": round(ms_gate + ms_mask + ms_att, 4),
                         "active_tflops": round(fl / (ms_att * 1e-3) / 1e12, 1),
                         "frac_of_bf16_peak": round(fl / (ms_att * 1e-3) / 1e12 / pk["bf16_tflops"], 4)}
            del wq, wk, gws, scores, mask
        del q, k, v, o, x
        torch.cuda.empty_cache()
    return out


def oracle_sample_subprocess(args, mask_np):
    """Run the CPU-baseline leg in a child process (it regenerates the same
    inputs from the workload's seed and reads the benchmark's mask from a file)."""
    import tempfile

    import numpy as np
    with tempfile.NamedTemporaryFile(suffix=".npy", delete=False) as f:
        path = f.name
    try:
        np.save(path, mask_np)
        cmd = [sys.executable, os.path.abspath(__file__), "--cpu-baseline-worker", path, "--workload",
               args.workload, "--cpu-budget", str(args.cpu_budget)]
        r = subprocess.run(cmd, capture_output=True, text=True, timeout=600)
        lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
        if r.returncode != 0 or not lines:
            return {"unavailable": f"cpu baseline child exited {r.returncode}: {r.stderr.strip()[-200:]}"}
        return json.loads(lines[-1])
    finally:
        os.unlink(path)


def cpu_baseline_worker(args):
    import numpy as np
    import torch  # noqa: F401  (synthetic inputs are drawn with torch on the CPU)

    from long_context_prefill_attngate_b200 import synthetic as syn
    w = syn.WORKLOADS[args.workload]
    x = syn.make_inputs(w)
    mask_np = np.load(args.cpu_baseline_worker)
    print(json.dumps(oracle_sample(w, x, mask_np, budget_s=args.cpu_budget)), flush=True)


def count_step_launches(step_fn):
    """Kernels of this library that one step launches, counted from the CUDA
    activity trace of one extra (untimed) step."""
    import torch
    from torch.profiler import ProfilerActivity, profile

    try:
        torch.cuda.synchronize()
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            step_fn()
            torch.cuda.synchronize()
        n = sum(ev.count for ev in prof.key_averages() if "seer::" in ev.key and ev.device_time_total > 0)
        return n, "cuda activity trace of one step (kernels in namespace seer)"
    except Exception as exc:   # the profiler is optional; the count is then the static one
        return 5, f"static count (gate 3 + mask 1 + attention 1); trace unavailable: {exc!r}"[:200]


def oracle_sample(w, x, mask_np, budget_s: float):
    """Time the fp64 oracle on a bounded sample of query blocks of the workload."""
    import numpy as np

    import oracle
    from long_context_prefill_attngate_b200 import synthetic as syn

    oracle.build()
    qb, kb, vb = (syn.bf16_bits(x[n]) for n in ("q", "k", "v"))
    rng = np.random.default_rng(0)
    nb = w.nb
    units, flops, spent = [], 0.0, 0.0
    t0 = time.time()
    # grow the sample until the budget is used (units of 8 query blocks across heads)
    while spent < budget_s:
        batch = np.stack([np.zeros(8, np.int32), rng.integers(0, w.Hq, 8).astype(np.int32),
                          rng.integers(0, nb, 8).astype(np.int32)], 1)
        t = time.time()
        oracle.masked_attention(qb, kb, vb, mask_np, units=batch)
        spent += time.time() - t
        units.append(batch)
        flops += sum(attn_flops(int(mask_np[b, h, i].sum()), w.d) for b, h, i in batch)
        if time.time() - t0 > 3 * budget_s:
            break
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    n = sum(len(u) for u in units)
    # the oracle's gate (a1-a3) in full on the same layer, timed on its own
    t = time.time()
    oracle.gate_scores(qb, kb, syn.bf16_bits(x["wq"]), syn.bf16_bits(x["wk"]), theta=w.rope_theta)
    gate_s = time.time() - t
    return {"value": flops / spent / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n} random (head, query block) units of {w.name} at the benchmark mask "
                      f"(fp64 masked attention, {spent:.1f} s; gate/mask not included)",
            "gate_full_layer_s": round(gate_s, 3)}


# --------------------------------------------------------------------------- reference arm
def run_reference(args, world, rank):
    if rank != 0:
        return
    import numpy as np

    import oracle
    from long_context_prefill_attngate_b200 import synthetic as syn

    oracle.build()
    w = syn.WORKLOADS[args.workload]
    x = syn.make_inputs(w)
    qb, kb, vb = (syn.bf16_bits(x[n]) for n in ("q", "k", "v"))
    # Mask from the oracle's own gate (fp64, cast to fp32 for the selection).
    scores = oracle.gate_scores(qb, kb, syn.bf16_bits(x["wq"]), syn.bf16_bits(x["wk"]), theta=w.rope_theta)
    mask = oracle.block_mask(scores.astype(np.float32), "topk", k_row=oracle.topk_counts(args.density, w.nb))
    del scores
    rng = np.random.default_rng(1)
    per_step = max(1, args.ref_units)

    def step():
        units = np.stack([np.zeros(per_step, np.int32), rng.integers(0, w.Hq, per_step).astype(np.int32),
                          rng.integers(0, w.nb, per_step).astype(np.int32)], 1)
        t = time.time()
        oracle.masked_attention(qb, kb, vb, mask, units=units)
        dt = time.time() - t
        return dt, sum(attn_flops(int(mask[b, h, i].sum()), w.d) for b, h, i in units)

    for _ in range(args.warmup):
        step()
    tt, ff = 0.0, 0.0
    for _ in range(args.steps):
        dt, fl = step()
        tt += dt
        ff += fl
    value = ff / tt / 1e12
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    sample = (f"each step: {per_step} random (head, query block) units of {w.name}, fp64 masked attention "
              f"with the oracle's own gate/TopK mask (computed once, untimed)")
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": tt / args.steps * 1e3,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic",
           "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "S": w.S, "d": w.d,
                      "mask": "gate-topk", "density_target": args.density,
                      "density": round(float(mask.sum()) / (w.B * w.Hq * w.nb * (w.nb + 1) / 2), 4),
                      "d_gate": w.d_gate, "rope_theta": w.rope_theta,
                      "l2": "flushed between timed GPU steps (256 MiB write, outside the step events); the host oracle arm has no GPU cache",
                      "parallelism": "single"},
           "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default="llama8b_32k")
    ap.add_argument("--density", type=float, default=0.1)
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-map", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-memory leg (profiling runs only)")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-units", type=int, default=16)
    ap.add_argument("--split", choices=["replicas", "heads"], default="replicas",
                    help="N>1: every rank its own layer (replicas) or one layer split by KV-head group (heads)")
    ap.add_argument("--steady-steps", type=int, default=500, help="back-to-back steps of the steady-state block")
    ap.add_argument("--settle-s", type=float, default=1.0,
                    help="seconds of untimed steps after the warm-up, before the timed steps")
    ap.add_argument("--no-configs", action="store_true", help="skip the 8k / 128k / Qwen-64k workloads")
    ap.add_argument("--cpu-baseline-worker", default=None, help=argparse.SUPPRESS)
    args = ap.parse_args()
    if args.cpu_baseline_worker:
        cpu_baseline_worker(args)
        return
    if args.warmup < 3 and args.impl == "native":
        args.warmup = 3
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_gpu(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
