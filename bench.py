#!/usr/bin/env python
"""TTT-E2E prefill benchmark on B200: tokens/s and % of bf16 tensor peak in model FLOPs.

One step = one ttt_prefill call over the whole 128K-token sequence of the ~1B
workload (V32000 d2048 L24, last 6 blocks adaptive, H16, k8192, b1024, T131072,
B1), after ttt_reset (a fresh per-sequence copy of W_init: review §7,
Algorithm 1). The step runs every row of the hot path: embedding, the frozen blocks
over all positions, then 128 sequential mini-batch steps of adaptive-block
forward, fused LM-head cross-entropy forward/backward, backward into the
adaptive MLPs and the fused SGD update. Inputs are synthetic (seeded Zipf +
span-copy tokens, N(0, 0.02) weights), resident in HBM for `value`; `e2e`
passes pinned host buffers through the same C-ABI call (H2D of the tokens and
D2H of the losses inside the timed region).

Beside the metric (rank 0, one GPU): decode on the ~125M architecture with its
model-FLOP and HBM fractions, the batched ~125M prefill, the fixed-128K-tokens
sweep, the full-attention comparator, and the key-value-binding variant of the
same workload with its own bounded oracle sample (--no-* flags skip each).

Multi-GPU: replicas only (each rank runs its own independent sequence batch,
no data-path collective; the path's chain W_{i-1} -> W_i is serial), time =
max over ranks; value = tokens of all ranks / that time.

--impl reference times the CPU oracle (test infrastructure) on a bounded
sample of the same workload: the first chunk of 1024 positions.
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
sys.path.insert(0, ROOT)

import synthetic as syn  # noqa: E402

METRIC = "TTT-E2E prefill tokens/s on 1 B200; % of bf16 tensor peak (model FLOPs)"
WORKLOAD = "b1_128k_bf16"


def model_flops(cfg, T=None, B=None):
    """Algorithmic FLOPs of one prefill (forward of all blocks, LM head, backward
    into the adaptive MLPs); recompute, norms and elementwise work not counted.
    Attention pairs P = sum_p min(p+1, k) (review eq. (1)); P_in = pairs inside chunks.
    With the key-value-binding inner loss (review §8, eq. (10)) the adaptive MLP reads
    the key projection (2Td^2 more forward per block), and the update needs no LM-head
    or cross-block backward: per adaptive block, the value projection (2Td^2) and the
    binding MLP's backward into W1t, W2t (3 x 2Td h_t); its forward is the block's."""
    T = cfg.T if T is None else T
    B = cfg.batch if B is None else B
    d, V, L, Lt, h, ht, hs, k, b = (cfg.d, cfg.vocab, cfg.n_layers, cfg.n_ttt, cfg.mlp_hidden, cfg.ttt_hidden,
                                    cfg.static_hidden, cfg.window_k, cfg.minibatch_b)
    p = np.arange(T, dtype=np.float64)
    P = float(np.minimum(p + 1, k).sum())
    n_full = T // b
    P_in = n_full * b * (b + 1) / 2 + (T % b) * ((T % b) + 1) / 2
    fwd = (L - Lt) * (8 * T * d * d + 4 * T * d * h + 4 * d * P) + \
        Lt * (8 * T * d * d + 4 * T * d * (ht + hs) + 4 * d * P) + 2 * T * d * V
    if getattr(cfg, "inner_loss", "e2e") == "kvb":
        return B * (fwd + Lt * (4 * T * d * d + 6 * T * d * ht))
    bwd = 2 * T * d * V
    for j in range(Lt):
        bwd += 4 * T * d * hs + 2 * T * d * ht * (3 if j == 0 else 4)
        if j > 0:
            bwd += 8 * T * d * d + 4 * d * P + 4 * d * P_in
    return B * (fwd + bwd)


def decode_bytes_per_step(cfg, pos):
    """Least HBM bytes one decode token step reads at position pos (bf16): every frozen
    weight once (E, attention, frozen and static MLPs, the shared W_init), each
    sequence's bf16 fast-weight update copies, and each sequence's window of keys and
    values in every layer (min(pos + 1, k) positions)."""
    d, V, L, Lt = cfg.d, cfg.vocab, cfg.n_layers, cfg.n_ttt
    h, ht, hs, B = cfg.mlp_hidden, cfg.ttt_hidden, cfg.static_hidden, cfg.batch
    frozen = V * d + L * 4 * d * d + (L - Lt) * 2 * d * h + Lt * 2 * d * (hs + ht)
    fast = B * Lt * 2 * d * ht
    kv = B * L * 2 * min(pos + 1, cfg.window_k) * d
    return 2 * (frozen + fast + kv)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        return dict(hbm=m["hbm_gbs"], bf16=m["bf16_tflops"], bf16_sustained=m["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.idx)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [s for s, p in zip(sm, power) if p > 0.5 * max(power)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws == 1:
        return None, 0, 0, 1
    import torch.distributed as dist
    import datetime
    rank = int(os.environ["RANK"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    return dist, rank, local, ws


def _max_over_ranks(dist, value, device):
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _sum_over_ranks(dist, value, device):
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def cpu_baseline(cfg, n_tokens=1024):
    """The oracle (as it stands) on the first chunk of the workload: a bounded sample."""
    from oracle import Oracle
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [os.cpu_count()])
    except Exception:  # noqa: BLE001
        cores = os.cpu_count()
    sample = cfg.replace(T=n_tokens, batch=1)
    w = syn.make_weights(sample)
    toks = syn.make_token_batch(sample)
    t0 = time.perf_counter()
    Oracle(sample, w).prefill(toks)
    dt = time.perf_counter() - t0
    return {"value": n_tokens / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"first {n_tokens} positions (one full mini-batch incl. its update) of 1 sequence of the "
                      f"{cfg.name} workload, float64 numpy oracle, {dt:.1f} s"}


def run_reference(args):
    dist, rank, local, ws = _dist()
    if rank != 0:
        return 0
    over = {"T": args.T} if args.T else {}
    if args.inner_loss == "kvb":
        over.update(inner_loss="kvb", eta=args.kvb_eta)
    cfg = syn.config(args.workload, **over)
    per_step = []
    for _ in range(args.warmup):
        pass  # the oracle has no warm-up state; each step is a fresh bounded sample
    for _ in range(args.steps):
        r = cpu_baseline(cfg, n_tokens=args.ref_tokens)
        per_step.append(r)
    v = statistics.median([r["value"] for r in per_step])
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * args.ref_tokens / v,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "tokens_per_step": args.ref_tokens},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": per_step[0]["cores"], "kind": "oracle",
                             "sample": per_step[0]["sample"]},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_decode(T, args, device, peaks):
    """Decode on the ~125M architecture: prefill a prefix, then greedy tokens with an
    update after every b decoded tokens (review Alg. 3). Reported beside the metric, as
    tokens/s, as a fraction of the bf16 peak in model FLOPs (the forward of every decoded
    position and the update of every completed chunk: the prefill count of the decoded
    positions) and as a fraction of HBM bandwidth (decode_bytes_per_step)."""
    import torch
    cfg = syn.config("m125_decode_bf16", **({"T": args.decode_prefix} if args.decode_prefix else {}))
    n = args.decode_n or cfg.decode_n
    w = syn.make_weights(cfg)
    wd = {k: torch.from_numpy(v).to(device) for k, v in w.items()}
    toks = torch.from_numpy(syn.make_token_batch(cfg)).to(device)
    h = T.ttt_create(cfg, wd)
    del wd
    T.ttt_prefill(h, toks)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    T.ttt_decode(h, n, device=device)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    launches = T.ttt_last_launch_count(h)
    flops = model_flops(cfg, T=cfg.T + n) - model_flops(cfg, T=cfg.T)
    nbytes = float(sum(decode_bytes_per_step(cfg, cfg.T + i) for i in range(n)))
    return {"tokens_per_s": cfg.batch * n / (ms / 1e3), "ms_per_token_step": ms / n, "batch": cfg.batch,
            "prefix": cfg.T, "n": n, "updates": (cfg.T + n) // cfg.minibatch_b - cfg.T // cfg.minibatch_b,
            "gpu_launches": launches,
            "model_flops": {"tflop": flops / 1e12, "achieved_tflops": flops / (ms / 1e3) / 1e12,
                            "frac_of_peak": flops / (ms / 1e3) / 1e12 / peaks["bf16"]},
            "hbm": {"bytes_per_token_step": nbytes / n, "achieved_gbs": nbytes / (ms / 1e3) / 1e9,
                    "peak_gbs": peaks["hbm"], "frac": nbytes / (ms / 1e3) / 1e9 / peaks["hbm"],
                    "floor_ms_per_token_step": nbytes / n / (peaks["hbm"] * 1e9) * 1e3}}


def _time_prefill(T, h, tok, loss, steps, warmup, check=True):
    """Device time (ms) of `steps` reset+prefill calls after `warmup` untimed ones."""
    import torch
    for _ in range(warmup):
        T.ttt_reset(h)
        T.ttt_prefill(h, tok, loss)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        T.ttt_reset(h)
        T.ttt_prefill(h, tok, loss)
    e1.record()
    torch.cuda.synchronize()
    if check:
        assert torch.isfinite(loss).all().item(), "non-finite loss"
    return e0.elapsed_time(e1) / steps


def run_batched_prefill(T, args, device, peaks):
    """Prefill of the ~125M model on B = 4 independent sequences of T = 32768 positions,
    each with its own fast weights (review §7, Algorithm 1: a fresh copy of W per
    sequence). Reported beside the metric: the only batched prefill workload."""
    import torch
    cfg = syn.config("m125_bf16")
    w = syn.make_weights(cfg)
    wd = {k: torch.from_numpy(v).to(device) for k, v in w.items()}
    del w
    tok = torch.from_numpy(syn.make_token_batch(cfg)).to(device)
    loss = torch.empty((cfg.batch, cfg.T), dtype=torch.float32, device=device)
    h = T.ttt_create(cfg, wd)
    del wd
    ms = _time_prefill(T, h, tok, loss, args.batched_steps, 1)
    del h
    torch.cuda.empty_cache()
    fl = model_flops(cfg)
    return {"workload": f"{cfg.name}: V{cfg.vocab} d{cfg.d} L{cfg.n_layers} (last {cfg.n_ttt} adaptive) "
                        f"H{cfg.n_heads} k{cfg.window_k} b{cfg.minibatch_b} T{cfg.T} B{cfg.batch}",
            "tokens_per_s": cfg.batch * cfg.T / (ms / 1e3), "ms_per_step": ms, "steps": args.batched_steps,
            "warmup": 1, "model_tflop_per_step": fl / 1e12,
            "frac_of_peak": fl / (ms / 1e3) / 1e12 / peaks["bf16"]}


def run_sweep(T, cfg, args, device, peaks):
    """Fixed 128K tokens per batch, split as 8K x 16, 16K x 8, 32K x 4, 64K x 2 and
    128K x 1 sequences of the ~1B model (technical review Fig. 1 and §11.1 eq. (11):
    prefill seconds per 1K tokens against context length, nearly flat for TTT-E2E).
    Every sequence carries its own fast weights; each point is one prefill call."""
    import torch
    total = cfg.batch * cfg.T
    w = syn.make_weights(cfg)
    wd = {k: torch.from_numpy(v).to(device) for k, v in w.items()}
    del w
    points = []
    for Tp in args.sweep_lengths:
        if total % Tp:
            continue
        B = total // Tp
        pcfg = cfg.replace(T=Tp, batch=B)
        tok = torch.from_numpy(syn.make_token_batch(pcfg)).to(device)
        loss = torch.empty((B, Tp), dtype=torch.float32, device=device)
        h = T.ttt_create(pcfg, wd, max_segment=min(Tp, 32768))
        ms = _time_prefill(T, h, tok, loss, args.sweep_steps, 1)
        fl = model_flops(pcfg)
        points.append({"T": Tp, "B": B, "ms_per_step": ms, "s_per_1k_tokens": ms / 1e3 / (total / 1e3),
                       "tokens_per_s": total / (ms / 1e3), "model_tflop_per_step": fl / 1e12,
                       "frac_of_peak": fl / (ms / 1e3) / 1e12 / peaks["bf16"],
                       "device_bytes": T.ttt_device_bytes(h)})
        del h, tok, loss
        torch.cuda.empty_cache()
    del wd
    torch.cuda.empty_cache()
    return {"tokens_per_step": total, "steps": args.sweep_steps, "warmup": 1, "points": points}


def run_full_attention(cfg, tok_dev, args, device):
    """Comparator of the pages' speed claim (summary "Results": TTT-E2E prefill 2.7x
    faster than full attention at 128K on one H100): the same architecture with no
    adaptive block and full causal attention (window >= T), same tokens, same
    kernels; prefill records the per-position losses. Reported beside the metric."""
    import torch
    import long_context_prefill_ttt_b200 as T
    fcfg = cfg.replace(n_ttt=0, window_k=max(cfg.T, cfg.window_k))
    w = syn.make_weights(fcfg)
    wd = {k: torch.from_numpy(v).to(device) for k, v in w.items()}
    del w
    loss = torch.empty((fcfg.batch, fcfg.T), dtype=torch.float32, device=device)
    h = T.ttt_create(fcfg, wd)
    del wd
    steps = args.comparator_steps
    T.ttt_reset(h)
    T.ttt_prefill(h, tok_dev, loss)  # warm-up
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        T.ttt_reset(h)
        T.ttt_prefill(h, tok_dev, loss)
    e1.record()
    torch.cuda.synchronize()
    assert torch.isfinite(loss).all().item(), "non-finite comparator loss"
    ms = e0.elapsed_time(e1) / steps
    del h
    torch.cuda.empty_cache()
    return {"workload": f"{fcfg.name} without adaptive blocks, full causal attention (k = {fcfg.window_k})",
            "tokens_per_s": fcfg.batch * fcfg.T / (ms / 1e3), "ms_per_step": ms, "steps": steps, "warmup": 1,
            "model_tflop_per_step": model_flops(fcfg) / 1e12}


def run_kvb_variant(cfg, tok_dev, args, device, peaks):
    """The key-value-binding variant (technical review §8, eq. (10); summary,
    "Alternative Derivation"): the same model and tokens, each adaptive block updated
    by its own layer-wise reconstruction loss with frozen theta_K, theta_V instead of
    the next-token loss. The pages give no step size for it; its squared error sums
    over d outputs, so the step that suits the next-token loss diverges at this width,
    and --kvb-eta (default 1e-4) sets it. The cost does not depend on it. Reported
    beside the metric."""
    import torch
    import long_context_prefill_ttt_b200 as T
    kcfg = cfg.replace(inner_loss="kvb", eta=args.kvb_eta)
    w = syn.make_weights(kcfg)
    wd = {k: torch.from_numpy(v).to(device) for k, v in w.items()}
    del w
    loss = torch.empty((kcfg.batch, kcfg.T), dtype=torch.float32, device=device)
    h = T.ttt_create(kcfg, wd, max_segment=args.segment)
    del wd
    ms = _time_prefill(T, h, tok_dev, loss, args.kvb_steps, 1, check=False)
    del h
    torch.cuda.empty_cache()
    bad = (~torch.isfinite(loss)).nonzero()
    if bad.numel():
        raise FloatingPointError(f"non-finite loss from position {int(bad[0, 1])} "
                                 f"(chunk {int(bad[0, 1]) // kcfg.minibatch_b})")
    fl = model_flops(kcfg)
    tokens = kcfg.batch * kcfg.T
    return {"workload": f"{kcfg.name} with the key-value-binding inner loss (eta {kcfg.eta})",
            "tokens_per_s": tokens / (ms / 1e3), "ms_per_step": ms, "s_per_1k_tokens": ms / 1e3 / (tokens / 1e3),
            "steps": args.kvb_steps, "warmup": 1, "model_tflop_per_step": fl / 1e12,
            "frac_of_peak": fl / (ms / 1e3) / 1e12 / peaks["bf16"]}


def run_ours(args):
    import torch

    dist, rank, local, ws = _dist()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if dist is not None:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=device)
    import long_context_prefill_ttt_b200 as T

    over = {"T": args.T} if args.T else {}
    if args.inner_loss == "kvb":  # the variant as the measured workload (e.g. for its launch list)
        over.update(inner_loss="kvb", eta=args.kvb_eta)
    cfg = syn.config(args.workload, **over)
    w = syn.make_weights(cfg)
    wd = {k: torch.from_numpy(v).to(device) for k, v in w.items()}
    del w
    toks_np = syn.make_token_batch(cfg, seed=cfg.token_seed + 97 * rank)
    tok_dev = torch.from_numpy(toks_np).to(device)
    loss_dev = torch.empty((cfg.batch, cfg.T), dtype=torch.float32, device=device)
    tok_host = torch.from_numpy(toks_np).pin_memory()
    loss_host = torch.empty((cfg.batch, cfg.T), dtype=torch.float32).pin_memory()
    h = T.ttt_create(cfg, wd, max_segment=args.segment)
    del wd
    torch.cuda.synchronize()

    def step(host=False):
        T.ttt_reset(h)
        if host:
            T.ttt_prefill(h, tok_host, loss_host)
        else:
            T.ttt_prefill(h, tok_dev, loss_dev)
        return T.ttt_last_launch_count(h)

    for _ in range(args.warmup):
        step()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    # timed region of `value`: no instrumentation inside it
    sampler = ClockSampler(local)
    sampler.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches = 0
    e0.record()
    for _ in range(args.steps):
        launches += step()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    clocks = sampler.stop()
    if dist is not None:
        dist.barrier()
    ms_max = _max_over_ranks(dist, ms, device)
    tokens = _sum_over_ranks(dist, float(cfg.batch * cfg.T * args.steps), device)
    value = tokens / (ms_max / 1e3)
    assert torch.isfinite(loss_dev).all().item(), "non-finite loss"

    # per-class kernel timing in a separate pass: CUDA events around every launch of a
    # class on the library's stream (their recording would slow the step above)
    prof, ms_prof = {}, 0.0
    if args.profile_steps > 0:
        T.ttt_profile(h, True)
        e0.record()
        for _ in range(args.profile_steps):
            step()
        e1.record()
        torch.cuda.synchronize()
        ms_prof = e0.elapsed_time(e1)
        prof = T.ttt_profile_read(h)
        T.ttt_profile(h, False)

    # end to end through the same call with pinned host buffers
    e2e_value = None
    if args.e2e_steps > 0:
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(args.e2e_steps):
            step(host=True)
        e1.record()
        torch.cuda.synchronize()
        ms_e2e = _max_over_ranks(dist, e0.elapsed_time(e1), device)
        e2e_value = _sum_over_ranks(dist, float(cfg.batch * cfg.T * args.e2e_steps), device) / (ms_e2e / 1e3)

    # Mean DRAM bytes (read + write) per launch of a kernel class, from one ncu capture of
    # the current kernels (the GEMM launches of one adaptive step, whose shapes do not depend
    # on T; the profile summary under profiles/ names the command). Classes without such a
    # capture, or whose kernels changed since it was taken, report null.
    traffic_per_launch = dict(args.traffic) if cfg.name == "b1_128k_bf16" and cfg.batch == 1 else {}
    peaks = measured_peaks()
    flops_step = model_flops(cfg)
    achieved_model = flops_step * args.steps / (ms / 1e3) / 1e12
    # dominant kernel class by device time
    dom = max(prof, key=lambda c: prof[c]["ms"]) if prof else None
    dp = prof[dom] if prof else {"flops": 0.0, "ms": 0.0}
    ach = dp["flops"] / (dp["ms"] / 1e3) / 1e12 if dp["ms"] > 0 else 0.0
    peak = peaks["bf16_sustained"]
    dev_bytes = T.ttt_device_bytes(h)
    decode = None
    if args.decode and rank == 0 and ws == 1:
        decode = run_decode(T, args, device, peaks)
    batched = None
    if args.batched and rank == 0 and ws == 1:
        batched = run_batched_prefill(T, args, device, peaks)
    sweep = None
    if args.sweep and rank == 0 and ws == 1:
        del h
        torch.cuda.empty_cache()
        h = None
        sweep = run_sweep(T, cfg, args, device, peaks)
    comparator = None
    if args.comparator and rank == 0 and ws == 1:
        del h
        torch.cuda.empty_cache()
        h = None
        comparator = run_full_attention(cfg, tok_dev, args, device)
        comparator["ttt_e2e_speedup"] = value / comparator["tokens_per_s"]
        # the pages' own figure, for context only (another model on another GPU)
        comparator["pages_figure"] = {"ttt_e2e_speedup": 2.7, "context": "128K", "hardware": "1x H100",
                                      "model": "3B", "source": "b-lab.team summary, Results; abstract"}
    kvb = None
    if args.kvb and rank == 0 and ws == 1 and cfg.n_ttt > 0 and cfg.inner_loss == "e2e":
        if h is not None:
            del h
            torch.cuda.empty_cache()
            h = None
        try:
            kvb = run_kvb_variant(cfg, tok_dev, args, device, peaks)
            kvb["ttt_e2e_s_per_1k_tokens"] = (ms_max / args.steps) / 1e3 / (cfg.batch * cfg.T / 1e3)
            if args.cpu_baseline:  # the oracle of the variant on a bounded sample, beside it
                kvb["cpu_baseline"] = cpu_baseline(cfg.replace(inner_loss="kvb", eta=args.kvb_eta),
                                                   n_tokens=args.ref_tokens)
        except Exception as ex:  # the metric above stands without it
            kvb = {"error": f"{type(ex).__name__}: {ex}"}
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{cfg.name}: V{cfg.vocab} d{cfg.d} L{cfg.n_layers} (last {cfg.n_ttt} adaptive) "
                               f"H{cfg.n_heads} h{cfg.mlp_hidden} ({cfg.ttt_hidden}+{cfg.static_hidden}) "
                               f"k{cfg.window_k} b{cfg.minibatch_b} T{cfg.T} B{cfg.batch}"
                               + (f", key-value-binding inner loss (eta {cfg.eta})" if cfg.inner_loss == "kvb" else ""),
                   "tokens_per_step_per_gpu": cfg.batch * cfg.T, "parallelism": f"replicas x{ws}",
                   "device_bytes": dev_bytes,
                   "l2": "no flush: every step streams > 2.5 GB of weights and GBs of activations (L2 126 MB)"},
        "model_flops": {"tflop_per_step": flops_step / 1e12, "achieved_tflops": achieved_model,
                        "frac_of_peak": achieved_model / peaks["bf16"], "peak_tflops": peaks["bf16"],
                        "peak_source": f"{peaks['source']} bf16 burst"},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": int(tok_host.numel() * 4),
                "d2h_bytes_per_step": int(loss_host.numel() * 4)},
        "gpu_launches": launches,
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                     "frac": ach / peak, "traffic": traffic_per_launch.get(dom),
                     "peak_source": f"{peaks['source']} bf16 sustained (kernel timed inside a long step)"},
        "profile": {"steps": args.profile_steps, "ms_per_step": ms_prof / max(1, args.profile_steps),
                    "note": "separate instrumented pass (CUDA events around every launch of a class)",
                    "classes": {c: {"ms_per_step": v["ms"] / args.profile_steps, "share": v["ms"] / ms_prof,
                                    "launches_per_step": v["launches"] / args.profile_steps,
                                    "tflops": (v["flops"] / (v["ms"] / 1e3) / 1e12) if v["ms"] else 0.0}
                                for c, v in prof.items()}},
        "clocks": clocks,
    }
    if decode is not None:
        line["decode"] = decode
    if batched is not None:
        line["batched_prefill"] = batched
    if sweep is not None:
        line["fixed_128k_tokens_sweep"] = sweep
    if comparator is not None:
        line["full_attention_comparator"] = comparator
    if kvb is not None:
        line["kvb_variant"] = kvb
    if rank == 0 and ws == 1 and args.cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, n_tokens=args.ref_tokens)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del h
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--T", type=int, default=0, help="override positions per sequence (quick runs)")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--segment", type=int, default=0, help="frozen-phase segment length (0 = library default)")
    ap.add_argument("--ref-tokens", type=int, default=1024)
    ap.add_argument("--no-decode", dest="decode", action="store_false")
    ap.add_argument("--decode-prefix", type=int, default=0)
    ap.add_argument("--decode-n", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--no-comparator", dest="comparator", action="store_false",
                    help="skip the full-attention comparator (same architecture, no adaptive blocks, k >= T)")
    ap.add_argument("--comparator-steps", type=int, default=2)
    ap.add_argument("--no-kvb", dest="kvb", action="store_false",
                    help="skip the key-value-binding variant beside the metric")
    ap.add_argument("--kvb-steps", type=int, default=2)
    ap.add_argument("--kvb-eta", type=float, default=1e-4)
    ap.add_argument("--inner-loss", default="e2e", choices=["e2e", "kvb"],
                    help="inner loss of the measured workload (kvb: the key-value-binding variant)")
    ap.add_argument("--profile-steps", type=int, default=1,
                    help="steps of the separate instrumented pass that gives the per-class profile")
    ap.add_argument("--no-batched", dest="batched", action="store_false",
                    help="skip the ~125M B=4 T=32768 batched prefill line")
    ap.add_argument("--batched-steps", type=int, default=3)
    ap.add_argument("--no-sweep", dest="sweep", action="store_false",
                    help="skip the fixed-128K-tokens-per-batch sweep (8K x 16 ... 128K x 1)")
    ap.add_argument("--sweep-steps", type=int, default=2)
    ap.add_argument("--sweep-lengths", type=lambda s: [int(x) for x in s.split(",")],
                    default=[8192, 16384, 32768, 65536, 131072])
    ap.add_argument("--traffic", type=lambda s: [(k, float(v)) for k, v in (x.split("=") for x in s.split(","))],
                    default=[], help="class=bytes per launch from an ncu capture of the current kernels")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
