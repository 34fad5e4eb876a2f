"""Host-side checks of the benchmark (CPU only): the model-FLOP count, the
replica reductions over a world of two gloo ranks, and the rank-0-only output of
the reference arm under a two-rank launch."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synthetic as syn  # noqa: E402


def _direct_model_flops(cfg):
    """The same algorithmic count assembled product by product (forward matmuls of
    every block and the head, window attention QK^T and PV, the head's data
    gradient, and per adaptive block the static-MLP data gradient, the TTT-MLP
    data and weight gradients, and below the first adaptive block the attention
    data gradients with dK, dV only over the chunk's own keys)."""
    T, d, V, L, Lt = cfg.T, cfg.d, cfg.vocab, cfg.n_layers, cfg.n_ttt
    k, b = cfg.window_k, cfg.minibatch_b
    mm = lambda m, n, kk: 2.0 * m * n * kk  # noqa: E731
    pairs = sum(min(p + 1, k) for p in range(T))
    intra = sum(min(i + 1, k) for c0 in range(0, T, b) for i in range(min(b, T - c0)))
    attn_fwd = 2 * 2.0 * d * pairs                    # S = QK^T and O = PV over the window
    fwd = 0.0
    for l in range(L):
        fwd += mm(T, 3 * d, d) + mm(T, d, d) + attn_fwd
        if l < L - Lt:
            fwd += mm(T, cfg.mlp_hidden, d) + mm(T, d, cfg.mlp_hidden)
        else:
            fwd += mm(T, cfg.ttt_hidden, d) + mm(T, d, cfg.ttt_hidden)
            fwd += mm(T, cfg.static_hidden, d) + mm(T, d, cfg.static_hidden)
    fwd += mm(T, V, d)
    if cfg.inner_loss == "kvb":                        # each block's binding loss only
        upd = 0.0
        for j in range(Lt):
            upd += mm(T, d, d) + mm(T, d, d)                                   # k (MLP input), v projections
            upd += mm(T, cfg.ttt_hidden, d)                                    # du = de W2t
            upd += mm(cfg.ttt_hidden, d, T) + mm(d, cfg.ttt_hidden, T)         # dW1t, dW2t
        return (fwd + upd) * cfg.batch
    bwd = mm(T, d, V)                                  # dh = dz E
    for j in range(Lt):
        bwd += mm(T, cfg.static_hidden, d) + mm(T, d, cfg.static_hidden)   # static MLP data gradient
        bwd += mm(T, cfg.ttt_hidden, d)                                    # du = dm W2t (into gelu')
        bwd += mm(cfg.ttt_hidden, d, T) + mm(d, cfg.ttt_hidden, T)         # dW1t, dW2t
        if j > 0:
            bwd += mm(T, d, cfg.ttt_hidden)                                # dx through W1t
            bwd += mm(T, d, d) + mm(T, d, 3 * d)                           # through Wo and Wqkv
            bwd += 2 * 2.0 * d * pairs + 2 * 2.0 * d * intra               # dP, dQ over the window; dK, dV own keys
    return (fwd + bwd) * cfg.batch


@pytest.mark.parametrize("name,overrides", [("tiny_fp32", {}), ("small_bf16", {"T": 4096}),
                                            ("tiny_fp32", {"n_ttt": 0, "window_k": 256}),
                                            ("tiny_fp32", {"n_ttt": 3, "T": 200}),
                                            ("small_bf16", {"T": 4096, "inner_loss": "kvb"})])
def test_model_flops_equals_the_product_by_product_count(name, overrides):
    cfg = syn.config(name, **overrides)
    assert bench.model_flops(cfg) == pytest.approx(_direct_model_flops(cfg), rel=1e-12)


def test_model_flops_of_the_128k_workload():
    cfg = syn.config("b1_128k_bf16")
    assert bench.model_flops(cfg) / 1e12 == pytest.approx(699.84, abs=0.01)
    full = cfg.replace(n_ttt=0, window_k=cfg.T)
    assert bench.model_flops(full) / 1e12 == pytest.approx(2039.88, abs=0.01)


def _replica_worker(rank, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    d, r, local, ws = bench._dist()
    assert (r, local, ws) == (rank, rank, 2)
    d.init_process_group("gloo", rank=rank, world_size=2)
    try:
        ms = [120.0, 150.0][rank]           # per-rank step time
        tokens = [1000.0, 1000.0][rank]     # tokens each replica processed
        out[rank] = (bench._max_over_ranks(d, ms, "cpu"), bench._sum_over_ranks(d, tokens, "cpu"))
    finally:
        d.destroy_process_group()


def test_replica_reductions_take_the_slowest_rank_and_all_tokens():
    port = 29500 + (os.getpid() % 1000)
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_replica_worker, args=(port, out), nprocs=2, join=True)
        res = dict(out)
    for rank in (0, 1):
        ms_max, tokens = res[rank]
        assert ms_max == 150.0 and tokens == 2000.0
    # value = all ranks' tokens / the slowest rank's time
    assert 2000.0 / (150.0 / 1e3) == pytest.approx(13333.33, rel=1e-6)


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_prints_once_from_rank_zero(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
               MASTER_PORT="29999")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "tiny_fp32", "--steps", "1", "--warmup", "0", "--ref-tokens", "32", "--gpus", "2"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    if rank == 0:
        assert len(lines) == 1
        line = json.loads(lines[0])
        assert line["impl"] == "reference" and line["value"] > 0 and line["n_gpus"] == 2
        assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    else:
        assert lines == []


def test_decode_accounting_of_the_125m_decode_workload():
    """Decode's model FLOPs per decoded token (forward of the position plus its share of
    the chunk update) and its least HBM bytes per token step, assembled tensor by tensor:
    weights once, each sequence's bf16 fast-weight copies, each sequence's windows."""
    cfg = syn.config("m125_decode_bf16")
    n = cfg.decode_n
    per_token = (bench.model_flops(cfg, T=cfg.T + n) - bench.model_flops(cfg, T=cfg.T)) / (cfg.batch * n)
    assert per_token / 1e9 == pytest.approx(0.295 + 0.114, rel=5e-3)
    d, L, Lt, B = cfg.d, cfg.n_layers, cfg.n_ttt, cfg.batch
    tensors = [cfg.vocab * d] + [d * d] * 4 * L + [cfg.mlp_hidden * d] * 2 * (L - Lt) + \
        [cfg.static_hidden * d] * 2 * Lt + [cfg.ttt_hidden * d] * 2 * Lt
    fast = [cfg.ttt_hidden * d] * 2 * Lt * B
    windows = [cfg.window_k * d] * 2 * L * B
    assert bench.decode_bytes_per_step(cfg, cfg.T) == 2 * (sum(tensors) + sum(fast) + sum(windows))
    assert bench.decode_bytes_per_step(cfg, 9) == 2 * (sum(tensors) + sum(fast) + 10 * d * 2 * L * B)
