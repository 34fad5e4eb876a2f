"""Helpers of the GPU-vs-oracle parity tests: run both sides on the same seeded
inputs and measure the errors the way the tolerances are stated.

Tolerances (written in the tests): fp32 workloads — max relative error
max|a-b| / max|b| <= 1e-4 per tensor (the losses of a sequence, each fast-weight
matrix); bf16 workloads — per-token relative loss error |l_a - l_b| / |l_b| <=
2e-2 and relative Frobenius error ||W_a - W_b|| / ||W_b|| <= 5e-3 per matrix.
Because W is dominated by W_init, the update itself is also compared:
||dW_a - dW_b|| / ||dW_b|| with dW = W_final - W_init (reported, loosely gated).
"""
import numpy as np

import synthetic as syn
from oracle import Oracle


def max_rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def rel_fro(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def gpu_fast_weights(T, h, cfg):
    return [[T.ttt_get_weights(h, s, j) for j in range(cfg.n_ttt)] for s in range(cfg.batch)]


def oracle_fast_weights(orc, cfg):
    return [[orc.fast_weights(s, j) for j in range(cfg.n_ttt)] for s in range(cfg.batch)]


def init_fast_weights(w, cfg):
    return [(w[f"layers.{l}.W1t"].astype(np.float64), w[f"layers.{l}.W2t"].astype(np.float64))
            for l in range(cfg.first_ttt, cfg.n_layers)]


def compare(cfg, w, gpu_losses, orc_losses, gpu_w, orc_w, report=None):
    """Return a dict of error figures; asserts the stated tolerances."""
    out = {"loss": [], "w": [], "dw": []}
    init = init_fast_weights(w, cfg)
    for s in range(len(gpu_losses)):
        gl, ol = np.asarray(gpu_losses[s], np.float64), np.asarray(orc_losses[s], np.float64)
        assert np.all(np.isfinite(gl))
        if cfg.dtype == "fp32":
            out["loss"].append(max_rel(gl, ol))
        else:
            out["loss"].append(float(np.max(np.abs(gl - ol) / np.abs(ol))))
        for j in range(len(gpu_w[s])):
            for m in range(2):
                ga, ob = gpu_w[s][j][m], orc_w[s][j][m]
                out["w"].append(max_rel(ga, ob) if cfg.dtype == "fp32" else rel_fro(ga, ob))
                if np.any(ob != init[j][m]):
                    out["dw"].append(rel_fro(ga - init[j][m], ob - init[j][m]))
    summary = {k: (max(v) if v else 0.0) for k, v in out.items()}
    if report is not None:
        report.update(summary)
    if cfg.dtype == "fp32":
        assert summary["loss"] <= 1e-4, summary
        assert summary["w"] <= 1e-4, summary
    else:
        assert summary["loss"] <= 2e-2, summary
        assert summary["w"] <= 5e-3, summary
    return summary


def prefill_both(T, cfg, w=None, toks=None, max_segment=0, oracle=True):
    w = syn.make_weights(cfg) if w is None else w
    toks = syn.make_token_batch(cfg) if toks is None else toks
    h = T.ttt_create(cfg, w, max_segment=max_segment)
    gl = T.ttt_prefill(h, np.ascontiguousarray(toks, dtype=np.int32))
    res = {"w": w, "toks": toks, "h": h, "gpu_losses": gl, "gpu_w": gpu_fast_weights(T, h, cfg)}
    if oracle:
        orc = Oracle(cfg, w)
        res["orc"] = orc
        res["orc_losses"] = orc.prefill(toks)
        res["orc_w"] = oracle_fast_weights(orc, cfg)
    return res
