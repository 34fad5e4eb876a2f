"""Seeded synthetic inputs shared by the oracle, the tests and the benchmark.

This module holds configuration presets and the generators of weights and token
streams. It contains none of the method's arithmetic: no norm, attention, loss,
gradient or update. Both the CPU oracle and the CUDA library receive the arrays
produced here, so the two sides see the same bytes.

Random numbers come from numpy's Philox-4x32-10 counter-based bit generator
(Salmon et al., "Parallel random numbers: as easy as 1, 2, 3", SC'11), keyed by
(seed, tensor index), and numpy's standard-normal sampler on top of it.

Workload shapes follow the End-to-End Test-Time Training method as described in
"TTT-E2E: Learning a Long Context into Weights" (technical review, §5 and §6:
8K window, 1K mini-batch, last quarter of the blocks adaptive, a static second
MLP in each adaptive block) and the b-lab.team summary ("Implementation Details
for TTT"). The pages' own data (DCLM, Books) and trained weights are not
available; these generators stand in for them.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "TTTConfig", "CONFIGS", "config", "make_weights", "make_tokens",
    "make_token_batch", "to_bf16_bits", "from_bf16_bits", "round_to_dtype",
    "weight_shapes", "layer_is_ttt",
]


@dataclass(frozen=True)
class TTTConfig:
    """Shape and hyper-parameters of one TTT-E2E model/workload.

    Notation follows the pages: V vocab, d width, L layers, the last L_t of them
    adaptive ("TTT blocks"), H heads, k attention window, b inner mini-batch,
    eta inner step size, T processed positions per sequence, B sequences.
    """
    name: str
    vocab: int
    d: int
    n_layers: int
    n_heads: int
    n_ttt: int
    mlp_hidden: int
    ttt_hidden: int
    static_hidden: int
    window_k: int
    minibatch_b: int
    batch: int
    eta: float
    T: int
    dtype: str = "bf16"          # storage/compute dtype of activations and frozen weights
    rms_eps: float = 1e-6
    rope_base: float = 10000.0
    decode_n: int = 0            # tokens generated after the prefill (decode workload)
    weight_seed: int = 0
    token_seed: int = 0
    # inner loss of the adaptive blocks: "e2e" (next-token cross-entropy at the output)
    # or "kvb" (each block's layer-wise key-value-binding reconstruction loss, which
    # adds the frozen projections theta_K, theta_V to every adaptive block)
    inner_loss: str = "e2e"

    @property
    def head_dim(self) -> int:
        return self.d // self.n_heads

    @property
    def first_ttt(self) -> int:
        return self.n_layers - self.n_ttt

    def replace(self, **kw) -> "TTTConfig":
        return dataclasses.replace(self, **kw)


def _cfg(idx: int, **kw) -> TTTConfig:
    kw.setdefault("weight_seed", 1000 + idx)
    kw.setdefault("token_seed", 2000 + 16 * idx)
    return TTTConfig(**kw)


# The five workloads. Names describe the model; indices are for seeds only.
CONFIGS = {
    # Tiny fp32 decoder: V256 d64 L4 (block 4 adaptive) H4 h256 (128+128) k16 b16 eta0.1 T256 B1.
    "tiny_fp32": _cfg(1, name="tiny_fp32", vocab=256, d=64, n_layers=4, n_heads=4, n_ttt=1,
                      mlp_hidden=256, ttt_hidden=128, static_hidden=128, window_k=16,
                      minibatch_b=16, batch=1, eta=0.1, T=256, dtype="fp32"),
    # Small bf16: V8192 d512 L8 (last 2 adaptive) H8 h2048 (1024+1024) k1024 b256 eta0.05 T8192 B1.
    "small_bf16": _cfg(2, name="small_bf16", vocab=8192, d=512, n_layers=8, n_heads=8, n_ttt=2,
                       mlp_hidden=2048, ttt_hidden=1024, static_hidden=1024, window_k=1024,
                       minibatch_b=256, batch=1, eta=0.05, T=8192),
    # ~125M: V32000 d768 L12 (last 3 adaptive) H12 h3072 (1536+1536) k2048 b1024 eta0.02 T32768 B4.
    "m125_bf16": _cfg(3, name="m125_bf16", vocab=32000, d=768, n_layers=12, n_heads=12, n_ttt=3,
                      mlp_hidden=3072, ttt_hidden=1536, static_hidden=1536, window_k=2048,
                      minibatch_b=1024, batch=4, eta=0.02, T=32768),
    # ~1B long-context prefill: V32000 d2048 L24 (last 6 adaptive) H16 hd128 h8192 (4096+4096)
    # k8192 b1024 eta0.01 T131072 B1 (128K tokens per batch).
    "b1_128k_bf16": _cfg(4, name="b1_128k_bf16", vocab=32000, d=2048, n_layers=24, n_heads=16,
                         n_ttt=6, mlp_hidden=8192, ttt_hidden=4096, static_hidden=4096,
                         window_k=8192, minibatch_b=1024, batch=1, eta=0.01, T=131072),
    # Decode on the ~125M architecture: 32K prefix, 4096 greedy tokens, update every 1024, B8.
    "m125_decode_bf16": _cfg(5, name="m125_decode_bf16", vocab=32000, d=768, n_layers=12,
                             n_heads=12, n_ttt=3, mlp_hidden=3072, ttt_hidden=1536,
                             static_hidden=1536, window_k=2048, minibatch_b=1024, batch=8,
                             eta=0.02, T=32768, decode_n=4096),
}


def config(name: str, **overrides) -> TTTConfig:
    """Return a preset, optionally with fields replaced (e.g. a shorter T)."""
    return CONFIGS[name].replace(**overrides)


# ----------------------------------------------------------------------------- dtypes

def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    # finite inputs only: u + 0x8000 cannot wrap for any finite float32
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def from_bf16_bits(bits: np.ndarray) -> np.ndarray:
    """Expand bfloat16 bits (uint16) to exactly equal float32 values."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def round_to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round to the storage dtype, returned as float32 values that the dtype represents exactly."""
    x32 = np.asarray(x, dtype=np.float32)
    if dtype == "fp32":
        return x32
    if dtype == "bf16":
        return from_bf16_bits(to_bf16_bits(x32))
    raise ValueError(f"unknown dtype {dtype}")


# ----------------------------------------------------------------------------- weights

def layer_is_ttt(cfg: TTTConfig, layer: int) -> bool:
    """Only the last quarter of the blocks (the last n_ttt) carry fast weights."""
    return layer >= cfg.first_ttt


def weight_shapes(cfg: TTTConfig):
    """Ordered (name, shape) list of every tensor. Matrices are stored [out][in]: y = x @ W.T."""
    d, V = cfg.d, cfg.vocab
    out = [("E", (V, d)), ("final_norm", (d,))]
    for l in range(cfg.n_layers):
        p = f"layers.{l}."
        out += [(p + "attn_norm", (d,)), (p + "Wq", (d, d)), (p + "Wk", (d, d)),
                (p + "Wv", (d, d)), (p + "Wo", (d, d))]
        if layer_is_ttt(cfg, l):
            out += [(p + "ttt_norm", (d,)), (p + "W1t", (cfg.ttt_hidden, d)),
                    (p + "W2t", (d, cfg.ttt_hidden)), (p + "static_norm", (d,)),
                    (p + "W1s", (cfg.static_hidden, d)), (p + "W2s", (d, cfg.static_hidden))]
            if cfg.inner_loss == "kvb":
                out += [(p + "theta_K", (d, d)), (p + "theta_V", (d, d))]
        else:
            out += [(p + "mlp_norm", (d,)), (p + "W1", (cfg.mlp_hidden, d)),
                    (p + "W2", (d, cfg.mlp_hidden))]
    return out


def make_weights(cfg: TTTConfig, std: float = 0.02, seed: int | None = None) -> dict:
    """Every matrix (embedding included) ~ N(0, std^2), norm gains 1.

    Standard normals are drawn in float32, scaled by std in float32 and rounded
    to the config's storage dtype. Returned as float32 arrays holding exactly
    representable values of that dtype. Tensor i draws from Philox keyed by
    (seed, i), so each tensor is independent of the others' sizes; tensors are
    generated on a small thread pool (the result does not depend on it).
    """
    seed = cfg.weight_seed if seed is None else seed
    shapes = weight_shapes(cfg)

    def one(i):
        name, shape = shapes[i]
        if len(shape) == 1:
            return np.ones(shape, dtype=np.float32)
        gen = np.random.Generator(np.random.Philox(key=[seed, i]))
        vals = gen.standard_normal(size=shape, dtype=np.float32)
        vals *= np.float32(std)
        return round_to_dtype(vals, cfg.dtype)

    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=8) as ex:
        arrays = list(ex.map(one, range(len(shapes))))
    return {name: a for (name, _), a in zip(shapes, arrays)}


# ----------------------------------------------------------------------------- tokens

def _zipf_cdf(vocab: int, s: float) -> np.ndarray:
    ranks = np.arange(1, vocab + 1, dtype=np.float64)
    p = ranks ** (-s)
    c = np.cumsum(p)
    return c / c[-1]


def make_tokens(cfg: TTTConfig, n: int, seq: int = 0, seed: int | None = None,
                zipf_s: float = 1.1, copy_prob: float = 0.5,
                span_min: int = 8, span_max: int = 32) -> np.ndarray:
    """One int32 token stream of length n.

    Walk a position p from 0. Once p >= span_min, with probability copy_prob a
    copy starts: a length L uniform in [span_min, span_max] (clipped to p and to
    the end) and a uniform start s in [0, p - L]; tokens s..s+L-1 are appended.
    Otherwise one Zipf(zipf_s) token is drawn: rank r with P(r) ~ r^-zipf_s over
    1..V by inverse CDF, id r - 1.
    """
    seed = cfg.token_seed if seed is None else seed
    gen = np.random.Generator(np.random.Philox(key=[seed, seq]))
    cdf = _zipf_cdf(cfg.vocab, zipf_s)
    out = np.empty(n, dtype=np.int32)
    p = 0
    while p < n:
        if p >= span_min and gen.random() < copy_prob:
            L = int(gen.integers(span_min, span_max + 1))
            L = min(L, p, n - p)
            s = int(gen.integers(0, p - L + 1))
            out[p:p + L] = out[s:s + L]
            p += L
        else:
            r = int(np.searchsorted(cdf, gen.random(), side="right"))
            out[p] = min(r, cfg.vocab - 1)
            p += 1
    return out


def make_token_batch(cfg: TTTConfig, n: int | None = None, batch: int | None = None,
                     seed: int | None = None) -> np.ndarray:
    """[B][n] int32 streams; default n = T + 1 ids (x_0..x_T) for a prefill of T positions."""
    n = cfg.T + 1 if n is None else n
    batch = cfg.batch if batch is None else batch
    return np.stack([make_tokens(cfg, n, seq=s, seed=seed) for s in range(batch)])
