"""An independent whole-sequence forward of the TTT-E2E model in float64 PyTorch (CPU).

Test-only. It is written separately from the oracle (no shared code) and uses
library routines where they exist (rms_norm, scaled_dot_product_attention with
an explicit window mask, exact gelu, cross_entropy); RoPE is written as a
complex rotation of the pairs (i, i + hd/2). It processes all positions at once
with fixed weights, so it is the static sliding-window model; with autograd it
also gives the gradient of a chunk's mean loss w.r.t. the fast weights when
nothing cached depends on them.
"""
import torch
import torch.nn.functional as F


def _t(a):
    return torch.as_tensor(a, dtype=torch.float64)


def _rope_complex(x, pos, base):
    # x [T, H, hd] -> complex view over pairs (i, i + hd/2)
    hd = x.shape[-1]
    half = hd // 2
    freqs = base ** (-torch.arange(half, dtype=torch.float64) * 2.0 / hd)
    ang = pos.to(torch.float64)[:, None] * freqs[None, :]
    rot = torch.polar(torch.ones_like(ang), ang)[:, None, :]
    zc = torch.complex(x[..., :half], x[..., half:]) * rot
    return torch.cat([zc.real, zc.imag], dim=-1)


def static_forward(cfg, weights, tokens, fast=None, start_pos=0):
    """Per-token losses [T] of tokens [T+1] with all weights fixed.

    fast: optional list (one per adaptive block) of dicts with W1t/W2t tensors
    replacing the initial fast weights (may require grad).
    """
    w = {k: _t(v) for k, v in weights.items()}
    tok = torch.as_tensor(tokens, dtype=torch.long)
    T = tok.shape[0] - 1
    d, H = cfg.d, cfg.n_heads
    hd = d // H
    x = w["E"][tok[:T]]
    pos = torch.arange(start_pos, start_pos + T)
    qp = pos[:, None]
    kp = pos[None, :]
    mask = (kp <= qp) & (kp >= qp - cfg.window_k + 1)
    for l in range(cfg.n_layers):
        p = f"layers.{l}."
        r = F.rms_norm(x, (d,), weight=w[p + "attn_norm"], eps=cfg.rms_eps)
        q = _rope_complex((r @ w[p + "Wq"].T).view(T, H, hd), pos, cfg.rope_base)
        k = _rope_complex((r @ w[p + "Wk"].T).view(T, H, hd), pos, cfg.rope_base)
        v = (r @ w[p + "Wv"].T).view(T, H, hd)
        o = F.scaled_dot_product_attention(q.transpose(0, 1), k.transpose(0, 1), v.transpose(0, 1),
                                           attn_mask=mask)
        x = x + o.transpose(0, 1).reshape(T, d) @ w[p + "Wo"].T
        if l >= cfg.n_layers - cfg.n_ttt:
            j = l - (cfg.n_layers - cfg.n_ttt)
            W1t = fast[j]["W1t"] if fast is not None else w[p + "W1t"]
            W2t = fast[j]["W2t"] if fast is not None else w[p + "W2t"]
            r2 = F.rms_norm(x, (d,), weight=w[p + "ttt_norm"], eps=cfg.rms_eps)
            x = x + F.gelu(r2 @ W1t.T, approximate="none") @ W2t.T
            r3 = F.rms_norm(x, (d,), weight=w[p + "static_norm"], eps=cfg.rms_eps)
            x = x + F.gelu(r3 @ w[p + "W1s"].T, approximate="none") @ w[p + "W2s"].T
        else:
            r2 = F.rms_norm(x, (d,), weight=w[p + "mlp_norm"], eps=cfg.rms_eps)
            x = x + F.gelu(r2 @ w[p + "W1"].T, approximate="none") @ w[p + "W2"].T
    rf = F.rms_norm(x, (d,), weight=w["final_norm"], eps=cfg.rms_eps)
    z = rf @ w["E"].T
    return F.cross_entropy(z, tok[1:], reduction="none")


def initial_fast(cfg, weights, requires_grad=False):
    out = []
    for l in range(cfg.n_layers - cfg.n_ttt, cfg.n_layers):
        p = f"layers.{l}."
        out.append({n: _t(weights[p + n]).clone().requires_grad_(requires_grad) for n in ("W1t", "W2t")})
    return out


def mini_batch_ttt_single_adaptive_block(cfg, weights, tokens):
    """Mini-batch TTT for a model with exactly one adaptive block, by autograd.

    With one adaptive block, everything upstream of its MLP (including the K/V
    of every attention layer) is independent of the fast weights, so chunk i's
    losses are the static model's losses at those positions with W_{i-1}, and
    W_i = W_{i-1} - eta * grad of the chunk mean. Returns (losses [T], fast).
    """
    assert cfg.n_ttt == 1
    tok = torch.as_tensor(tokens, dtype=torch.long)
    T = tok.shape[0] - 1
    b = cfg.minibatch_b
    fast = initial_fast(cfg, weights)
    losses = torch.zeros(T, dtype=torch.float64)
    for c0 in range(0, T, b):
        c1 = min(T, c0 + b)
        cur = [{n: t.detach().clone().requires_grad_(True) for n, t in f.items()} for f in fast]
        # only positions < c1 influence the chunk's losses (causality)
        all_losses = static_forward(cfg, weights, tok[:c1 + 1], fast=cur)
        chunk = all_losses[c0:c1]
        losses[c0:c1] = chunk.detach()
        if c1 - c0 == b:
            (chunk.sum() / b).backward()
            fast = [{n: (t - cfg.eta * t.grad).detach() for n, t in f.items()} for f in cur]
    return losses, fast
