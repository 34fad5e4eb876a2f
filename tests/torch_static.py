"""An independent whole-sequence forward of the TTT-E2E model in float64 PyTorch (CPU).

Test-only. It is written separately from the oracle (no shared code) and uses
library routines where they exist (rms_norm, scaled_dot_product_attention with
an explicit window mask, exact gelu, cross_entropy); RoPE is written as a
complex rotation of the pairs (i, i + hd/2). static_forward processes all
positions at once with fixed weights, so it is the static sliding-window model;
with autograd it also gives the gradient of a chunk's mean loss w.r.t. the fast
weights when nothing cached depends on them. mini_batch_ttt_chunked runs the
method chunk by chunk with an explicit key/value cache for any number of
adaptive blocks, under a selectable rule for what the cache holds.
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


# ----------------------------------------------------------------------------- chunk-wise loop with a K/V cache

def _attend(q, keys, vals, q_pos, k_pos, window):
    """Windowed causal attention of q [n,H,hd] over keys/vals [m,H,hd] (library SDPA, boolean mask)."""
    mask = (k_pos[None, :] <= q_pos[:, None]) & (k_pos[None, :] >= q_pos[:, None] - window + 1)
    o = F.scaled_dot_product_attention(q.transpose(0, 1), keys.transpose(0, 1), vals.transpose(0, 1),
                                       attn_mask=mask)
    return o.transpose(0, 1)


def _adaptive_layer(cfg, w, l, fast_j, x, pos, k_hist, v_hist, hist_pos, mlp_in=None):
    """One adaptive block over rows x at positions pos; attention sees the given
    earlier keys/values (constants) and the rows' own keys/values. mlp_in, when given,
    maps the normalised rows to the adaptive MLP's input (the key projection of the
    key-value-binding variant). Returns (output, post-RoPE keys of the rows, values of
    the rows, the normalised rows ahead of the adaptive MLP)."""
    d, H = cfg.d, cfg.n_heads
    hd = d // H
    n = x.shape[0]
    p = f"layers.{l}."
    r = F.rms_norm(x, (d,), weight=w[p + "attn_norm"], eps=cfg.rms_eps)
    q = _rope_complex((r @ w[p + "Wq"].T).view(n, H, hd), pos, cfg.rope_base)
    k = _rope_complex((r @ w[p + "Wk"].T).view(n, H, hd), pos, cfg.rope_base)
    v = (r @ w[p + "Wv"].T).view(n, H, hd)
    keys = torch.cat([k_hist.detach(), k], dim=0)
    vals = torch.cat([v_hist.detach(), v], dim=0)
    o = _attend(q, keys, vals, pos, torch.cat([hist_pos, pos]), cfg.window_k)
    x = x + o.reshape(n, d) @ w[p + "Wo"].T
    r2 = F.rms_norm(x, (d,), weight=w[p + "ttt_norm"], eps=cfg.rms_eps)
    xin = r2 if mlp_in is None else mlp_in(r2)
    x = x + F.gelu(xin @ fast_j["W1t"].T, approximate="none") @ fast_j["W2t"].T
    r3 = F.rms_norm(x, (d,), weight=w[p + "static_norm"], eps=cfg.rms_eps)
    x = x + F.gelu(r3 @ w[p + "W1s"].T, approximate="none") @ w[p + "W2s"].T
    return x, k, v, r2


def _frozen_stack(cfg, w, tok_in, pos):
    """Embedding and every frozen block over all positions at once (they do not depend on W)."""
    d, H = cfg.d, cfg.n_heads
    hd = d // H
    T = tok_in.shape[0]
    x = w["E"][tok_in]
    for l in range(cfg.n_layers - cfg.n_ttt):
        p = f"layers.{l}."
        r = F.rms_norm(x, (d,), weight=w[p + "attn_norm"], eps=cfg.rms_eps)
        q = _rope_complex((r @ w[p + "Wq"].T).view(T, H, hd), pos, cfg.rope_base)
        k = _rope_complex((r @ w[p + "Wk"].T).view(T, H, hd), pos, cfg.rope_base)
        v = (r @ w[p + "Wv"].T).view(T, H, hd)
        x = x + _attend(q, k, v, pos, pos, cfg.window_k).reshape(T, d) @ w[p + "Wo"].T
        r2 = F.rms_norm(x, (d,), weight=w[p + "mlp_norm"], eps=cfg.rms_eps)
        x = x + F.gelu(r2 @ w[p + "W1"].T, approximate="none") @ w[p + "W2"].T
    return x


def _static_adaptive_kv(cfg, w, x, pos, fast):
    """Keys/values of every adaptive block over the rows x, all computed with the one set
    of fast weights `fast` (a static pass of the adaptive stack). Used by the negative controls."""
    H, hd = cfg.n_heads, cfg.d // cfg.n_heads
    empty = torch.zeros(0, H, hd, dtype=torch.float64)
    none = torch.zeros(0, dtype=torch.long)
    ks, vs = [], []
    with torch.no_grad():
        for j in range(cfg.n_ttt):
            l = cfg.n_layers - cfg.n_ttt + j
            x, k, v, _ = _adaptive_layer(cfg, w, l, fast[j], x, pos, empty, empty, none)
            ks.append(k)
            vs.append(v)
    return ks, vs


def mini_batch_ttt_chunked(cfg, weights, tokens, cache_rule="as_computed"):
    """Mini-batch TTT by autograd, chunk by chunk, for any number of adaptive blocks.

    Chunk i (positions [(i-1)b, ib)) runs the adaptive blocks with W_{i-1}; its
    attention reads earlier positions' keys/values as constants (no gradient)
    and its own rows' keys/values with gradient; its losses are recorded, and
    W_i = W_{i-1} - eta * autograd gradient of the chunk's mean loss.

    cache_rule decides what the earlier positions' keys/values of the adaptive
    blocks are:
      "as_computed"       - the values computed when their own chunk ran, i.e.
                            with the weights in force then (W_{j-1} for chunk j),
                            never recomputed;
      "recompute_current" - recomputed for every chunk with the current W_{i-1};
      "initial_weights"   - computed with the initial fast weights W_0.
    The frozen blocks' keys/values do not depend on W under any rule.
    Returns (losses [T], fast weights after the last full chunk).
    """
    w = {k: _t(v) for k, v in weights.items()}
    tok = torch.as_tensor(tokens, dtype=torch.long)
    T = tok.shape[0] - 1
    H, hd = cfg.n_heads, cfg.d // cfg.n_heads
    b, first = cfg.minibatch_b, cfg.n_layers - cfg.n_ttt
    x0 = _frozen_stack(cfg, w, tok[:T], torch.arange(T))
    fast = initial_fast(cfg, weights)
    init = [{n: t.clone() for n, t in f.items()} for f in fast]
    k_cache = [torch.zeros(0, H, hd, dtype=torch.float64) for _ in range(cfg.n_ttt)]
    v_cache = [torch.zeros(0, H, hd, dtype=torch.float64) for _ in range(cfg.n_ttt)]
    losses = torch.zeros(T, dtype=torch.float64)
    for c0 in range(0, T, b):
        c1 = min(T, c0 + b)
        cur = [{n: t.detach().clone().requires_grad_(True) for n, t in f.items()} for f in fast]
        lo = max(0, c0 - cfg.window_k + 1)
        if cache_rule == "as_computed":
            ks, vs = k_cache, v_cache
        elif cache_rule == "recompute_current":
            ks, vs = _static_adaptive_kv(cfg, w, x0[:c0], torch.arange(c0), [
                {n: t.detach() for n, t in f.items()} for f in cur])
        elif cache_rule == "initial_weights":
            ks, vs = _static_adaptive_kv(cfg, w, x0[:c0], torch.arange(c0), init)
        else:
            raise ValueError(cache_rule)
        x = x0[c0:c1]
        pos = torch.arange(c0, c1)
        new = []
        for j in range(cfg.n_ttt):
            x, k, v, _ = _adaptive_layer(cfg, w, first + j, cur[j], x, pos, ks[j][lo:c0], vs[j][lo:c0],
                                         torch.arange(lo, c0))
            new.append((k.detach(), v.detach()))
        rf = F.rms_norm(x, (cfg.d,), weight=w["final_norm"], eps=cfg.rms_eps)
        ell = F.cross_entropy(rf @ w["E"].T, tok[c0 + 1:c1 + 1], reduction="none")
        losses[c0:c1] = ell.detach()
        if c1 - c0 == b:
            (ell.sum() / b).backward()
            fast = [{n: (t - cfg.eta * t.grad).detach() for n, t in f.items()} for f in cur]
        for j in range(cfg.n_ttt):
            k_cache[j] = torch.cat([k_cache[j], new[j][0]])
            v_cache[j] = torch.cat([v_cache[j], new[j][1]])
    return losses, fast


# ----------------------------------------------------------------------------- key-value-binding inner loss

def mini_batch_ttt_kvb_chunked(cfg, weights, tokens, layerwise=True, output_from_keys=True):
    """Mini-batch TTT with the key-value-binding inner loss, by autograd, chunk by chunk.

    Each adaptive block j maps keys theta_K x to values theta_V x through its own MLP
    W2t gelu(W1t .), x being the block's normalised rows ahead of that MLP; the chunk's
    inner loss of the block is the summed squared error (library mse_loss) divided by
    b, and W_i = W_{i-1} - eta * its gradient. The block's MLP output is the same
    prediction, g(theta_K x; W_{i-1}) (output_from_keys=False applies g to x itself on
    the output path instead: a misreading, for negative controls). With layerwise=True
    the rows x are taken as given, so block j's loss moves only W_j; layerwise=False
    lets every block's loss reach the earlier blocks' weights through x (a misreading,
    for negative controls). Keys/values of earlier chunks are cached as computed. The
    recorded losses are the next-token losses with W_{i-1}. Returns (losses [T], fast
    weights).
    """
    w = {k: _t(v) for k, v in weights.items()}
    tok = torch.as_tensor(tokens, dtype=torch.long)
    T = tok.shape[0] - 1
    H, hd = cfg.n_heads, cfg.d // cfg.n_heads
    b, first = cfg.minibatch_b, cfg.n_layers - cfg.n_ttt
    x0 = _frozen_stack(cfg, w, tok[:T], torch.arange(T))
    fast = initial_fast(cfg, weights)
    k_cache = [torch.zeros(0, H, hd, dtype=torch.float64) for _ in range(cfg.n_ttt)]
    v_cache = [torch.zeros(0, H, hd, dtype=torch.float64) for _ in range(cfg.n_ttt)]
    losses = torch.zeros(T, dtype=torch.float64)
    for c0 in range(0, T, b):
        c1 = min(T, c0 + b)
        cur = [{n: t.detach().clone().requires_grad_(True) for n, t in f.items()} for f in fast]
        lo = max(0, c0 - cfg.window_k + 1)
        x = x0[c0:c1]
        pos = torch.arange(c0, c1)
        new, inner = [], []
        for j in range(cfg.n_ttt):
            l = first + j
            theta_k = w[f"layers.{l}.theta_K"]
            proj = (lambda r, th=theta_k: r @ th.T) if output_from_keys else None
            x, k, v, xin = _adaptive_layer(cfg, w, l, cur[j], x, pos, k_cache[j][lo:c0], v_cache[j][lo:c0],
                                           torch.arange(lo, c0), mlp_in=proj)
            new.append((k.detach(), v.detach()))
            if layerwise:
                xin = xin.detach()
            keys = xin @ w[f"layers.{l}.theta_K"].T
            vals = xin @ w[f"layers.{l}.theta_V"].T
            pred = F.gelu(keys @ cur[j]["W1t"].T, approximate="none") @ cur[j]["W2t"].T
            inner.append(F.mse_loss(pred, vals, reduction="sum") / b)
        with torch.no_grad():
            rf = F.rms_norm(x, (cfg.d,), weight=w["final_norm"], eps=cfg.rms_eps)
            losses[c0:c1] = F.cross_entropy(rf @ w["E"].T, tok[c0 + 1:c1 + 1], reduction="none")
        if c1 - c0 == b:
            sum(inner).backward()
            fast = [{n: (t - cfg.eta * t.grad).detach() for n, t in f.items()} for f in cur]
        for j in range(cfg.n_ttt):
            k_cache[j] = torch.cat([k_cache[j], new[j][0]])
            v_cache[j] = torch.cat([v_cache[j], new[j][1]])
    return losses, fast


# ----------------------------------------------------------------------------- outer loop (meta-gradient)

def outer_gradient_chunked(cfg, weights, tokens):
    """The outer objective L(W_0) = (1/N) sum_i A_i(W_{i-1}) and its gradient w.r.t. the
    initial fast weights, by autograd through the unrolled inner updates.

    Chunk by chunk as mini_batch_ttt_chunked (earlier chunks' keys/values detached, as
    the inner loop holds them), but the update keeps the graph: each inner gradient is
    taken with create_graph=True, W_i = W_{i-1} - eta * grad, and the final backward
    differentiates through every step (the library's reverse-over-reverse).
    Returns (L, [{"W1t", "W2t"} per adaptive block]).
    """
    w = {k: _t(v) for k, v in weights.items()}
    tok = torch.as_tensor(tokens, dtype=torch.long)
    T = tok.shape[0] - 1
    H, hd = cfg.n_heads, cfg.d // cfg.n_heads
    b, first = cfg.minibatch_b, cfg.n_layers - cfg.n_ttt
    assert T % b == 0
    x0 = _frozen_stack(cfg, w, tok[:T], torch.arange(T))
    w0 = initial_fast(cfg, weights, requires_grad=True)
    fast = w0
    k_cache = [torch.zeros(0, H, hd, dtype=torch.float64) for _ in range(cfg.n_ttt)]
    v_cache = [torch.zeros(0, H, hd, dtype=torch.float64) for _ in range(cfg.n_ttt)]
    total = torch.zeros((), dtype=torch.float64)
    for c0 in range(0, T, b):
        c1 = c0 + b
        lo = max(0, c0 - cfg.window_k + 1)
        x = x0[c0:c1]
        pos = torch.arange(c0, c1)
        new = []
        for j in range(cfg.n_ttt):
            x, k, v, _ = _adaptive_layer(cfg, w, first + j, fast[j], x, pos, k_cache[j][lo:c0], v_cache[j][lo:c0],
                                         torch.arange(lo, c0))
            new.append((k.detach(), v.detach()))
        rf = F.rms_norm(x, (cfg.d,), weight=w["final_norm"], eps=cfg.rms_eps)
        A = F.cross_entropy(rf @ w["E"].T, tok[c0 + 1:c1 + 1], reduction="mean")
        total = total + A
        params = [f[n] for f in fast for n in ("W1t", "W2t")]
        grads = iter(torch.autograd.grad(A, params, create_graph=True))
        fast = [{n: f[n] - cfg.eta * next(grads) for n in ("W1t", "W2t")} for f in fast]
        for j in range(cfg.n_ttt):
            k_cache[j] = torch.cat([k_cache[j], new[j][0]])
            v_cache[j] = torch.cat([v_cache[j], new[j][1]])
    L = total / (T // b)
    g = iter(torch.autograd.grad(L, [f[n] for f in w0 for n in ("W1t", "W2t")]))
    return float(L.detach()), [{n: next(g) for n in ("W1t", "W2t")} for _ in w0]
