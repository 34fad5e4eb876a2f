"""CPU oracle of the TTT-E2E inner loop (prefill and decode).

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this module:
only the tests, the package's smoke check and the benchmark's CPU-baseline leg
call it. It shares no code with the CUDA library.

What it computes follows the pages describing End-to-End Test-Time Training
(TTT-E2E) for long context:
  * per-token loss l_t(W) = CE(f(x_{t-1}; W), x_t)
      - b-lab.team summary, "Test-Time Training (Inner Loop)", loss equation;
      - technical review §3, eq. (3);
  * mini-batch GD W_i = W_{i-1} - eta * (1/b) * sum_k grad l_k(W_{i-1}), every
    target of chunk i scored with W_{i-1} before the update
      - summary, "Mini-Batch Gradient Descent"; review §5, eq. (9);
  * sliding-window attention with k >= b, causal inside the chunk
      - summary, "Integration with Sliding-Window Attention"; review §5;
  * only the MLPs of the last quarter of the blocks update; a static second MLP
    follows the adaptive one in those blocks; embeddings, norms and attention
    are frozen - summary, "Implementation Details for TTT"; review §6;
  * Algorithm 1 (causal prefill with adaptation) and Algorithm 3 (generation
    with periodic adaptation, update after a full mini-batch of generated
    tokens) - review §7; per-sequence fresh copy of the fast weights -
    review §7, Algorithm 1.

Readings taken where the pages are silent:
  R1 T+1 ids x_0..x_T in, T positions processed, out_losses[t-1] = l_t.
  R2 query at position p attends to keys [p-k+1, p]; k >= T is full attention.
  R3 K/V cached from earlier chunks are constants: gradients flow only through
     the current chunk's K/V. They hold the values computed when their chunk
     was processed (with that step's weights) and are never recomputed.
  R4 both TTT-MLP matrices (W1t, W2t) update; no biases anywhere.
  R5 pre-norm blocks; adaptive block = attention, TTT-MLP, static MLP, each
     with its own RMSNorm gain and residual.
  R6 final RMSNorm then the tied LM head z = E r.
  R7 exact GELU 0.5u(1+erf(u/sqrt2)); RMSNorm y = g x / sqrt(mean(x^2)+eps).
  R8 RoPE rotate-half pairing (i, i+hd/2), theta_i = base^(-2i/hd), absolute
     positions; scale 1/sqrt(hd); softmax without bias or dropout.
  R9 one constant eta for every adaptive block; the chunk loss is the mean
     over its b positions; sequences are independent (no 1/B).
  R10 a trailing partial chunk is scored but not used for an update; its
     positions stay pending until later positions (decode) complete it.
  R11 greedy decode takes the lowest id among equal maxima; decode's loss
     output is -log p(chosen token) under the weights in force.

Variant with the layer-wise key-value-binding inner loss (cfg.inner_loss ==
"kvb"; technical review §8, eq. (10); summary, "Alternative Derivation
(Connection to TTT-KVB)"): each adaptive block's fast weights W = (W1t, W2t)
fit g(theta_K x_t; W) to theta_V x_t instead of descending the next-token loss.
The model is otherwise the one above (adaptive MLPs in the last quarter of the
blocks); the pages' own TTT-KVB models used multi-head LoRA MLPs in every layer,
whose shapes they do not give. Readings taken:
  K1 x_t is the block's RMSNorm output r2 ahead of its adaptive MLP, and
     g(k; W) = W2t gelu(W1t k) is the adaptive two-layer MLP; theta_K, theta_V are
     frozen d x d matrices of the block. Output rule: the sub-layer's output is the
     binding prediction itself, m = a + g(theta_K r2; W_{i-1}), i.e. the pre-update
     weights and the key projection (technical review §8: the simplified
     construction; summary, "Alternative Derivation", step 3, Simplified Output
     Rule: the prediction of g is reused as the output embedding).
  K2 the chunk's inner loss is (1/b) sum_t ||g(theta_K x_t; W) - theta_V x_t||^2
     (squared Euclidean norm, mean over the b positions as in R9); each block
     descends its own loss w.r.t. its own W only (layer-wise: no gradient passes
     between blocks), with the same eta, schedule and per-sequence state.
  K3 the recorded per-token losses are still the next-token losses of the
     model with the weights in force (the inner loss only drives the update).

Outer-loop meta-gradient (technical review §4, eqs. (5)-(7) and §7 Algorithm 2;
summary, "Outer Loop"): meta_gradient() differentiates the mean of the scored
losses, L(W_0; X) = (1/N) sum_i A_i(W_{i-1}), with respect to the initial fast
weights W_0 through the whole update trajectory, by eq. (7) as written. Reading:
  M1 A_i and its Hessian are those the inner loop defines: the window cache of
     earlier chunks is a constant (R3) in the outer derivative too, and the
     static parameters phi stay fixed (eq. (7) suppresses their paths).
  M2 T is a multiple of b (every scored loss belongs to a chunk that updates).
The Hessian-vector products come from the complex-step derivative of the
hand-written chunk gradient (Squire and Trapp, SIAM Review 40(1), 1998):
H v = Im grad A(W + i h v) / h, exact up to rounding because that gradient is
a real-analytic function of W. This is the only place where the oracle runs on
complex arrays.

Arithmetic is float64 throughout. Matrix products use numpy's matmul as the
library primitive. Queries are processed in groups only to bound memory; each
row is the plain definition. This oracle is pinned by the tests in
tests/test_oracle_pins.py (finite differences, an independent whole-sequence
forward and autograd, and the special cases eta=0, k>=T, b=T, b=1).
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf

__all__ = ["Oracle", "rms_norm", "rms_norm_backward", "gelu", "gelu_prime", "rope",
           "rope_backward", "rope_tables", "window_attention", "window_attention_backward"]


# ----------------------------------------------------------------------------- primitives

def rms_norm(x, g, eps):
    """RMSNorm (reading R7): y = g * x / sqrt(mean(x^2) + eps). Returns (y, rstd)."""
    rstd = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return g * x * rstd, rstd


def rms_norm_backward(x, g, rstd, dy):
    """Derivative of rms_norm w.r.t. x for upstream dy (g and eps are frozen)."""
    n = x.shape[-1]
    gdy = g * dy
    dot = np.sum(gdy * x, axis=-1, keepdims=True)
    return rstd * gdy - x * (rstd ** 3) * dot / n


def gelu(u):
    """Exact GELU (reading R7)."""
    return 0.5 * u * (1.0 + erf(u / math.sqrt(2.0)))


def gelu_prime(u):
    """d gelu / du = Phi(u) + u * phi(u)."""
    return 0.5 * (1.0 + erf(u / math.sqrt(2.0))) + u * np.exp(-0.5 * u * u) / math.sqrt(2.0 * math.pi)


def rope_tables(positions, hd, base):
    """cos/sin [n, hd/2] of angle p * base^(-2i/hd) (reading R8)."""
    i = np.arange(hd // 2, dtype=np.float64)
    theta = base ** (-2.0 * i / hd)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * theta[None, :]
    return np.cos(ang), np.sin(ang)


def rope(x, cos, sin):
    """Rotate pairs (i, i+hd/2) of x [n, H, hd] by the per-position angles."""
    h = x.shape[-1] // 2
    x1, x2 = x[..., :h], x[..., h:]
    c, s = cos[:, None, :], sin[:, None, :]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def rope_backward(dy, cos, sin):
    """Transpose (= inverse) of the rotation applied by rope()."""
    h = dy.shape[-1] // 2
    d1, d2 = dy[..., :h], dy[..., h:]
    c, s = cos[:, None, :], sin[:, None, :]
    return np.concatenate([d1 * c + d2 * s, d2 * c - d1 * s], axis=-1)


def _window_mask(q_pos, k_pos, window):
    qp = np.asarray(q_pos)[:, None]
    kp = np.asarray(k_pos)[None, :]
    return (kp <= qp) & (kp >= qp - window + 1)


def window_attention(q, keys, vals, q_pos, k_pos, window, keep_probs=False, group=512):
    """Causal sliding-window softmax attention (reading R2, R8).

    q [n, H, hd] at positions q_pos; keys/vals [m, H, hd] at positions k_pos.
    Query p uses the keys with p-window+1 <= position <= p; k_pos is ascending.
    Returns o [n, H, hd]
    and, if keep_probs, the probabilities [H, n, m].
    """
    n, H, hd = q.shape
    scale = 1.0 / math.sqrt(hd)
    o = np.empty_like(q)
    probs = np.empty((H, n, keys.shape[0]), dtype=np.result_type(q, keys)) if keep_probs else None
    k_pos = np.asarray(k_pos)
    for g0 in range(0, n, group):
        g1 = min(n, g0 + group)
        # keys outside [first query - window + 1, last query] are masked for every
        # query of the group, so they are skipped (their probability is exactly 0)
        lo = int(np.searchsorted(k_pos, q_pos[g0] - window + 1, side="left"))
        hi = int(np.searchsorted(k_pos, q_pos[g1 - 1], side="right"))
        mask = _window_mask(q_pos[g0:g1], k_pos[lo:hi], window)
        for h in range(H):
            s = (q[g0:g1, h, :] @ keys[lo:hi, h, :].T) * scale
            s = np.where(mask, s, -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)
            o[g0:g1, h, :] = p @ vals[lo:hi, h, :]
            if keep_probs:
                probs[h, g0:g1, :] = 0.0
                probs[h, g0:g1, lo:hi] = p
    return o, probs


def window_attention_backward(q, keys, vals, o, probs, do):
    """Gradients of window_attention w.r.t. q, keys and vals (all keys given)."""
    n, H, hd = q.shape
    scale = 1.0 / math.sqrt(hd)
    dq = np.empty_like(q)
    dk = np.empty_like(keys)
    dv = np.empty_like(vals)
    for h in range(H):
        p = probs[h]
        dp = do[:, h, :] @ vals[:, h, :].T
        dsum = np.sum(do[:, h, :] * o[:, h, :], axis=1, keepdims=True)
        ds = p * (dp - dsum)
        dq[:, h, :] = (ds @ keys[:, h, :]) * scale
        dk[:, h, :] = (ds.T @ q[:, h, :]) * scale
        dv[:, h, :] = p.T @ do[:, h, :]
    return dq, dk, dv


def _logsumexp(z):
    m = z.max(axis=-1, keepdims=True)
    return (m + np.log(np.sum(np.exp(z - m), axis=-1, keepdims=True)))[..., 0]


# ----------------------------------------------------------------------------- state

class _History:
    """Post-RoPE keys and values of every processed position of one layer."""

    def __init__(self, H, hd):
        self.K = np.empty((0, H, hd))
        self.V = np.empty((0, H, hd))

    def append(self, k, v):
        self.K = np.concatenate([self.K, k], axis=0)
        self.V = np.concatenate([self.V, v], axis=0)


class _Seq:
    """Per-sequence state: a fresh copy of the fast weights (review §7, Algorithm 1)."""

    def __init__(self, cfg, w0):
        self.fast = [{"W1t": w0[f"layers.{l}.W1t"].copy(), "W2t": w0[f"layers.{l}.W2t"].copy()}
                     for l in range(cfg.first_ttt, cfg.n_layers)]
        self.hist = [_History(cfg.n_heads, cfg.head_dim) for _ in range(cfg.n_layers)]
        self.n_pos = 0
        self.pending_token = None
        self.pend_inputs = []
        self.pend_targets = []


class Oracle:
    """Plain implementation of Algorithms 1 and 3 for B independent sequences."""

    def __init__(self, cfg, weights):
        self.cfg = cfg
        self.w = {k: np.asarray(v, dtype=np.float64) for k, v in weights.items()}
        self.reset()

    def reset(self):
        self.seqs = [_Seq(self.cfg, self.w) for _ in range(self.cfg.batch)]

    # --------------------------------------------------------------- blocks
    def _attn(self, seq, l, x, s, commit, keep):
        """Pre-norm attention sub-block of layer l for positions [s, s+n)."""
        cfg, w, p = self.cfg, self.w, f"layers.{l}."
        n, H, hd = x.shape[0], cfg.n_heads, cfg.head_dim
        r1, rstd1 = rms_norm(x, w[p + "attn_norm"], cfg.rms_eps)
        pos = np.arange(s, s + n)
        cos, sin = rope_tables(pos, hd, cfg.rope_base)
        q = rope((r1 @ w[p + "Wq"].T).reshape(n, H, hd), cos, sin)
        k = rope((r1 @ w[p + "Wk"].T).reshape(n, H, hd), cos, sin)
        v = (r1 @ w[p + "Wv"].T).reshape(n, H, hd)
        hist = seq.hist[l]
        lo = max(0, s - cfg.window_k + 1)
        keys = np.concatenate([hist.K[lo:s], k], axis=0)
        vals = np.concatenate([hist.V[lo:s], v], axis=0)
        k_pos = np.arange(lo, s + n)
        o, probs = window_attention(q, keys, vals, pos, k_pos, cfg.window_k, keep_probs=keep)
        a = x + o.reshape(n, -1) @ w[p + "Wo"].T
        if commit:
            hist.append(k, v)
        cache = dict(x=x, rstd1=rstd1, q=q, keys=keys, vals=vals, o=o, probs=probs,
                     n_cached=s - lo, cos=cos, sin=sin) if keep else None
        return a, cache

    def _frozen_block(self, seq, l, x, s, commit):
        cfg, w, p = self.cfg, self.w, f"layers.{l}."
        a, _ = self._attn(seq, l, x, s, commit, keep=False)
        r2, _ = rms_norm(a, w[p + "mlp_norm"], cfg.rms_eps)
        return a + gelu(r2 @ w[p + "W1"].T) @ w[p + "W2"].T

    def _ttt_block(self, seq, j, x, s, commit, keep):
        """Adaptive block j: attention, TTT-MLP with fast weights, static MLP (reading R5)."""
        cfg, w = self.cfg, self.w
        l = cfg.first_ttt + j
        p = f"layers.{l}."
        fw = seq.fast[j]
        a, c = self._attn(seq, l, x, s, commit, keep)
        r2, rstd2 = rms_norm(a, w[p + "ttt_norm"], cfg.rms_eps)
        # key-value binding (reading K1): the MLP reads the key projection of r2
        xin = r2 @ w[p + "theta_K"].T if getattr(cfg, "inner_loss", "e2e") == "kvb" else r2
        u = xin @ fw["W1t"].T
        g = gelu(u)
        m = a + g @ fw["W2t"].T
        r3, rstd3 = rms_norm(m, w[p + "static_norm"], cfg.rms_eps)
        us = r3 @ w[p + "W1s"].T
        y = m + gelu(us) @ w[p + "W2s"].T
        if keep:
            c.update(a=a, rstd2=rstd2, r2=r2, xin=xin, u=u, g=g, m=m, rstd3=rstd3, us=us)
        return y, c

    def _head(self, y):
        """Final RMSNorm and tied LM head (reading R6)."""
        rf, rstdf = rms_norm(y, self.w["final_norm"], self.cfg.rms_eps)
        return rf @ self.w["E"].T, rf, rstdf

    def _frozen_forward(self, seq, tokens_in, s, commit):
        x = self.w["E"][np.asarray(tokens_in)]
        for l in range(self.cfg.first_ttt):
            x = self._frozen_block(seq, l, x, s, commit)
        return x

    # --------------------------------------------------------------- one chunk
    def _chunk(self, seq, h_in, s, targets, need_grad, commit):
        """Forward the adaptive blocks for positions [s, s+n) with the weights in force.

        Returns the per-position losses, the fast-weight gradients of the chunk's
        mean loss (if need_grad) and nothing else; commits K/V when asked.
        """
        cfg, w = self.cfg, self.w
        n = h_in.shape[0]
        y = h_in
        caches = []
        for j in range(cfg.n_ttt):
            y, c = self._ttt_block(seq, j, y, s, commit, keep=need_grad)
            caches.append(c)
        z, rf, rstdf = self._head(y)
        t = np.asarray(targets)
        lse = _logsumexp(z)
        losses = lse - z[np.arange(n), t]
        if not need_grad:
            return losses, None
        if getattr(cfg, "inner_loss", "e2e") == "kvb":
            return losses, self._kvb_losses_and_grads(seq, caches)[1]
        # mean over the b positions of the chunk (reading R9)
        pz = np.exp(z - lse[:, None])
        pz[np.arange(n), t] -= 1.0
        dz = pz / cfg.minibatch_b
        dy = rms_norm_backward(y, w["final_norm"], rstdf, dz @ w["E"])
        grads = [None] * cfg.n_ttt
        for j in reversed(range(cfg.n_ttt)):
            c = caches[j]
            l = cfg.first_ttt + j
            p = f"layers.{l}."
            fw = seq.fast[j]
            # static MLP (frozen): only the data gradient
            dus = (dy @ w[p + "W2s"]) * gelu_prime(c["us"])
            dm = dy + rms_norm_backward(c["m"], w[p + "static_norm"], c["rstd3"], dus @ w[p + "W1s"])
            # TTT-MLP: weight gradients and data gradient, all at W_{i-1}
            dW2t = dm.T @ c["g"]
            du = (dm @ fw["W2t"]) * gelu_prime(c["u"])
            dW1t = du.T @ c["r2"]
            grads[j] = {"W1t": dW1t, "W2t": dW2t}
            if j == 0:
                break  # upstream of the first adaptive MLP does not depend on W
            da = dm + rms_norm_backward(c["a"], w[p + "ttt_norm"], c["rstd2"], du @ fw["W1t"])
            # frozen attention: data gradients; cached keys are constants (reading R3)
            do = (da @ w[p + "Wo"]).reshape(n, cfg.n_heads, cfg.head_dim)
            dq, dk_all, dv_all = window_attention_backward(c["q"], c["keys"], c["vals"], c["o"], c["probs"], do)
            nc = c["n_cached"]
            dq = rope_backward(dq, c["cos"], c["sin"]).reshape(n, -1)
            dk = rope_backward(dk_all[nc:], c["cos"], c["sin"]).reshape(n, -1)
            dv = dv_all[nc:].reshape(n, -1)
            dr1 = dq @ w[p + "Wq"] + dk @ w[p + "Wk"] + dv @ w[p + "Wv"]
            dy = da + rms_norm_backward(c["x"], w[p + "attn_norm"], c["rstd1"], dr1)
        return losses, grads

    def _kvb_losses_and_grads(self, seq, caches):
        """Layer-wise key-value-binding inner loss of every adaptive block and its
        gradient w.r.t. that block's fast weights (review §8, eq. (10); readings K1-K2)."""
        cfg, w = self.cfg, self.w
        losses, grads = [], []
        for j in range(cfg.n_ttt):
            p = f"layers.{cfg.first_ttt + j}."
            fw = seq.fast[j]
            c = caches[j]
            k = c["xin"]                      # theta_K r2: the MLP's input (reading K1)
            v = c["r2"] @ w[p + "theta_V"].T
            u, g = c["u"], c["g"]             # the forward's prediction g(k; W_{i-1})
            e = g @ fw["W2t"].T - v
            losses.append(float(np.sum(e * e)) / cfg.minibatch_b)
            de = (2.0 / cfg.minibatch_b) * e
            du = (de @ fw["W2t"]) * gelu_prime(u)
            grads.append({"W1t": du.T @ k, "W2t": de.T @ g})
        return losses, grads

    def _sgd(self, seq, grads):
        """W_i = W_{i-1} - eta * mean-gradient (summary, mini-batch GD equation)."""
        for j, g in enumerate(grads):
            for name in ("W1t", "W2t"):
                seq.fast[j][name] = seq.fast[j][name] - self.cfg.eta * g[name]

    # --------------------------------------------------------------- Algorithm 1
    def prefill(self, tokens):
        """tokens [B][T+1] -> losses [B][T] (reading R1). Updates the state."""
        cfg = self.cfg
        tokens = np.asarray(tokens)
        assert tokens.shape[0] == cfg.batch
        T = tokens.shape[1] - 1
        out = np.zeros((cfg.batch, T))
        b = cfg.minibatch_b
        for si, seq in enumerate(self.seqs):
            tok = tokens[si]
            if seq.pend_inputs:
                raise ValueError("prefill while a decode chunk is pending")
            if seq.n_pos > 0 and tok[0] != seq.pending_token:
                raise ValueError("stream continuity: first id must be the pending token")
            s0 = seq.n_pos
            h = self._frozen_forward(seq, tok[:T], s0, commit=True)
            for c0 in range(0, T, b):
                c1 = min(T, c0 + b)
                full = (c1 - c0) == b
                losses, grads = self._chunk(seq, h[c0:c1], s0 + c0, tok[c0 + 1:c1 + 1],
                                            need_grad=full, commit=True)
                out[si, c0:c1] = losses
                if full:
                    self._sgd(seq, grads)
                else:  # reading R10
                    seq.pend_inputs = list(h[c0:c1])
                    seq.pend_targets = list(tok[c0 + 1:c1 + 1])
            seq.n_pos = s0 + T
            seq.pending_token = int(tok[T])
        return out

    # --------------------------------------------------------------- Algorithm 3
    def decode(self, n, forced=None):
        """Generate n tokens per sequence (greedy unless forced [B][n] is given).

        Returns dict(tokens, losses, z_chosen, z_max), each [B][n].
        """
        cfg = self.cfg
        b = cfg.minibatch_b
        res = {k: np.zeros((cfg.batch, n)) for k in ("losses", "z_chosen", "z_max")}
        res["tokens"] = np.zeros((cfg.batch, n), dtype=np.int64)
        for si, seq in enumerate(self.seqs):
            for t in range(n):
                p = seq.n_pos
                h = self._frozen_forward(seq, [seq.pending_token], p, commit=True)
                y = h
                for j in range(cfg.n_ttt):
                    y, _ = self._ttt_block(seq, j, y, p, commit=True, keep=False)
                z = self._head(y)[0][0]
                zmax = z.max()
                tok = int(np.argmax(z)) if forced is None else int(forced[si][t])  # reading R11
                res["tokens"][si, t] = tok
                res["losses"][si, t] = _logsumexp(z[None])[0] - z[tok]
                res["z_chosen"][si, t] = z[tok]
                res["z_max"][si, t] = zmax
                seq.pend_inputs.append(h[0])
                seq.pend_targets.append(tok)
                seq.n_pos = p + 1
                seq.pending_token = tok
                if seq.n_pos % b == 0:
                    s = seq.n_pos - b
                    _, grads = self._chunk(seq, np.stack(seq.pend_inputs), s, seq.pend_targets,
                                           need_grad=True, commit=False)
                    self._sgd(seq, grads)
                    seq.pend_inputs, seq.pend_targets = [], []
        return res

    # --------------------------------------------------------------- outer loop (Algorithm 2)
    def meta_gradient(self, tokens, step=1e-30):
        """Outer-loop gradient for one sequence (tokens [T+1], T = N b; readings M1-M2).

        Forward: Algorithm 1 from W_0 with the chunk gradients g_i = grad A_i(W_{i-1})
        and the states W_{i-1} kept. Backward, eq. (7) accumulated from the last chunk:
        lambda_N = g_N, lambda_i = g_i + (I - eta H_{A_i}(W_{i-1})) lambda_{i+1}
        (H symmetric, so J^T products become this recursion); grad = lambda_1 / N.
        The oracle's own state is not used or changed. Returns (L, grads) with grads
        a list of {"W1t", "W2t"} per adaptive block.
        """
        cfg = self.cfg
        assert getattr(cfg, "inner_loss", "e2e") == "e2e", "eq. (7) is written for the next-token inner loss"
        tok = np.asarray(tokens)
        T = tok.shape[0] - 1
        b, eta = cfg.minibatch_b, cfg.eta
        assert T > 0 and T % b == 0, "reading M2: T must be a multiple of b"
        N = T // b
        st = _Seq(cfg, self.w)
        h = self._frozen_forward(st, tok[:T], 0, commit=True)
        Ws, gs, means = [], [], []
        for i in range(N):
            c0 = i * b
            Ws.append([{n: W.copy() for n, W in f.items()} for f in st.fast])
            losses, grads = self._chunk(st, h[c0:c0 + b], c0, tok[c0 + 1:c0 + b + 1], need_grad=True, commit=True)
            means.append(float(np.mean(losses)))
            gs.append(grads)
            self._sgd(st, grads)

        def hvp(i, v):
            # H_{A_i}(W_{i-1}) v by the complex step; chunk i reads the cache of positions < i b
            c0 = i * b
            st.fast = [{n: Ws[i][j][n] + 1j * step * v[j][n] for n in ("W1t", "W2t")} for j in range(cfg.n_ttt)]
            _, gc = self._chunk(st, h[c0:c0 + b], c0, tok[c0 + 1:c0 + b + 1], need_grad=True, commit=False)
            return [{n: np.imag(gc[j][n]) / step for n in ("W1t", "W2t")} for j in range(cfg.n_ttt)]

        lam = [{n: G.copy() for n, G in g.items()} for g in gs[N - 1]]
        for i in range(N - 2, -1, -1):
            hv = hvp(i, lam)
            lam = [{n: gs[i][j][n] + lam[j][n] - eta * hv[j][n] for n in ("W1t", "W2t")} for j in range(cfg.n_ttt)]
        return float(np.mean(means)), [{n: G / N for n, G in g.items()} for g in lam]

    def chunk_hvp(self, seq, tokens_chunk, v, step=1e-30):
        """H v of the next full chunk's mean loss at the current fast weights (the
        complex-step product used by meta_gradient), without changing any state."""
        st = self.seqs[seq]
        cfg = self.cfg
        assert len(tokens_chunk) == cfg.minibatch_b + 1 and not st.pend_inputs
        h = self._frozen_forward(st, tokens_chunk[:-1], st.n_pos, commit=False)
        saved = st.fast
        st.fast = [{n: saved[j][n] + 1j * step * v[j][n] for n in ("W1t", "W2t")} for j in range(cfg.n_ttt)]
        try:
            _, gc = self._chunk(st, h, st.n_pos, tokens_chunk[1:], need_grad=True, commit=False)
        finally:
            st.fast = saved
        return [{n: np.imag(gc[j][n]) / step for n in ("W1t", "W2t")} for j in range(cfg.n_ttt)]

    # --------------------------------------------------------------- inspection
    def fast_weights(self, seq, j):
        """(W1t [h_t][d], W2t [d][h_t]) of adaptive block j of sequence seq."""
        f = self.seqs[seq].fast[j]
        return f["W1t"].copy(), f["W2t"].copy()

    def chunk_loss_and_grad(self, seq, tokens_chunk):
        """Mean loss and gradient of the next full chunk, without changing any state.

        tokens_chunk holds b+1 ids: the pending token followed by the chunk's b
        targets. Used by the finite-difference pins.
        """
        st = self.seqs[seq]
        cfg = self.cfg
        assert len(tokens_chunk) == cfg.minibatch_b + 1 and not st.pend_inputs
        h = self._frozen_forward(st, tokens_chunk[:-1], st.n_pos, commit=False)
        losses, grads = self._chunk(st, h, st.n_pos, tokens_chunk[1:], need_grad=True, commit=False)
        return float(np.mean(losses)), grads

    def chunk_inner_losses_and_grads(self, seq, tokens_chunk):
        """Key-value-binding variant: each adaptive block's inner loss on the next full
        chunk and its gradient, without changing any state (tokens_chunk as above)."""
        st = self.seqs[seq]
        cfg = self.cfg
        assert len(tokens_chunk) == cfg.minibatch_b + 1 and not st.pend_inputs
        y = self._frozen_forward(st, tokens_chunk[:-1], st.n_pos, commit=False)
        caches = []
        for j in range(cfg.n_ttt):
            y, c = self._ttt_block(st, j, y, st.n_pos, commit=False, keep=True)
            caches.append(c)
        return self._kvb_losses_and_grads(st, caches)
