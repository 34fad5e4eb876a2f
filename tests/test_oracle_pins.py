"""Pins of the CPU oracle against facts fixed by the pages and by mathematics.

Each test names what it pins:
  * finite differences (float64, central) of every primitive and of a chunk's
    mean loss w.r.t. the fast weights, with the window cache held constant;
  * an independent whole-sequence float64 PyTorch forward (tests/torch_static.py)
    and its autograd: eta=0 gives the static sliding-window model's losses
    ("disable updates", review §9.3); b=T gives exactly one update
    (review §5 and §9.2); with one adaptive block the whole mini-batch
    trajectory equals the autograd loop (summary, mini-batch GD equation;
    review eq. (9)); b=1 is online GD (review eq. (3));
  * k >= T equals textbook causal softmax attention (review §9.2: an 8K window
    at 8K length is full attention);
  * causality of scoring (review §2.2 and §7, Algorithm 1), only the
    adaptive MLPs change (summary, "Selective Parameter Update"), sequences are
    independent (review §7, Algorithms 1 and 2), decode updates only
    after a full chunk (summary, "Decoding Multiple Tokens"; review Alg. 3).
"""
import math

import numpy as np
import pytest
import torch

import synthetic as syn
from oracle import Oracle
from oracle import ttt_oracle as O
from tests import torch_static as TS


def tiny(n_ttt=1, **kw):
    base = dict(name="pin", vocab=16, d=8, n_layers=4, n_heads=2, n_ttt=n_ttt, mlp_hidden=16,
                ttt_hidden=8, static_hidden=8, window_k=4, minibatch_b=4, batch=1, eta=0.5,
                T=16, dtype="fp32", weight_seed=7, token_seed=9)
    base.update(kw)
    return syn.TTTConfig(**base)


def weights(cfg, std=0.5):
    return syn.make_weights(cfg, std=std)


def tokens(cfg, n=None, batch=None):
    return syn.make_token_batch(cfg, n=n, batch=batch)


# ----------------------------------------------------------------------------- primitives

def _fd(f, x, eps=1e-6):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = x[i]
        x[i] = old + eps
        fp = f()
        x[i] = old - eps
        fm = f()
        x[i] = old
        g[i] = (fp - fm) / (2 * eps)
    return g


def test_rms_norm_backward_matches_finite_differences():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((3, 8))
    g = rng.standard_normal(8)
    dy = rng.standard_normal((3, 8))
    _, rstd = O.rms_norm(x, g, 1e-6)
    an = O.rms_norm_backward(x, g, rstd, dy)
    num = _fd(lambda: float(np.sum(O.rms_norm(x, g, 1e-6)[0] * dy)), x)
    np.testing.assert_allclose(an, num, rtol=1e-7, atol=1e-8)


def test_rms_norm_is_library_rms_norm():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 16))
    g = rng.standard_normal(16)
    ref = torch.nn.functional.rms_norm(torch.tensor(x), (16,), weight=torch.tensor(g), eps=1e-6).numpy()
    np.testing.assert_allclose(O.rms_norm(x, g, 1e-6)[0], ref, rtol=1e-12, atol=1e-12)


def test_gelu_is_exact_erf_form_and_derivative():
    u = np.linspace(-6, 6, 101)
    ref = torch.nn.functional.gelu(torch.tensor(u), approximate="none").numpy()
    np.testing.assert_allclose(O.gelu(u), ref, rtol=1e-12, atol=1e-14)
    num = (O.gelu(u + 1e-6) - O.gelu(u - 1e-6)) / 2e-6
    np.testing.assert_allclose(O.gelu_prime(u), num, rtol=1e-6, atol=1e-8)


def test_rope_is_rotation_and_backward_is_its_transpose():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((6, 2, 8))
    cos, sin = O.rope_tables(np.arange(10, 16), 8, 10000.0)
    y = O.rope(x, cos, sin)
    # a rotation keeps pairwise norms
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-12)
    # position 0 is the identity
    c0, s0 = O.rope_tables(np.array([0]), 8, 10000.0)
    np.testing.assert_allclose(O.rope(x[:1], c0, s0), x[:1], rtol=0, atol=0)
    # backward = transpose: <rope(x), dy> = <x, rope_backward(dy)>
    dy = rng.standard_normal(x.shape)
    assert abs(np.sum(y * dy) - np.sum(x * O.rope_backward(dy, cos, sin))) < 1e-10
    # pair (i, i+hd/2) at position p rotates by p * base^(-2i/hd): check one entry by hand
    p, i, hd = 13, 1, 8
    ang = p * 10000.0 ** (-2 * i / hd)
    row = 3  # position 13
    exp0 = x[row, 0, i] * math.cos(ang) - x[row, 0, i + 4] * math.sin(ang)
    assert abs(y[row, 0, i] - exp0) < 1e-12
    # relative-position property of the scores: <R_p q, R_s k> depends on p - s only
    q, k = rng.standard_normal((1, 1, 8)), rng.standard_normal((1, 1, 8))
    def score(pq, pk):
        cq, sq = O.rope_tables(np.array([pq]), 8, 10000.0)
        ck, sk = O.rope_tables(np.array([pk]), 8, 10000.0)
        return float(np.sum(O.rope(q, cq, sq) * O.rope(k, ck, sk)))
    assert abs(score(20, 17) - score(103, 100)) < 1e-10


def test_window_attention_full_window_is_textbook_causal_attention():
    rng = np.random.default_rng(3)
    n, H, hd = 12, 3, 4
    q, k, v = (rng.standard_normal((n, H, hd)) for _ in range(3))
    pos = np.arange(n)
    o, _ = O.window_attention(q, k, v, pos, pos, window=n + 5)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q).transpose(0, 1), torch.tensor(k).transpose(0, 1), torch.tensor(v).transpose(0, 1),
        is_causal=True).transpose(0, 1).numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-12)


def test_window_attention_window_one_returns_values():
    rng = np.random.default_rng(4)
    q, k, v = (rng.standard_normal((5, 2, 4)) for _ in range(3))
    pos = np.arange(5)
    o, _ = O.window_attention(q, k, v, pos, pos, window=1)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-15)


def test_window_attention_backward_matches_finite_differences():
    rng = np.random.default_rng(5)
    n, m, H, hd = 4, 7, 2, 4
    q = rng.standard_normal((n, H, hd))
    keys = rng.standard_normal((m, H, hd))
    vals = rng.standard_normal((m, H, hd))
    qpos = np.arange(3, 7)
    kpos = np.arange(0, 7)
    do = rng.standard_normal((n, H, hd))
    o, p = O.window_attention(q, keys, vals, qpos, kpos, window=4, keep_probs=True)
    dq, dk, dv = O.window_attention_backward(q, keys, vals, o, p, do)
    f = lambda: float(np.sum(O.window_attention(q, keys, vals, qpos, kpos, 4)[0] * do))
    np.testing.assert_allclose(dq, _fd(f, q), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dk, _fd(f, keys), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dv, _fd(f, vals), rtol=1e-6, atol=1e-8)


# ----------------------------------------------------------------------------- whole method

@pytest.mark.parametrize("n_ttt", [1, 2])
def test_chunk_gradient_matches_finite_differences_with_constant_cache(n_ttt):
    """Hand-written reverse mode of a chunk's mean loss, chunk 3 (cache non-empty)."""
    cfg = tiny(n_ttt=n_ttt, T=8)
    w = weights(cfg)
    toks = tokens(cfg, n=cfg.T + 1 + cfg.minibatch_b)
    orc = Oracle(cfg, w)
    orc.prefill(toks[:, :cfg.T + 1])
    chunk = toks[0, cfg.T:cfg.T + cfg.minibatch_b + 1]
    _, grads = orc.chunk_loss_and_grad(0, chunk)
    for j in range(cfg.n_ttt):
        for name in ("W1t", "W2t"):
            W = orc.seqs[0].fast[j][name]
            num = _fd(lambda: orc.chunk_loss_and_grad(0, chunk)[0], W)
            np.testing.assert_allclose(grads[j][name], num, rtol=1e-5, atol=1e-9)


@pytest.mark.parametrize("n_ttt", [0, 1, 2])
def test_eta_zero_reproduces_static_swa_model(n_ttt):
    cfg = tiny(n_ttt=n_ttt, eta=0.0, T=24)
    w = weights(cfg)
    toks = tokens(cfg)
    orc = Oracle(cfg, w)
    losses = orc.prefill(toks)
    ref = TS.static_forward(cfg, w, toks[0]).numpy()
    np.testing.assert_allclose(losses[0], ref, rtol=1e-10, atol=1e-12)
    for j in range(cfg.n_ttt):
        l = cfg.first_ttt + j
        W1, W2 = orc.fast_weights(0, j)
        assert np.array_equal(W1, w[f"layers.{l}.W1t"].astype(np.float64))
        assert np.array_equal(W2, w[f"layers.{l}.W2t"].astype(np.float64))


@pytest.mark.parametrize("n_ttt", [0, 1, 2])
def test_full_window_reproduces_full_causal_attention_model(n_ttt):
    cfg = tiny(n_ttt=n_ttt, eta=0.0, window_k=64, minibatch_b=8, T=24)
    w = weights(cfg)
    toks = tokens(cfg)
    losses = Oracle(cfg, w).prefill(toks)
    # independent: textbook causal attention through SDPA's is_causal flag
    big = cfg.replace(window_k=10 ** 6)
    ref = TS.static_forward(big, w, toks[0]).numpy()
    np.testing.assert_allclose(losses[0], ref, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("n_ttt", [1, 2])
def test_b_equals_T_is_exactly_one_update(n_ttt):
    cfg = tiny(n_ttt=n_ttt, T=16, minibatch_b=16, window_k=16)
    w = weights(cfg)
    toks = tokens(cfg)
    orc = Oracle(cfg, w)
    losses = orc.prefill(toks)
    fast = TS.initial_fast(cfg, w, requires_grad=True)
    ref_losses = TS.static_forward(cfg, w, toks[0], fast=fast)
    np.testing.assert_allclose(losses[0], ref_losses.detach().numpy(), rtol=1e-10, atol=1e-12)
    ref_losses.mean().backward()
    for j in range(cfg.n_ttt):
        W1, W2 = orc.fast_weights(0, j)
        np.testing.assert_allclose(W1, (fast[j]["W1t"] - cfg.eta * fast[j]["W1t"].grad).detach().numpy(),
                                   rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(W2, (fast[j]["W2t"] - cfg.eta * fast[j]["W2t"].grad).detach().numpy(),
                                   rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("b,k", [(4, 4), (4, 8), (1, 3)])
def test_single_adaptive_block_trajectory_matches_autograd_loop(b, k):
    """Chunk i scored with W_{i-1}; W_i = W_{i-1} - eta grad A_i(W_{i-1}); b=1 is eq. (3)."""
    cfg = tiny(n_ttt=1, minibatch_b=b, window_k=k, T=14)
    w = weights(cfg)
    toks = tokens(cfg)
    orc = Oracle(cfg, w)
    losses = orc.prefill(toks)
    ref_losses, ref_fast = TS.mini_batch_ttt_single_adaptive_block(cfg, w, toks[0])
    np.testing.assert_allclose(losses[0], ref_losses.numpy(), rtol=1e-10, atol=1e-12)
    W1, W2 = orc.fast_weights(0, 0)
    np.testing.assert_allclose(W1, ref_fast[0]["W1t"].numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(W2, ref_fast[0]["W2t"].numpy(), rtol=1e-10, atol=1e-12)


def test_first_chunk_losses_do_not_depend_on_eta():
    cfg = tiny(n_ttt=2, T=16)
    w = weights(cfg)
    toks = tokens(cfg)
    a = Oracle(cfg, w).prefill(toks)
    b = Oracle(cfg.replace(eta=0.0), w).prefill(toks)
    assert np.array_equal(a[0, :4], b[0, :4])
    assert not np.allclose(a[0, 4:], b[0, 4:])


def test_scoring_is_causal():
    cfg = tiny(n_ttt=2, T=20)
    w = weights(cfg)
    toks = tokens(cfg)
    base = Oracle(cfg, w).prefill(toks)
    for q in (3, 9, 14):
        t2 = toks.copy()
        t2[0, q] = (t2[0, q] + 5) % cfg.vocab
        pert = Oracle(cfg, w).prefill(t2)
        # l_t uses x_{t-1} as input and x_t as target: positions t <= q-1 (0-based losses[:q]) see nothing of x_q
        assert np.array_equal(base[0, :q - 1], pert[0, :q - 1])
        assert not np.array_equal(base[0, q - 1:], pert[0, q - 1:])


def test_information_beyond_the_window_flows_only_through_fast_weights():
    # receptive field of the attention stack is n_layers * (k - 1) positions
    cfg = tiny(n_ttt=2, window_k=4, minibatch_b=4, T=40)
    w = weights(cfg)
    toks = tokens(cfg)
    t2 = toks.copy()
    t2[0, 1] = (t2[0, 1] + 3) % cfg.vocab
    far = slice(32, 40)  # beyond 4 * 3 positions of the perturbed chunk
    with_upd = Oracle(cfg, w).prefill(toks), Oracle(cfg, w).prefill(t2)
    assert not np.allclose(with_upd[0][0, far], with_upd[1][0, far])
    z = cfg.replace(eta=0.0)
    no_upd = Oracle(z, w).prefill(toks), Oracle(z, w).prefill(t2)
    assert np.array_equal(no_upd[0][0, far], no_upd[1][0, far])


def test_only_adaptive_mlps_change():
    cfg = tiny(n_ttt=2, T=16)
    w = weights(cfg)
    orc = Oracle(cfg, w)
    before = {k: v.copy() for k, v in orc.w.items()}
    orc.prefill(tokens(cfg))
    for k in before:
        assert np.array_equal(before[k], orc.w[k])
    for j in range(cfg.n_ttt):
        W1, _ = orc.fast_weights(0, j)
        assert not np.array_equal(W1, before[f"layers.{cfg.first_ttt + j}.W1t"])


def test_sequences_are_independent():
    cfg = tiny(n_ttt=2, T=12, batch=3)
    w = weights(cfg)
    toks = tokens(cfg)
    together = Oracle(cfg, w).prefill(toks)
    one = cfg.replace(batch=1)
    for s in range(3):
        alone = Oracle(one, w).prefill(toks[s:s + 1])
        np.testing.assert_array_equal(together[s], alone[0])


def test_prefill_split_at_chunk_boundary_equals_one_call():
    cfg = tiny(n_ttt=2, T=20)
    w = weights(cfg)
    toks = tokens(cfg)
    one = Oracle(cfg, w)
    l1 = one.prefill(toks)
    two = Oracle(cfg, w)
    a = two.prefill(toks[:, :9])
    b = two.prefill(toks[:, 8:])
    np.testing.assert_allclose(np.concatenate([a, b], axis=1), l1, rtol=1e-12, atol=1e-13)
    for j in range(cfg.n_ttt):
        np.testing.assert_allclose(two.fast_weights(0, j)[0], one.fast_weights(0, j)[0], rtol=1e-12, atol=1e-13)


def test_teacher_forced_decode_equals_prefill():
    cfg = tiny(n_ttt=2, T=8)
    w = weights(cfg)
    toks = tokens(cfg, n=8 + 1 + 10)
    full = Oracle(cfg, w)
    lf = full.prefill(toks)
    dec = Oracle(cfg, w)
    lp = dec.prefill(toks[:, :9])
    r = dec.decode(10, forced=toks[:, 9:])
    np.testing.assert_allclose(np.concatenate([lp, r["losses"]], axis=1), lf, rtol=1e-10, atol=1e-12)
    # 8 + 10 = 18 positions: chunks 1..4 updated, positions 16, 17 pending
    for j in range(cfg.n_ttt):
        np.testing.assert_allclose(dec.fast_weights(0, j)[1], full.fast_weights(0, j)[1], rtol=1e-10, atol=1e-12)
    assert len(dec.seqs[0].pend_inputs) == 2


def test_partial_prefill_chunk_is_completed_by_decode():
    cfg = tiny(n_ttt=2, T=10)
    w = weights(cfg)
    toks = tokens(cfg, n=17)
    full = Oracle(cfg, w)
    lf = full.prefill(toks)
    dec = Oracle(cfg, w)
    lp = dec.prefill(toks[:, :11])       # positions 0..9: chunks 1, 2 updated; 8, 9 pending
    w_before = dec.fast_weights(0, 1)[0]
    r = dec.decode(6, forced=toks[:, 11:])
    np.testing.assert_allclose(np.concatenate([lp, r["losses"]], axis=1), lf, rtol=1e-10, atol=1e-12)
    assert not np.array_equal(w_before, dec.fast_weights(0, 1)[0])
    np.testing.assert_allclose(dec.fast_weights(0, 1)[0], full.fast_weights(0, 1)[0], rtol=1e-10, atol=1e-12)


def test_greedy_decode_picks_argmax_and_reports_its_loss():
    cfg = tiny(n_ttt=1, T=8)
    w = weights(cfg)
    orc = Oracle(cfg, w)
    orc.prefill(tokens(cfg))
    r = orc.decode(6)
    assert np.array_equal(r["z_chosen"], r["z_max"])
    assert np.all(r["losses"] > 0)


def test_cross_entropy_gradient_rows_sum_to_zero():
    # dz = (softmax - onehot)/b sums to zero per row, so E's mean row does not move drf
    cfg = tiny(n_ttt=1)
    w = weights(cfg)
    orc = Oracle(cfg, w)
    z = np.random.default_rng(0).standard_normal((4, cfg.vocab))
    lse = O._logsumexp(z)
    p = np.exp(z - lse[:, None])
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=1e-14)
    assert np.all(lse - z.max(axis=1) >= 0)


# ----------------------------------------------------------------------------- window cache of later adaptive blocks

@pytest.mark.parametrize("n_ttt,b,k,T", [(2, 4, 6, 16), (3, 4, 9, 18), (2, 3, 5, 14)])
def test_multi_block_trajectory_matches_chunkwise_autograd_with_cache_as_computed(n_ttt, b, k, T):
    """With two or more adaptive blocks the keys/values that a later adaptive block caches
    depend on W. Reading R4: a cached key/value keeps the value computed when its chunk ran
    (with that chunk's W_{i-1}) and is a constant afterwards (technical review §7,
    Algorithm 1, attention state carried across chunks; §5, eq. (9)). An independent
    chunk-wise loop (library SDPA and autograd, tests/torch_static.py) must reproduce the
    oracle's losses and final fast weights; the two plausible misreadings must not."""
    cfg = tiny(n_ttt=n_ttt, minibatch_b=b, window_k=k, T=T, eta=0.5)
    w = weights(cfg)
    toks = tokens(cfg)
    orc = Oracle(cfg, w)
    losses = orc.prefill(toks)
    ref_losses, ref_fast = TS.mini_batch_ttt_chunked(cfg, w, toks[0], "as_computed")
    np.testing.assert_allclose(losses[0], ref_losses.numpy(), rtol=1e-10, atol=1e-12)
    for j in range(n_ttt):
        W1, W2 = orc.fast_weights(0, j)
        np.testing.assert_allclose(W1, ref_fast[j]["W1t"].numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(W2, ref_fast[j]["W2t"].numpy(), rtol=1e-10, atol=1e-12)
    # negative controls, far outside the tolerance above: recomputing the cache with the
    # current W changes chunk 2 on (chunk 1's K/V would carry W_1 instead of W_0); keeping
    # the K/V of W_0 agrees through chunk 2 (chunk 1 ran with W_0) and changes chunk 3 on
    for rule, same in (("recompute_current", b), ("initial_weights", 2 * b)):
        alt, _ = TS.mini_batch_ttt_chunked(cfg, w, toks[0], rule)
        np.testing.assert_allclose(alt[:same].numpy(), losses[0, :same], rtol=1e-10, atol=1e-12)
        assert np.max(np.abs(alt[same:same + b].numpy() - losses[0, same:same + b])) > 1e-6, rule


def test_chunkwise_autograd_reduces_to_the_static_loop_with_one_adaptive_block():
    """Cross-check of the two autograd references: with one adaptive block nothing cached
    depends on W, so every cache rule gives the whole-sequence loop's trajectory."""
    cfg = tiny(n_ttt=1, minibatch_b=4, window_k=6, T=14)
    w = weights(cfg)
    toks = tokens(cfg)
    ref_losses, ref_fast = TS.mini_batch_ttt_single_adaptive_block(cfg, w, toks[0])
    for rule in ("as_computed", "recompute_current", "initial_weights"):
        got, fast = TS.mini_batch_ttt_chunked(cfg, w, toks[0], rule)
        np.testing.assert_allclose(got.numpy(), ref_losses.numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(fast[0]["W1t"].numpy(), ref_fast[0]["W1t"].numpy(), rtol=1e-10, atol=1e-12)


# ----------------------------------------------------------------------------- key-value-binding inner loss (variant)

def tiny_kvb(n_ttt=2, **kw):
    # a smaller step than the next-token pins: with these weights (std 0.5) the
    # reconstruction errors are O(1) per component and eta = 0.5 diverges
    kw.setdefault("eta", 0.02)
    return tiny(n_ttt=n_ttt, inner_loss="kvb", **kw)


@pytest.mark.parametrize("n_ttt", [1, 2])
def test_kvb_gradient_matches_finite_differences(n_ttt):
    """Hand-written gradient of each block's reconstruction loss (technical review §8,
    eq. (10)) w.r.t. that block's fast weights, on chunk 3 (window cache non-empty)."""
    cfg = tiny_kvb(n_ttt=n_ttt, T=8)
    w = weights(cfg)
    toks = tokens(cfg, n=cfg.T + 1 + cfg.minibatch_b)
    orc = Oracle(cfg, w)
    orc.prefill(toks[:, :cfg.T + 1])
    chunk = toks[0, cfg.T:cfg.T + cfg.minibatch_b + 1]
    losses, grads = orc.chunk_inner_losses_and_grads(0, chunk)
    assert all(v > 0 for v in losses)
    for j in range(cfg.n_ttt):
        for name in ("W1t", "W2t"):
            W = orc.seqs[0].fast[j][name]
            num = _fd(lambda: orc.chunk_inner_losses_and_grads(0, chunk)[0][j], W)
            # central differences of losses of size ~100 carry ~1e-8 of rounding
            np.testing.assert_allclose(grads[j][name], num, rtol=1e-5, atol=1e-7)


@pytest.mark.parametrize("n_ttt,b,k,T", [(2, 4, 6, 16), (3, 4, 9, 18), (1, 3, 5, 14)])
def test_kvb_trajectory_matches_chunkwise_autograd(n_ttt, b, k, T):
    """The whole prefill with the reconstruction inner loss against an independent
    chunk-wise loop (library mse_loss, SDPA and autograd, tests/torch_static.py): losses
    and final fast weights. Negative controls: letting each block's loss reach the
    earlier blocks' weights (not layer-wise) and the next-token inner loss both move the
    first adaptive block's weights far outside the tolerance, and applying the MLP to
    the normalised rows themselves on the output path (instead of reusing the
    prediction from the key projection, technical review §8 / summary step 3) moves
    the recorded losses far outside it."""
    cfg = tiny_kvb(n_ttt=n_ttt, minibatch_b=b, window_k=k, T=T)
    w = weights(cfg)
    toks = tokens(cfg)
    orc = Oracle(cfg, w)
    losses = orc.prefill(toks)
    ref_losses, ref_fast = TS.mini_batch_ttt_kvb_chunked(cfg, w, toks[0])
    np.testing.assert_allclose(losses[0], ref_losses.numpy(), rtol=1e-10, atol=1e-12)
    for j in range(n_ttt):
        W1, W2 = orc.fast_weights(0, j)
        np.testing.assert_allclose(W1, ref_fast[j]["W1t"].numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(W2, ref_fast[j]["W2t"].numpy(), rtol=1e-10, atol=1e-12)
    W1_0 = orc.fast_weights(0, 0)[0]
    if n_ttt > 1:
        _, joint = TS.mini_batch_ttt_kvb_chunked(cfg, w, toks[0], layerwise=False)
        assert np.max(np.abs(joint[0]["W1t"].numpy() - W1_0)) > 1e-6
    e2e = Oracle(cfg.replace(inner_loss="e2e"), w)
    e2e.prefill(toks)
    assert np.max(np.abs(e2e.fast_weights(0, 0)[0] - W1_0)) > 1e-6
    other, _ = TS.mini_batch_ttt_kvb_chunked(cfg, w, toks[0], output_from_keys=False)
    assert np.max(np.abs(other.numpy() - losses[0])) > 1e-6


def test_kvb_zero_key_projection_never_moves_the_weights():
    """theta_K = 0: every key is 0, so the MLP's prediction gelu(W1t k) W2t, which is
    also the sub-layer's output, is 0, and both weight gradients vanish (dW2t pairs the
    error with gelu(0) = 0, dW1t pairs it with k = 0): the prefill is the static model
    without the adaptive MLPs (their W2t zeroed) and the fast weights stay W_init."""
    cfg = tiny_kvb(n_ttt=2, T=16)
    w = weights(cfg)
    for l in range(cfg.first_ttt, cfg.n_layers):
        w[f"layers.{l}.theta_K"] = np.zeros_like(w[f"layers.{l}.theta_K"])
    toks = tokens(cfg)
    orc = Oracle(cfg, w)
    losses = orc.prefill(toks)
    w_off = dict(w)
    for l in range(cfg.first_ttt, cfg.n_layers):
        w_off[f"layers.{l}.W2t"] = np.zeros_like(w[f"layers.{l}.W2t"])
    np.testing.assert_allclose(losses[0], TS.static_forward(cfg, w_off, toks[0]).numpy(), rtol=1e-10, atol=1e-12)
    assert np.max(np.abs(losses[0] - TS.static_forward(cfg, w, toks[0]).numpy())) > 1e-6
    for j in range(cfg.n_ttt):
        l = cfg.first_ttt + j
        assert np.array_equal(orc.fast_weights(0, j)[0], w[f"layers.{l}.W1t"].astype(np.float64))
        assert np.array_equal(orc.fast_weights(0, j)[1], w[f"layers.{l}.W2t"].astype(np.float64))


def test_kvb_teacher_forced_decode_equals_prefill():
    """Decode's update after a full chunk of generated tokens uses the same inner loss
    (review §7, Algorithm 3)."""
    cfg = tiny_kvb(n_ttt=2, T=8)
    w = weights(cfg)
    toks = tokens(cfg, n=8 + 1 + 10)
    full = Oracle(cfg, w)
    lf = full.prefill(toks)
    dec = Oracle(cfg, w)
    lp = dec.prefill(toks[:, :9])
    r = dec.decode(10, forced=toks[:, 9:])
    np.testing.assert_allclose(np.concatenate([lp, r["losses"]], axis=1), lf, rtol=1e-10, atol=1e-12)
    for j in range(cfg.n_ttt):
        np.testing.assert_allclose(dec.fast_weights(0, j)[0], full.fast_weights(0, j)[0], rtol=1e-10, atol=1e-12)


# ----------------------------------------------------------------------------- outer-loop meta-gradient

def _outer_loss(cfg, w, toks):
    return float(np.mean(Oracle(cfg, w).prefill(toks)[0]))


def _with_initial_fast(cfg, w, delta, scale):
    w2 = dict(w)
    for j in range(cfg.n_ttt):
        l = cfg.first_ttt + j
        for n in ("W1t", "W2t"):
            w2[f"layers.{l}.{n}"] = w[f"layers.{l}.{n}"].astype(np.float64) + scale * delta[j][n]
    return w2


def test_meta_gradient_matches_finite_differences_of_the_outer_loss():
    """Eq. (7) of the technical review (§4) against central differences of the scored
    mean loss L(W_0) = mean of Algorithm 1's losses, along random directions. One
    adaptive block: its keys/values do not depend on W, so eq. (7) is the whole
    derivative. Negative control: dropping the -eta H term (the first-order
    approximation eq. (6) warns against) misses far outside the tolerance."""
    cfg = tiny(n_ttt=1, T=16)
    w = weights(cfg)
    toks = tokens(cfg)
    orc = Oracle(cfg, w)
    L, grad = orc.meta_gradient(toks[0])
    assert L == pytest.approx(_outer_loss(cfg, w, toks), rel=1e-12)
    first_order = [{n: np.zeros_like(g[n]) for n in g} for g in grad]
    st = Oracle(cfg, w)
    b, N = cfg.minibatch_b, cfg.T // cfg.minibatch_b
    for i in range(N):                    # (1/N) sum_i grad A_i(W_{i-1}) along the same trajectory
        _, g = st.chunk_loss_and_grad(0, toks[0, i * b:(i + 1) * b + 1])
        for j in range(cfg.n_ttt):
            for n in g[j]:
                first_order[j][n] += g[j][n] / N
        st.prefill(toks[:, i * b:(i + 1) * b + 1])
    rng = np.random.default_rng(3)
    eps = 1e-5
    for _ in range(3):
        v = [{n: rng.standard_normal(grad[j][n].shape) for n in grad[j]} for j in range(cfg.n_ttt)]
        fd = (_outer_loss(cfg, _with_initial_fast(cfg, w, v, eps), toks)
              - _outer_loss(cfg, _with_initial_fast(cfg, w, v, -eps), toks)) / (2 * eps)
        dot = sum(float(np.sum(grad[j][n] * v[j][n])) for j in range(cfg.n_ttt) for n in v[j])
        fo = sum(float(np.sum(first_order[j][n] * v[j][n])) for j in range(cfg.n_ttt) for n in v[j])
        assert dot == pytest.approx(fd, rel=1e-6, abs=1e-8)
        assert abs(fo - fd) > 1e-3 * abs(fd)


@pytest.mark.parametrize("n_ttt,b,k,T", [(1, 4, 4, 16), (2, 4, 6, 16), (3, 3, 5, 12)])
def test_meta_gradient_matches_autograd_through_the_unrolled_updates(n_ttt, b, k, T):
    """Eq. (7) against the library's reverse-over-reverse (tests/torch_static.py:
    create_graph through every inner gradient, earlier keys/values detached as the
    inner loop holds them, reading M1), for 1-3 adaptive blocks and 4 chunks."""
    cfg = tiny(n_ttt=n_ttt, minibatch_b=b, window_k=k, T=T)
    w = weights(cfg)
    toks = tokens(cfg)
    L, grad = Oracle(cfg, w).meta_gradient(toks[0])
    Lr, ref = TS.outer_gradient_chunked(cfg, w, toks[0])
    assert L == pytest.approx(Lr, rel=1e-12)
    for j in range(n_ttt):
        for n in ("W1t", "W2t"):
            np.testing.assert_allclose(grad[j][n], ref[j][n].numpy(), rtol=1e-9, atol=1e-12)


def test_meta_gradient_with_eta_zero_is_the_static_model_gradient():
    """eta = 0: every J_i is the identity and every W_i = W_0, so eq. (7) reduces to the
    gradient of the static model's mean loss (autograd of the whole-sequence forward).
    One adaptive block, so that no key or value the whole-sequence autograd
    differentiates depends on W (with two, it would also follow the second block's
    earlier keys, which reading M1 holds constant)."""
    cfg = tiny(n_ttt=1, T=16, eta=0.0)
    w = weights(cfg)
    toks = tokens(cfg)
    _, grad = Oracle(cfg, w).meta_gradient(toks[0])
    fast = TS.initial_fast(cfg, w, requires_grad=True)
    TS.static_forward(cfg, w, toks[0], fast=fast).mean().backward()
    for j in range(cfg.n_ttt):
        for n in ("W1t", "W2t"):
            np.testing.assert_allclose(grad[j][n], fast[j][n].grad.numpy(), rtol=1e-10, atol=1e-13)


@pytest.mark.parametrize("n_ttt", [1, 2])
def test_complex_step_hessian_vector_product_matches_finite_differences(n_ttt):
    """The Hessian-vector product used by eq. (7), on chunk 3 (window cache non-empty),
    against central differences of the hand-written chunk gradient."""
    cfg = tiny(n_ttt=n_ttt, T=8)
    w = weights(cfg)
    toks = tokens(cfg, n=cfg.T + 1 + cfg.minibatch_b)
    orc = Oracle(cfg, w)
    orc.prefill(toks[:, :cfg.T + 1])
    chunk = toks[0, cfg.T:cfg.T + cfg.minibatch_b + 1]
    rng = np.random.default_rng(5)
    fast = orc.seqs[0].fast
    v = [{n: rng.standard_normal(fast[j][n].shape) for n in ("W1t", "W2t")} for j in range(n_ttt)]
    hv = orc.chunk_hvp(0, chunk, v)
    eps = 1e-5

    def grad_at(scale):
        saved = [{n: W.copy() for n, W in f.items()} for f in fast]
        for j in range(n_ttt):
            for n in ("W1t", "W2t"):
                fast[j][n] = saved[j][n] + scale * v[j][n]
        g = orc.chunk_loss_and_grad(0, chunk)[1]
        for j in range(n_ttt):
            fast[j].update(saved[j])
        return g

    gp, gm = grad_at(eps), grad_at(-eps)
    for j in range(n_ttt):
        for n in ("W1t", "W2t"):
            np.testing.assert_allclose(hv[j][n], (gp[j][n] - gm[j][n]) / (2 * eps), rtol=1e-5, atol=1e-7)


def test_meta_gradient_of_a_single_chunk_is_its_inner_gradient():
    """b = T: one chunk, scored with W_0 and never followed by a loss of W_1, so eq. (7)
    is grad A_1(W_0), the chunk gradient of the inner loop."""
    cfg = tiny(n_ttt=2, T=8, minibatch_b=8, window_k=8)
    w = weights(cfg)
    toks = tokens(cfg)
    L, grad = Oracle(cfg, w).meta_gradient(toks[0])
    mean, g = Oracle(cfg, w).chunk_loss_and_grad(0, toks[0])
    assert L == pytest.approx(mean, rel=1e-14)
    for j in range(cfg.n_ttt):
        for n in ("W1t", "W2t"):
            np.testing.assert_allclose(grad[j][n], g[j][n], rtol=1e-12, atol=1e-15)


def test_reading_m1_differs_from_the_total_derivative_with_two_adaptive_blocks():
    """With two adaptive blocks the second block's cached keys/values depend on W_0
    through the first block, so the total derivative of L (central differences)
    differs from eq. (7) under reading M1, where the cache is a constant as in the
    inner gradient: the reading is a real choice, not a restatement."""
    cfg = tiny(n_ttt=2, T=16)
    w = weights(cfg)
    toks = tokens(cfg)
    _, grad = Oracle(cfg, w).meta_gradient(toks[0])
    v = [{n: np.random.default_rng(3 + j).standard_normal(grad[j][n].shape) for n in grad[j]}
         for j in range(cfg.n_ttt)]
    eps = 1e-5
    fd = (_outer_loss(cfg, _with_initial_fast(cfg, w, v, eps), toks)
          - _outer_loss(cfg, _with_initial_fast(cfg, w, v, -eps), toks)) / (2 * eps)
    dot = sum(float(np.sum(grad[j][n] * v[j][n])) for j in range(cfg.n_ttt) for n in v[j])
    assert abs(dot - fd) > 1e-3 * abs(fd)
