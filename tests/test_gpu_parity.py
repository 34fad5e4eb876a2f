"""End-to-end parity of the CUDA path (through the C ABI) with the CPU oracle.

Workloads: the tiny fp32 model in full, the small bf16 model in full, the
~125M and ~1B models on prefixes the oracle finishes in about a minute, and
greedy decode on the ~125M architecture; plus the special cases the pages fix
(eta = 0 is the static model, b = T is one update, only the adaptive MLPs
change, sequences are independent, a prefill split at a chunk boundary equals
one call, teacher-forced decode equals prefill). Tolerances: see tests/parity.py.
"""
import numpy as np
import pytest
import torch

import synthetic as syn
from oracle import Oracle
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def T():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import long_context_prefill_ttt_b200 as T
    return T


# ----------------------------------------------------------------------------- fp32 (1e-4)

@pytest.mark.parametrize("overrides,seg", [
    ({}, 0),                                              # tiny fp32 workload as specified (T=256)
    ({}, 64),                                             # frozen phase in 4 segments (window cache across them)
    (dict(n_ttt=2), 0),                                   # attention backward inside the adaptive blocks
    (dict(n_ttt=2, batch=3, window_k=40, T=200), 48),     # batch, window > b, ragged tail chunk pending
    (dict(n_ttt=4, T=96, minibatch_b=32, window_k=32), 0),  # every block adaptive
    (dict(n_ttt=0), 0),                                   # no adaptive block: the plain SWA model
    (dict(n_ttt=0, window_k=512), 64),                    # ... with full causal attention (k >= T), 4 segments
])
def test_tiny_fp32_matches_oracle(T, overrides, seg):
    cfg = syn.config("tiny_fp32", **overrides)
    r = P.prefill_both(T, cfg, max_segment=seg)
    P.compare(cfg, r["w"], r["gpu_losses"], r["orc_losses"], r["gpu_w"], r["orc_w"])


def test_tiny_fp32_eta_zero_is_static_model_and_weights_untouched(T):
    cfg = syn.config("tiny_fp32", eta=0.0, n_ttt=2)
    r = P.prefill_both(T, cfg)
    P.compare(cfg, r["w"], r["gpu_losses"], r["orc_losses"], r["gpu_w"], r["orc_w"])
    init = P.init_fast_weights(r["w"], cfg)
    for j in range(cfg.n_ttt):
        assert np.array_equal(r["gpu_w"][0][j][0], init[j][0].astype(np.float32))
        assert np.array_equal(r["gpu_w"][0][j][1], init[j][1].astype(np.float32))


def test_tiny_fp32_b_equals_T_is_one_update(T):
    cfg = syn.config("tiny_fp32", T=64, minibatch_b=64, window_k=64, n_ttt=2)
    r = P.prefill_both(T, cfg)
    P.compare(cfg, r["w"], r["gpu_losses"], r["orc_losses"], r["gpu_w"], r["orc_w"])
    static = Oracle(cfg.replace(eta=0.0), r["w"]).prefill(r["toks"])
    assert P.max_rel(r["gpu_losses"][0], static[0]) <= 1e-4


def test_prefill_split_at_chunk_boundary_equals_one_call(T):
    cfg = syn.config("tiny_fp32", n_ttt=2, T=160)
    w = syn.make_weights(cfg)
    toks = syn.make_token_batch(cfg)
    h1 = T.ttt_create(cfg, w)
    l1 = T.ttt_prefill(h1, toks)
    h2 = T.ttt_create(cfg, w)
    a = T.ttt_prefill(h2, np.ascontiguousarray(toks[:, :65]))
    b = T.ttt_prefill(h2, np.ascontiguousarray(toks[:, 64:]))
    assert P.max_rel(np.concatenate([a, b], 1), l1) <= 1e-5
    with pytest.raises(T.TTTError):  # continuity: first id must be the pending token
        bad = toks[:, 64:].copy()
        bad[0, 0] = (bad[0, 0] + 1) % cfg.vocab
        h3 = T.ttt_create(cfg, w)
        T.ttt_prefill(h3, np.ascontiguousarray(toks[:, :65]))
        T.ttt_prefill(h3, np.ascontiguousarray(bad))


def test_sequences_are_independent(T):
    cfg = syn.config("tiny_fp32", n_ttt=2, batch=3, T=96)
    w = syn.make_weights(cfg)
    toks = syn.make_token_batch(cfg)
    together = T.ttt_prefill(T.ttt_create(cfg, w), toks)
    one = cfg.replace(batch=1)
    for s in range(3):
        alone = T.ttt_prefill(T.ttt_create(one, w), np.ascontiguousarray(toks[s:s + 1]))
        assert P.max_rel(together[s], alone[0]) <= 1e-6


@pytest.mark.parametrize("n_ttt", [2, 0])
def test_decode_fp32_greedy_and_teacher_forced(T, n_ttt):
    cfg = syn.config("tiny_fp32", n_ttt=n_ttt, T=40)
    w = syn.make_weights(cfg)
    toks = syn.make_token_batch(cfg)
    h = T.ttt_create(cfg, w)
    T.ttt_prefill(h, toks)
    gtok, gloss = T.ttt_decode(h, 30)          # 40 + 30 = 70 positions: chunks at 48 and 64 complete
    orc = Oracle(cfg, w)
    orc.prefill(toks)
    r = orc.decode(30)
    assert np.array_equal(gtok, r["tokens"])
    assert P.max_rel(gloss, r["losses"]) <= 1e-4
    for j in range(cfg.n_ttt):
        assert P.max_rel(T.ttt_get_weights(h, 0, j)[0], orc.fast_weights(0, j)[0]) <= 1e-4
    # teacher-forced decode equals one prefill over the same stream
    full = np.concatenate([toks, gtok.astype(np.int32)], axis=1)
    hp = T.ttt_create(cfg.replace(T=70), w)
    lp = T.ttt_prefill(hp, np.ascontiguousarray(full))
    hf = T.ttt_create(cfg, w)
    l0 = T.ttt_prefill(hf, toks)
    _, lf = T.ttt_decode(hf, 30, forced=gtok)
    assert P.max_rel(np.concatenate([l0, lf], 1), lp) <= 1e-5


def test_reset_restores_initial_state(T):
    cfg = syn.config("tiny_fp32", T=64)
    w = syn.make_weights(cfg)
    toks = syn.make_token_batch(cfg)
    h = T.ttt_create(cfg, w)
    a = T.ttt_prefill(h, toks)
    T.ttt_reset(h)
    assert T.ttt_position(h) == 0
    b = T.ttt_prefill(h, toks)
    assert np.array_equal(a, b)


def test_bad_token_is_rejected(T):
    cfg = syn.config("tiny_fp32", T=32)
    w = syn.make_weights(cfg)
    toks = syn.make_token_batch(cfg)
    toks[0, 5] = cfg.vocab + 3
    h = T.ttt_create(cfg, w)
    with pytest.raises(T.TTTError) as e:
        T.ttt_prefill(h, toks)
    assert e.value.code == T.TTT_ERR_INVALID_ARG


# ----------------------------------------------------------------------------- bf16 (2e-2 loss, 5e-3 weights)

def test_small_bf16_matches_oracle(T):
    cfg = syn.config("small_bf16")
    r = P.prefill_both(T, cfg)
    rep = {}
    P.compare(cfg, r["w"], r["gpu_losses"], r["orc_losses"], r["gpu_w"], r["orc_w"], report=rep)
    print("small_bf16", rep)
    assert rep["dw"] <= 5e-2


def test_small_bf16_full_attention_without_adaptive_blocks_matches_oracle(T):
    """The comparator model of the speed claim: no adaptive block, window >= T."""
    cfg = syn.config("small_bf16", n_ttt=0, T=2048, window_k=4096)
    r = P.prefill_both(T, cfg)
    P.compare(cfg, r["w"], r["gpu_losses"], r["orc_losses"], r["gpu_w"], r["orc_w"])


def test_bf16_update_effect_matches_oracle(T):
    """The update moves the next chunks' losses; in bf16 that move must match the
    oracle's (a bf16 copy of W_init + dW would round a small dW away)."""
    cfg = syn.config("small_bf16", T=1024)
    r = P.prefill_both(T, cfg)
    static = Oracle(cfg.replace(eta=0.0), r["w"]).prefill(r["toks"])[0]
    b = cfg.minibatch_b
    want = float(np.mean(r["orc_losses"][0][b:] - static[b:]))
    got = float(np.mean(r["gpu_losses"][0][b:] - static[b:]))
    assert abs(want) > 1e-3
    assert abs(got - want) <= 0.1 * abs(want), (got, want)


def test_small_bf16_device_buffers_match_host_buffers(T):
    cfg = syn.config("small_bf16", T=1024)
    w = syn.make_weights(cfg)
    toks = syn.make_token_batch(cfg)
    lh = T.ttt_prefill(T.ttt_create(cfg, w), toks)
    wd = {k: torch.from_numpy(v).cuda() for k, v in w.items()}
    hd = T.ttt_create(cfg, wd)
    ld = T.ttt_prefill(hd, torch.from_numpy(toks).cuda())
    assert np.array_equal(lh, ld.cpu().numpy())


def test_hd128_ring_wrap_and_segments_bf16_matches_oracle(T):
    """The ~1B workload's head geometry (head dim 128) at a width the oracle runs in
    seconds, long enough that the paths of the 128K run are all taken: the frozen
    phase runs in 4 segments, each reading the previous segment's keys from the ring;
    the window fills; the ring (C = 768 positions) wraps five times."""
    cfg = syn.config("b1_128k_bf16", vocab=8192, d=512, n_layers=8, n_heads=4, n_ttt=2, mlp_hidden=2048,
                     ttt_hidden=1024, static_hidden=1024, window_k=512, minibatch_b=256, T=4096)
    r = P.prefill_both(T, cfg, max_segment=1024)
    rep = {}
    P.compare(cfg, r["w"], r["gpu_losses"], r["orc_losses"], r["gpu_w"], r["orc_w"], report=rep)
    print("hd128 ring wrap", rep)
    assert rep["dw"] <= 5e-2


def test_batched_bf16_window_shorter_than_sequence_matches_oracle(T):
    """Four sequences with their own fast weights (the per-sequence W_init + dW GEMM
    operands) and a window shorter than the sequence: the batched path of the
    fixed-128K-tokens sweep."""
    cfg = syn.config("small_bf16", batch=4, T=2048)
    r = P.prefill_both(T, cfg)
    rep = {}
    P.compare(cfg, r["w"], r["gpu_losses"], r["orc_losses"], r["gpu_w"], r["orc_w"], report=rep)
    print("small_bf16 B=4", rep)
    assert rep["dw"] <= 5e-2


def test_m125_bf16_prefix_matches_oracle(T):
    cfg = syn.config("m125_bf16", T=2048, batch=2)
    r = P.prefill_both(T, cfg)
    rep = {}
    P.compare(cfg, r["w"], r["gpu_losses"], r["orc_losses"], r["gpu_w"], r["orc_w"], report=rep)
    print("m125_bf16 prefix", rep)
    assert rep["dw"] <= 5e-2


@pytest.mark.slow
def test_b1_128k_bf16_prefix_matches_oracle(T):
    cfg = syn.config("b1_128k_bf16", T=2048)
    r = P.prefill_both(T, cfg)
    rep = {}
    P.compare(cfg, r["w"], r["gpu_losses"], r["orc_losses"], r["gpu_w"], r["orc_w"], report=rep)
    print("b1_128k_bf16 prefix", rep)
    assert rep["dw"] <= 5e-2


def test_m125_decode_bf16_greedy_matches_oracle(T):
    """Greedy decode under bf16: ties and near-ties may flip, so the oracle is
    teacher-forced on the GPU's tokens; each GPU token must be within delta of
    the oracle's best logit, then losses and weights are compared."""
    cfg = syn.config("m125_decode_bf16", T=1024, batch=2)
    w = syn.make_weights(cfg)
    toks = syn.make_token_batch(cfg)
    h = T.ttt_create(cfg, w)
    T.ttt_prefill(h, toks)
    n = 1100  # completes the chunk [1024, 2048): one update from decoded tokens
    gtok, gloss = T.ttt_decode(h, n)
    orc = Oracle(cfg, w)
    orc.prefill(toks)
    r = orc.decode(n, forced=gtok)
    delta = 2e-2 * np.maximum(1.0, np.abs(r["z_max"]))
    assert np.all(r["z_chosen"] >= r["z_max"] - delta)
    assert float(np.max(np.abs(gloss - r["losses"]) / np.abs(r["losses"]))) <= 2e-2
    for s in range(cfg.batch):
        for j in range(cfg.n_ttt):
            g1, g2 = T.ttt_get_weights(h, s, j)
            o1, o2 = orc.fast_weights(s, j)
            assert P.rel_fro(g1, o1) <= 5e-3 and P.rel_fro(g2, o2) <= 5e-3


@pytest.mark.slow
def test_b1_128k_bf16_past_window_fill_matches_stored_oracle(T):
    """The ~1B workload on 16384 positions (16 chunks; chunks 9-16 see a full 8192-key
    window), run as the 128K benchmark runs it but in 4 frozen segments of 4096 so
    that every segment reads its predecessor's keys from the ring, whose 9216 slots
    wrap. The oracle's results come from tests/golden/make_b1_prefix_T16384.py."""
    import os
    g = np.load(os.path.join(os.path.dirname(__file__), "golden", "b1_128k_bf16_T16384.npz"))
    cfg = syn.config("b1_128k_bf16", T=int(g["T"]))
    w = syn.make_weights(cfg)
    toks = syn.make_token_batch(cfg)
    h = T.ttt_create(cfg, w, max_segment=4096)
    gl = T.ttt_prefill(h, np.ascontiguousarray(toks, dtype=np.int32))[0]
    ol = g["losses"]
    assert np.all(np.isfinite(gl))
    assert float(np.max(np.abs(gl - ol) / np.abs(ol))) <= 2e-2
    for j in range(cfg.n_ttt):
        w1, w2 = T.ttt_get_weights(h, 0, j)
        for W, r, ref, ref0 in ((w1, g["r1"], g["w1r"][j], g["w1r0"][j]), (w2, g["r2"], g["w2r"][j], g["w2r0"][j])):
            got = W.astype(np.float64) @ r
            assert P.rel_fro(got, ref) <= 5e-3
            assert P.rel_fro(got - ref0, ref - ref0) <= 5e-2
