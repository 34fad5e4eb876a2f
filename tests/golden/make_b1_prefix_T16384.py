"""Write b1_128k_bf16_T16384.npz: the CPU oracle's results for the ~1B workload
(V32000 d2048 L24, last 6 blocks adaptive, H16, k8192, b1024) on its first 16384
positions, one sequence.

16384 positions are 16 mini-batches, past the fill of the 8192-key window: the
chunks from 9 on see a full window, and on the GPU (run in 4 frozen-phase segments
of 4096 positions) the window ring of 9216 slots wraps. The oracle needs minutes
here, too long for a test, so its results are stored:
  losses        [16384]   per-position loss l_t (float64)
  r1 [d], r2 [h_t]        fixed random probe vectors
  w1r [6][h_t], w2r [6][d]  W1t @ r1 and W2t @ r2 of every adaptive block after the
                          last update (a sketch of each fast-weight matrix: for a
                          Gaussian probe, |A r| estimates the Frobenius norm of A)
  w1r0, w2r0              the same sketches of W_init
The inputs are the seeded generators of `synthetic` for that workload. This script
calls only `oracle` and `synthetic`; nothing from the CUDA library.

    python tests/golden/make_b1_prefix_T16384.py
"""
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import synthetic as syn  # noqa: E402
from oracle import Oracle  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "b1_128k_bf16_T16384.npz")


def main():
    cfg = syn.config("b1_128k_bf16", T=16384)
    w = syn.make_weights(cfg)
    toks = syn.make_token_batch(cfg)
    t0 = time.time()
    orc = Oracle(cfg, w)
    losses = orc.prefill(toks)[0]
    rng = np.random.default_rng(20260)
    r1 = rng.standard_normal(cfg.d)
    r2 = rng.standard_normal(cfg.ttt_hidden)
    w1r, w2r, w1r0, w2r0 = [], [], [], []
    for j in range(cfg.n_ttt):
        W1, W2 = orc.fast_weights(0, j)
        l = cfg.first_ttt + j
        w1r.append(W1 @ r1)
        w2r.append(W2 @ r2)
        w1r0.append(w[f"layers.{l}.W1t"].astype(np.float64) @ r1)
        w2r0.append(w[f"layers.{l}.W2t"].astype(np.float64) @ r2)
    np.savez_compressed(OUT, losses=losses, r1=r1, r2=r2, w1r=np.array(w1r), w2r=np.array(w2r),
                        w1r0=np.array(w1r0), w2r0=np.array(w2r0), T=cfg.T, workload=cfg.name)
    print(f"wrote {OUT} in {time.time() - t0:.0f} s; mean loss {losses.mean():.4f}")


if __name__ == "__main__":
    main()
