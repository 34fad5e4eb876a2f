"""Kernel-level checks through the per-kernel C ABI (include/ttt_kernels.h) on a GPU.

Each kernel is compared with a float64 PyTorch computation of the same
operation on the same (bf16- or fp32-valued) inputs.
"""
import math

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def T():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import long_context_prefill_ttt_b200 as T
    return T


def _rand(shape, dtype, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float32) * scale).to(dtype).cuda()


def _store(x_log, mn):
    """x_log [batch][rows][K] -> storage [batch][K][rows] when MN-major."""
    return x_log.transpose(1, 2).contiguous() if mn else x_log.contiguous()


# engine 0 picks CTA pairs for large products, the K split over CTA pairs where 128 x 256
# tiles fill at most half the SMs and K is long (test_gemm_k_split_pairs), single-CTA
# tiles otherwise; engine 3 runs single-CTA tiles only, engine 1 SIMT
SHAPES = [(256, 256, 128, 1), (200, 384, 192, 2), (1024, 512, 64, 1), (128, 2048, 256, 1), (384, 128, 1024, 3),
          (1024, 2048, 512, 1), (640, 4096, 128, 1), (100, 256, 64, 2)]


@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 1)])
@pytest.mark.parametrize("M,N,K,batch", SHAPES)
@pytest.mark.parametrize("engine", [0, 1, 3])
def test_gemm_store_f32(T, a_mn, b_mn, M, N, K, batch, engine):
    A = _rand((batch, M, K), torch.bfloat16, 1)
    B = _rand((batch, N, K), torch.bfloat16, 2)
    ref = A.double() @ B.double().transpose(1, 2)
    D = torch.full((batch, M, N), float("nan"), dtype=torch.float32, device="cuda")
    T.ttt_k_gemm(_store(A, a_mn), _store(B, b_mn), D, M, N, K, batch=batch, sA=M * K, a_mn=a_mn, sB=N * K,
                 b_mn=b_mn, sD=M * N, engine=engine)
    T.ttt_k_status()
    err = (D.double() - ref).abs().max().item() / ref.abs().max().item()
    assert err < 2e-6, err


@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1)])
@pytest.mark.parametrize("engine", [0, 1, 3])
def test_gemm_shared_plus_per_batch_operand(T, a_mn, b_mn, engine):
    """acc = A (B_shared + B2[z]): a small per-batch B2 must survive next to a large shared B."""
    M, N, K, batch = 200, 256, 192, 3
    A = _rand((batch, M, K), torch.bfloat16, 21)
    Bs = _rand((1, N, K), torch.bfloat16, 22)
    B2 = _rand((batch, N, K), torch.bfloat16, 23, 1e-3)
    ref = A.double() @ (Bs.double() + B2.double()).transpose(1, 2)
    D = torch.empty((batch, M, N), dtype=torch.float32, device="cuda")
    T.ttt_k_gemm(_store(A, a_mn), _store(Bs, b_mn), D, M, N, K, batch=batch, sA=M * K, a_mn=a_mn, sB=0,
                 b_mn=b_mn, B2=_store(B2, b_mn), sB2=N * K, sD=M * N, engine=engine)
    T.ttt_k_status()
    small = A.double() @ B2.double().transpose(1, 2)
    err = (D.double() - ref).abs().max().item()
    # fp32 accumulation of the large term leaves ~1e-5 absolute; losing B2 would leave |small| ~ 7e-2
    assert err < 1e-2 * small.abs().max().item(), (err, small.abs().max().item())


@pytest.mark.parametrize("M,N,K", [(256, 512, 256), (130, 256, 64)])
def test_gemm_store_bf16_and_fp32_simt(T, M, N, K):
    A = _rand((1, M, K), torch.bfloat16, 3)
    B = _rand((1, N, K), torch.bfloat16, 4)
    ref = A.double() @ B.double().transpose(1, 2)
    D = torch.empty((1, M, N), dtype=torch.bfloat16, device="cuda")
    T.ttt_k_gemm(A, B, D, M, N, K)
    T.ttt_k_status()
    assert torch.allclose(D.double(), ref, rtol=1e-2, atol=1e-2 * ref.abs().max().item())
    # fp32 operands (SIMT engine) against float64
    A32, B32 = A.float(), B.float() + 1e-3
    D32 = torch.empty((1, M, N), dtype=torch.float32, device="cuda")
    T.ttt_k_gemm(A32, B32, D32, M, N, K)
    T.ttt_k_status()
    ref32 = A32.double() @ B32.double().transpose(1, 2)
    assert ((D32.double() - ref32).abs().max() / ref32.abs().max()).item() < 1e-6


@pytest.mark.parametrize("engine", [0, 1, 3])
def test_gemm_epilogues(T, engine):
    M, N, K = 256, 384, 128
    A = _rand((1, M, K), torch.bfloat16, 5, 0.5)
    B = _rand((1, N, K), torch.bfloat16, 6, 0.5)
    acc = (A.double() @ B.double().transpose(1, 2))[0]
    # residual, in place
    R = _rand((M, N), torch.float32, 7)
    D = R.clone()
    T.ttt_k_gemm(A, B, D, M, N, K, X=D, ldx=N, epi=T.EPI_RESID, engine=engine)
    T.ttt_k_status()
    assert (D.double() - (acc + R.double())).abs().max().item() < 1e-4
    # gelu pair
    U = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    G = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    T.ttt_k_gemm(A, B, G, M, N, K, Y=U, ldy=N, epi=T.EPI_GELU, engine=engine)
    T.ttt_k_status()
    gelu = torch.nn.functional.gelu(acc, approximate="none")
    assert torch.allclose(U.double(), acc, rtol=1e-2, atol=1e-2)
    assert torch.allclose(G.double(), gelu, rtol=1e-2, atol=1e-2)
    # gelu' gate
    Xu = _rand((M, N), torch.bfloat16, 8)
    Dg = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    T.ttt_k_gemm(A, B, Dg, M, N, K, X=Xu, ldx=N, epi=T.EPI_DGELU, engine=engine)
    T.ttt_k_status()
    x = Xu.double()
    gp = 0.5 * (1 + torch.erf(x / math.sqrt(2))) + x * torch.exp(-0.5 * x * x) / math.sqrt(2 * math.pi)
    assert torch.allclose(Dg.double(), acc * gp, rtol=2e-2, atol=2e-2)
    # fused SGD: W += alpha * acc, shadow refreshed
    W = _rand((M, N), torch.float32, 9)
    W0 = W.double().clone()
    Sh = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    T.ttt_k_gemm(A, B, W, M, N, K, Y=Sh, ldy=N, alpha=-0.05, epi=T.EPI_SGD, engine=engine)
    T.ttt_k_status()
    assert (W.double() - (W0 - 0.05 * acc)).abs().max().item() < 1e-5
    assert torch.equal(Sh, W.to(torch.bfloat16))


# Thin products that engine 0 runs with K split over a CTA pair (two SMs per 128 x 256
# tile, each finishing half of its columns with the peer's partial): layouts, a
# ragged M tail with batches, and double-K (B + B2: the first CTA takes the B half, the
# second the B2 half), with an odd k-block count per operand.
K_SPLIT_CASES = [(1024, 2048, 8192, 1, 0, 0, False), (1024, 2048, 4096, 1, 0, 1, False),
                 (1024, 2048, 6144, 1, 1, 1, False), (300, 512, 6400, 2, 0, 0, False),
                 (1024, 2048, 3136, 1, 0, 0, True), (256, 768, 4160, 1, 0, 1, True)]


@pytest.mark.parametrize("M,N,K,batch,a_mn,b_mn,b2", K_SPLIT_CASES)
def test_gemm_k_split_pairs(T, M, N, K, batch, a_mn, b_mn, b2):
    A = _rand((batch, M, K), torch.bfloat16, 31, 0.5)
    B = _rand((batch, N, K), torch.bfloat16, 32, 0.5)
    B2 = _rand((batch, N, K), torch.bfloat16, 33, 0.05) if b2 else None
    Bt = B.double() + (B2.double() if b2 else 0)
    acc = A.double() @ Bt.transpose(1, 2)
    kw = dict(batch=batch, sA=M * K, a_mn=a_mn, sB=N * K, b_mn=b_mn, sD=M * N)
    if b2:
        kw.update(B2=_store(B2, b_mn), sB2=N * K)
    As, Bs = _store(A, a_mn), _store(B, b_mn)
    scale = acc.abs().max().item()
    # the tensor cores' fp32 accumulation error grows about linearly with the K steps
    tol = 2e-6 * max(1.0, K * (2 if b2 else 1) / 1024)
    # fp32 store, twice: the fixed order of the two halves makes the result reproducible
    D1 = torch.full((batch, M, N), float("nan"), dtype=torch.float32, device="cuda")
    D2 = torch.full_like(D1, float("nan"))
    T.ttt_k_gemm(As, Bs, D1, M, N, K, **kw)
    T.ttt_k_gemm(As, Bs, D2, M, N, K, **kw)
    T.ttt_k_status()
    assert (D1.double() - acc).abs().max().item() < tol * scale
    assert torch.equal(D1, D2)
    # residual in place
    R = _rand((batch, M, N), torch.float32, 34)
    D = R.clone()
    T.ttt_k_gemm(As, Bs, D, M, N, K, X=D, ldx=N, sX=M * N, epi=T.EPI_RESID, **kw)
    T.ttt_k_status()
    assert (D.double() - (acc + R.double())).abs().max().item() < tol * scale + 1e-5
    # GELU pair (bf16)
    U = torch.empty((batch, M, N), dtype=torch.bfloat16, device="cuda")
    G = torch.empty_like(U)
    T.ttt_k_gemm(As, Bs, G, M, N, K, Y=U, ldy=N, sY=M * N, epi=T.EPI_GELU, **kw)
    T.ttt_k_status()
    assert torch.allclose(U.double(), acc, rtol=1e-2, atol=1e-2 * scale)
    assert torch.allclose(G.double(), torch.nn.functional.gelu(acc), rtol=1e-2, atol=1e-2 * scale)
    # GELU' gate (bf16)
    Xu = _rand((batch, M, N), torch.bfloat16, 35)
    Dg = torch.empty_like(U)
    T.ttt_k_gemm(As, Bs, Dg, M, N, K, X=Xu, ldx=N, sX=M * N, epi=T.EPI_DGELU, **kw)
    T.ttt_k_status()
    x = Xu.double()
    gp = 0.5 * (1 + torch.erf(x / math.sqrt(2))) + x * torch.exp(-0.5 * x * x) / math.sqrt(2 * math.pi)
    assert torch.allclose(Dg.double(), acc * gp, rtol=2e-2, atol=2e-2 * scale)
    # fused SGD on fp32 master weights with the bf16 copy
    W = _rand((batch, M, N), torch.float32, 36)
    W0 = W.double().clone()
    Sh = torch.empty_like(U)
    T.ttt_k_gemm(As, Bs, W, M, N, K, Y=Sh, ldy=N, sY=M * N, alpha=-0.01, epi=T.EPI_SGD, **kw)
    T.ttt_k_status()
    assert (W.double() - (W0 - 0.01 * acc)).abs().max().item() < tol * 0.01 * scale + 1e-6
    assert torch.equal(Sh, W.to(torch.bfloat16))
    # the single-CTA engine agrees to fp32 rounding of the two summation orders
    D3 = torch.empty_like(D1)
    T.ttt_k_gemm(As, Bs, D3, M, N, K, engine=3, **kw)
    T.ttt_k_status()
    assert (D3.double() - D1.double()).abs().max().item() < tol * scale


# Two independent products through ttt_k_gemm_pair: (M, N) of each, shared K, batch,
# layout, epilogue. The first case is the adaptive MLP's two weight-gradient SGD steps at
# the ~1B workload's sizes (d 2048, hidden 8192, 1024-position mini-batch: 1024 tiles, so
# CTAs cross from the first product's tiles into the second's); the others span ragged M
# tails, batches and the forward / data-gradient layouts; the last has N % 256 != 0 and
# takes two separate launches.
PAIR_CASES = [((2048, 8192), (8192, 2048), 1024, 1, 1, 1, "sgd"), ((520, 1024), (1000, 512), 256, 2, 1, 1, "sgd"),
              ((300, 512), (200, 768), 192, 1, 0, 0, "gelu"), ((128, 256), (640, 256), 128, 3, 0, 1, "store"),
              ((256, 384), (256, 256), 128, 1, 0, 0, "store")]


@pytest.mark.parametrize("mn1,mn2,K,batch,a_mn,b_mn,epi", PAIR_CASES)
def test_gemm_pair(T, mn1, mn2, K, batch, a_mn, b_mn, epi):
    cases = []
    for i, (M, N) in enumerate((mn1, mn2)):
        A = _rand((batch, M, K), torch.bfloat16, 41 + 10 * i, 0.5)
        B = _rand((batch, N, K), torch.bfloat16, 42 + 10 * i, 0.5)
        acc = A.double() @ B.double().transpose(1, 2)
        kw = dict(A=_store(A, a_mn), B=_store(B, b_mn), M=M, N=N, K=K, batch=batch, sA=M * K, a_mn=a_mn,
                  sB=N * K, b_mn=b_mn, sD=M * N)
        if epi == "sgd":
            W = _rand((batch, M, N), torch.float32, 43 + 10 * i)
            Y = torch.empty((batch, M, N), dtype=torch.bfloat16, device="cuda")
            kw.update(D=W, Y=Y, ldy=N, sY=M * N, alpha=-0.01, epi=T.EPI_SGD)
            want = W.double() - 0.01 * acc
        elif epi == "gelu":
            U = torch.empty((batch, M, N), dtype=torch.bfloat16, device="cuda")
            kw.update(D=torch.empty_like(U), Y=U, ldy=N, sY=M * N, epi=T.EPI_GELU)
            want = acc
        else:
            kw.update(D=torch.full((batch, M, N), float("nan"), dtype=torch.float32, device="cuda"))
            want = acc
        cases.append((kw, want, acc.abs().max().item()))
    T.ttt_k_gemm_pair(cases[0][0], cases[1][0])
    T.ttt_k_status()
    tol = 2e-6 * max(1.0, K / 1024)
    for kw, want, scale in cases:
        if epi == "sgd":
            assert (kw["D"].double() - want).abs().max().item() < tol * 0.01 * scale + 1e-6
            assert torch.equal(kw["Y"], kw["D"].to(torch.bfloat16))
        elif epi == "gelu":
            assert torch.allclose(kw["Y"].double(), want, rtol=1e-2, atol=1e-2 * scale)
            assert torch.allclose(kw["D"].double(), torch.nn.functional.gelu(want), rtol=1e-2, atol=1e-2 * scale)
        else:
            assert (kw["D"].double() - want).abs().max().item() < tol * scale


def _attn_reference(qkv, ring_k, ring_v, B, H, hd, n, q0, window, C):
    """float64 keys/values at absolute positions, explicit window mask."""
    d = H * hd
    q = qkv[..., :d].double().view(B, n, H, hd)
    kc = qkv[..., d:2 * d].double().view(B, n, H, hd)
    vc = qkv[..., 2 * d:].double().view(B, n, H, hd)
    lo = max(0, q0 - window + 1)
    pos = torch.arange(lo, q0 + n)
    rk = ring_k.double().view(B, C, H, hd)
    rv = ring_v.double().view(B, C, H, hd)
    cached = torch.arange(lo, q0)
    K = torch.cat([rk[:, (cached % C).cuda()], kc], 1)  # position p < q0 sits in ring slot p % C
    V = torch.cat([rv[:, (cached % C).cuda()], vc], 1)
    qp = torch.arange(q0, q0 + n)[:, None]
    mask = (pos[None, :] <= qp) & (pos[None, :] >= qp - window + 1)
    return q, kc, vc, K, V, mask.cuda(), lo


ATTN_CASES = [
    # SIMT engine (q0 not 64-aligned, head dim 16, single query)
    (2, 2, 64, 96, 160, 128, 256), (1, 4, 16, 48, 0, 16, 32), (1, 2, 128, 64, 300, 200, 384),
    (3, 1, 64, 1, 777, 64, 128),
    # tensor-core engine for bf16 (q0 % 64 == 0): ragged rows, windows off the tile grid, window < tile
    (2, 2, 64, 96, 128, 128, 256), (1, 2, 128, 200, 256, 300, 640), (2, 3, 128, 64, 0, 64, 128),
    (1, 2, 64, 130, 64, 40, 128), (1, 1, 128, 256, 1024, 1024, 2048),
    # tcgen05 forward (q0 % 128 == 0, C % 128 == 0): many ring tiles, partial last query tile
    (2, 2, 128, 384, 512, 700, 1280), (1, 4, 64, 300, 1024, 1000, 2048),
    # tcgen05 dK/dV: window shorter than the rows (key blocks that some query blocks no
    # longer see), ragged last key block with the next sequence's rows behind it, no ring
    # (q0 = 0), window shorter than one query block
    (2, 2, 128, 520, 256, 200, 768), (1, 3, 64, 330, 0, 150, 384), (2, 2, 128, 256, 128, 40, 256),
    # enough (sequence, head) pairs that the forward gives each CTA two query tiles sharing
    # K/V: ragged rows with a short window, the second tile's keys one tile further on
    # (window a multiple of 128), and no ring with a window longer than the rows
    (2, 40, 64, 520, 256, 300, 768), (1, 80, 128, 384, 1024, 512, 1536), (1, 150, 64, 300, 0, 4096, 4224),
    # the ring has wrapped (q0 > C): the window's cached keys cross slot C-1 -> 0, with the
    # window's first key inside a ring tile, at head dims 128 and 64, ragged rows, and the
    # ~1B workload's geometry (k = 8192, b = 1024, C = 9216) one chunk after the first wrap
    (1, 2, 128, 256, 3072, 1000, 1280), (2, 4, 64, 300, 5120, 1500, 1664), (1, 3, 128, 200, 2816, 768, 896),
    (1, 2, 128, 1024, 10240, 8192, 9216),
]


@pytest.mark.parametrize("engine", [0, 1, 2])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("B,H,hd,n,q0,window,C", ATTN_CASES)
def test_attention_forward_and_backward(T, engine, dtype, B, H, hd, n, q0, window, C):
    d = H * hd
    qkv = _rand((B * n, 3 * d), dtype, 11)
    ring_k = _rand((B, C, d), dtype, 12)
    ring_v = _rand((B, C, d), dtype, 13)
    out = torch.empty((B * n, d), dtype=dtype, device="cuda")
    lse = torch.empty((B, H, n), dtype=torch.float32, device="cuda")
    T.ttt_k_attention_fwd(qkv, out, lse, B, H, hd, n, q0, window, ring_k, ring_v, C, engine=engine)
    T.ttt_k_status()
    q, kc, vc, K, V, mask, lo = _attn_reference(qkv, ring_k, ring_v, B, H, hd, n, q0, window, C)
    q.requires_grad_(True); kc.requires_grad_(True); vc.requires_grad_(True)
    # rebuild keys so autograd sees the current part
    ncached = q0 - lo
    Kf = torch.cat([K[:, :ncached], kc], 1)
    Vf = torch.cat([V[:, :ncached], vc], 1)
    s = torch.einsum("bqhd,bkhd->bhqk", q, Kf) / math.sqrt(hd)
    s = s.masked_fill(~mask, float("-inf"))
    ref_lse = torch.logsumexp(s, -1)
    o = torch.einsum("bhqk,bkhd->bqhd", torch.softmax(s, -1), Vf)
    tol = 1e-5 if dtype == torch.float32 else 2e-2
    assert (out.double().view(B, n, H, hd) - o).abs().max().item() < tol
    assert (lse.double() - ref_lse).abs().max().item() < tol
    dout = _rand((B * n, d), dtype, 14)
    o.backward(dout.double().view(B, n, H, hd))
    dqkv = torch.zeros((B * n, 3 * d), dtype=dtype, device="cuda")
    dsum = torch.empty((B, H, n), dtype=torch.float32, device="cuda")
    T.ttt_k_attention_bwd(qkv, out, lse, dout, dqkv, dsum, B, H, hd, n, q0, window, ring_k, ring_v, C,
                          engine=engine)
    T.ttt_k_status()
    for got, ref in ((dqkv[:, :d], q.grad), (dqkv[:, d:2 * d], kc.grad), (dqkv[:, 2 * d:], vc.grad)):
        scale = ref.abs().max().item() + 1e-12
        err = (got.double().view(B, n, H, hd) - ref).abs().max().item() / scale
        assert err < (1e-5 if dtype == torch.float32 else 3e-2), err


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("M,N,K,batch", [(1, 768, 768, 8), (8, 2304, 768, 1), (16, 384, 3072, 2), (8, 32000, 768, 1),
                                         (3, 1000, 3072, 2), (8, 776, 6144, 1), (4, 3072, 1024, 1)])
def test_skinny_gemm_rows_per_sequence(T, dtype, M, N, K, batch):
    """Decode-sized products (<= 16 rows per slice): shared W plus per-slice dW, residual and GELU epilogues.
    bf16 with <= 8 rows runs the few-row kernel with 8, 16 or 32 columns per CTA (all three occur
    here): N off its column grid, and A filling its 96 KB staging buffer (8 x 6144), are among
    the cases."""
    A = _rand((batch, M, K), dtype, 31)
    Bs = _rand((1, N, K), dtype, 32, 0.05)
    B2 = _rand((batch, N, K), dtype, 33, 1e-3)
    ref = A.double() @ (Bs.double() + B2.double()).transpose(1, 2)
    tol = 1e-5 if dtype == torch.float32 else 1e-2
    R = _rand((batch, M, N), torch.float32, 34)
    D = R.clone()
    T.ttt_k_gemm(A, Bs, D, M, N, K, batch=batch, sA=M * K, sB=0, B2=B2, sB2=N * K, sD=M * N, X=D, ldx=N, sX=M * N,
                 epi=T.EPI_RESID)
    T.ttt_k_status()
    assert (D.double() - (ref + R.double())).abs().max().item() <= tol * ref.abs().max().item()
    G = torch.empty((batch, M, N), dtype=dtype, device="cuda")
    U = torch.empty((batch, M, N), dtype=dtype, device="cuda")
    T.ttt_k_gemm(A, Bs, G, M, N, K, batch=batch, sA=M * K, sB=0, B2=B2, sB2=N * K, sD=M * N, Y=U, ldy=N, sY=M * N,
                 epi=T.EPI_GELU)
    T.ttt_k_status()
    assert torch.allclose(U.double(), ref, rtol=2 * tol, atol=2 * tol * ref.abs().max().item())
    assert torch.allclose(G.double(), torch.nn.functional.gelu(ref, approximate="none"), rtol=2 * tol,
                          atol=2 * tol * ref.abs().max().item())


@pytest.mark.parametrize("M,V,d", [(1024, 32000, 2048), (200, 8192, 512), (77, 256, 128)])
def test_fused_lm_head_cross_entropy(T, M, V, d):
    """LM head + softmax cross-entropy chunked over the vocabulary, against float64:
    loss = logsumexp(z) - z[target] from the fp32 accumulators, dz = (softmax - onehot) * s."""
    # the model's scales: normalised rows, embedding ~ N(0, 0.02) (logits of a few units;
    # dz is formed from bf16 logits, whose rounding grows with their magnitude)
    r = _rand((M, d), torch.bfloat16, 41)
    E = _rand((V, d), torch.bfloat16, 42, 0.02)
    g = torch.Generator().manual_seed(43)
    tgt = torch.randint(0, V, (M,), generator=g, dtype=torch.int32)
    tgt[0], tgt[-1] = 0, V - 1  # first and last vocabulary chunks
    tgt = tgt.cuda()
    zref = r.double() @ E.double().t()
    lref = torch.logsumexp(zref, 1) - zref[torch.arange(M), tgt.long()]
    z = torch.empty((M, V), dtype=torch.bfloat16, device="cuda")
    loss = torch.empty(M, dtype=torch.float32, device="cuda")
    scratch = torch.empty(2 * M * (V // 64) + M, dtype=torch.float32, device="cuda")
    T.ttt_k_lm_head_ce(r, E, tgt, z, loss, scratch, M, V, d)
    T.ttt_k_status()
    assert (loss.double() - lref).abs().max().item() <= 1e-4 * lref.abs().max().item() + 1e-4
    assert (z.double() - zref).abs().max().item() <= 1e-2 * zref.abs().max().item()
    s = 1.0 / 256
    T.ttt_k_lm_head_ce(r, E, tgt, z, loss, scratch, M, V, d, grad_scale=s)
    T.ttt_k_status()
    pref = torch.softmax(zref, 1)
    pref[torch.arange(M), tgt.long()] -= 1.0
    dref = pref * s
    assert (z.double() - dref).abs().max().item() <= 2e-2 * dref.abs().max().item()
    assert (z.double().sum(1)).abs().max().item() <= 1e-2 * s  # softmax rows sum to one
    # an id outside the vocabulary is reported, not read
    bad = tgt.clone()
    bad[3] = V + 5
    T.ttt_k_lm_head_ce(r, E, bad, z, loss, scratch, M, V, d)
    with pytest.raises(T.TTTError) as e:
        T.ttt_k_status()
    assert e.value.code == T.TTT_ERR_INVALID_ARG
