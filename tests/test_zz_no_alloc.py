"""The allocation-free attention backward matches the allocating one.

ttt_k_attention_bwd_noalloc serves callers that may not allocate device memory:
its scratch is a fixed array inside the library instead of a caller buffer. This
test calls it through the C ABI twice in a row (the second time on new inputs,
so the shared scratch is reused) and compares each result with
ttt_k_attention_bwd on the same inputs. It lives in its own file, collected
last, and passes both alone in a fresh process and after the other tests.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def T():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import long_context_prefill_ttt_b200 as T
    return T


def _inputs(dtype, seed, B, H, hd, n, C):
    g = torch.Generator().manual_seed(seed)
    d = H * hd
    r = lambda *s: torch.randn(*s, generator=g).to(dtype).cuda()
    return r(B * n, 3 * d), r(B, C, d), r(B, C, d), r(B * n, d)


@pytest.mark.parametrize("dtype,tol", [(torch.float32, 1e-5), (torch.bfloat16, 3e-2)])
@pytest.mark.parametrize("B,H,hd,n,q0,window,C", [(2, 2, 64, 96, 128, 128, 256), (1, 2, 128, 200, 300, 200, 384)])
def test_noalloc_backward_matches_allocating_backward_twice(T, dtype, tol, B, H, hd, n, q0, window, C):
    d = H * hd
    for call, seed in enumerate((101, 202)):
        qkv, ring_k, ring_v, dout = _inputs(dtype, seed, B, H, hd, n, C)
        out = torch.empty((B * n, d), dtype=dtype, device="cuda")
        lse = torch.empty((B, H, n), dtype=torch.float32, device="cuda")
        T.ttt_k_attention_fwd(qkv, out, lse, B, H, hd, n, q0, window, ring_k, ring_v, C)
        ref = torch.zeros((B * n, 3 * d), dtype=dtype, device="cuda")
        dsum = torch.empty((B, H, n), dtype=torch.float32, device="cuda")
        T.ttt_k_attention_bwd(qkv, out, lse, dout, ref, dsum, B, H, hd, n, q0, window, ring_k, ring_v, C)
        got = torch.zeros_like(ref)
        T.ttt_k_attention_bwd_noalloc(qkv, out, lse, dout, got, B, H, hd, n, q0, window, ring_k, ring_v, C)
        torch.cuda.synchronize()
        scale = ref.float().abs().max().item()
        err = (got.float() - ref.float()).abs().max().item() / scale
        assert err <= tol, (call, err)


def test_noalloc_rejects_sizes_beyond_its_scratch(T):
    qkv, ring_k, ring_v, dout = _inputs(torch.bfloat16, 7, 1, 1, 64, 8, 128)
    out = torch.empty((8, 64), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, 1, 8), dtype=torch.float32, device="cuda")
    dq = torch.empty((8, 192), dtype=torch.bfloat16, device="cuda")
    # B*H*n = 1 * 16 * 65537 > 1048576 rows of scratch: the library rejects the call before any
    # launch (called directly: the binding would already refuse the buffers as too small)
    rc = T.lib.ttt_k_attention_bwd_noalloc(T.TTT_BF16, 1, 16, 64, 65537, 0, 64, qkv.data_ptr(), None, None, 0,
                                           out.data_ptr(), lse.data_ptr(), dout.data_ptr(), dq.data_ptr(), 0, None)
    assert rc == T.TTT_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        T.ttt_k_attention_bwd_noalloc(qkv, out, lse, dout, dq, 1, 16, 64, 65537, 0, 64)
