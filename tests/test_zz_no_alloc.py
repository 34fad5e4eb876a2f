"""The allocation-free attention backward matches the allocating one.

ttt_k_attention_bwd_noalloc serves callers that may not allocate device memory:
its scratch is a fixed array inside the library instead of a caller buffer. This
test calls it through the C ABI twice in a row (the second time on new inputs,
so the shared scratch is reused), checks the device status after each call, and
compares each result with ttt_k_attention_bwd on the same inputs. A second test
makes it the very first call into the library in a fresh process, with every
device allocation of the library set to fail. It lives in its own file,
collected last, and passes both alone in a fresh process and after the other
tests.
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


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
@pytest.mark.parametrize("B,H,hd,n,q0,window,C", [(2, 2, 64, 96, 128, 128, 256), (1, 2, 128, 200, 300, 200, 384),
                                                  (1, 2, 128, 256, 1024, 512, 640)])
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
        T.ttt_k_status()
        got = torch.zeros_like(ref)
        T.ttt_k_attention_bwd_noalloc(qkv, out, lse, dout, got, B, H, hd, n, q0, window, ring_k, ring_v, C)
        T.ttt_k_status()  # raises unless the call's kernels finished without an expired wait
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


_FIRST_CALL = r"""
import sys, torch
sys.path.insert(0, sys.argv[1])
B, H, hd, n, q0, window, C = 1, 4, 128, 256, 1024, 512, 640
d = H * hd
g = torch.Generator().manual_seed(5)
r = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16).cuda()
qkv, ring_k, ring_v, dout = r(B * n, 3 * d), r(B, C, d), r(B, C, d), r(B * n, d)
out = r(B * n, d)
lse = torch.randn(B, H, n, generator=g).cuda() + 6.0
got = torch.zeros(B * n, 3 * d, dtype=torch.bfloat16, device="cuda")
torch.cuda.synchronize()
import long_context_prefill_ttt_b200 as T
T.ttt_test_fail_allocation(0)          # every device allocation of the library would now fail
T.ttt_k_attention_bwd_noalloc(qkv, out, lse, dout, got, B, H, hd, n, q0, window, ring_k, ring_v, C)
T.ttt_k_status()
T.ttt_test_fail_allocation(-1)
assert T.ttt_test_allocation_count() == 0, T.ttt_test_allocation_count()
ref = torch.zeros_like(got)
dsum = torch.empty(B, H, n, device="cuda")
T.ttt_k_attention_bwd(qkv, out, lse, dout, ref, dsum, B, H, hd, n, q0, window, ring_k, ring_v, C)
T.ttt_k_status()
err = (got.float() - ref.float()).abs().max().item() / ref.float().abs().max().item()
assert err <= 3e-2, err
print("first-call ok", err)
"""


def test_noalloc_as_the_first_library_call_of_a_fresh_process(T):
    """A caller that cannot allocate may call this entry point before anything else:
    no earlier call has set anything up for it, and no allocation may happen."""
    r = subprocess.run([sys.executable, "-c", _FIRST_CALL, ROOT], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "first-call ok" in r.stdout
