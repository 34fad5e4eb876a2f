"""CPU-only checks of the C ABI: the library loads and exports every symbol that
include/*.h declares, and argument validation happens before any device call."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import synthetic as syn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if not f.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", f)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b(ttt_\w+)\s*\(", src, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


def test_headers_declare_the_boundary():
    names = declared_functions()
    for n in ("ttt_create", "ttt_prefill", "ttt_decode", "ttt_get_weights", "ttt_reset", "ttt_destroy",
              "ttt_last_error", "ttt_k_gemm", "ttt_k_gemm_pair", "ttt_k_attention_fwd", "ttt_k_attention_bwd"):
        assert n in names


def test_library_exports_every_declared_symbol():
    import long_context_prefill_ttt_b200 as T
    lib = ctypes.CDLL(T.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert "sm_100a" in T.ttt_version()


def test_weight_tensor_count_and_order_match_the_generator():
    import long_context_prefill_ttt_b200 as T
    for name, loss in (("tiny_fp32", "e2e"), ("small_bf16", "e2e"), ("b1_128k_bf16", "e2e"),
                       ("tiny_fp32", "kvb"), ("small_bf16", "kvb")):
        cfg = syn.config(name, inner_loss=loss)
        c = T.make_config(cfg)
        assert c.inner_loss == (T.TTT_LOSS_KVB if loss == "kvb" else T.TTT_LOSS_E2E)
        assert T.lib.ttt_num_weight_tensors(ctypes.byref(c)) == len(syn.weight_shapes(cfg))
        assert T.weight_names(cfg) == [n for n, _ in syn.weight_shapes(cfg)]


@pytest.mark.parametrize("field,value", [("window_k", 8), ("n_ttt", -1), ("n_ttt", 9), ("d", 63),
                                         ("minibatch_b", 0), ("vocab", 0), ("n_heads", 5)])
def test_create_rejects_invalid_configs_without_touching_the_device(field, value):
    import long_context_prefill_ttt_b200 as T
    cfg = syn.config("tiny_fp32").replace(**{field: value})
    if field == "window_k":
        cfg = cfg.replace(minibatch_b=16)
    c = T.make_config(cfg)
    out = ctypes.c_void_p()
    w = T.ttt_weights()
    rc = T.lib.ttt_create(ctypes.byref(c), ctypes.byref(w), ctypes.byref(out))
    assert rc == T.TTT_ERR_INVALID_ARG
    assert not out.value


def test_create_rejects_an_unknown_inner_loss():
    import long_context_prefill_ttt_b200 as T
    c = T.make_config(syn.config("tiny_fp32"))
    c.inner_loss = 2
    with pytest.raises(ValueError):
        T.make_config(syn.config("tiny_fp32", inner_loss="KVB"))
    out = ctypes.c_void_p()
    w = T.ttt_weights()
    assert T.lib.ttt_create(ctypes.byref(c), ctypes.byref(w), ctypes.byref(out)) == T.TTT_ERR_INVALID_ARG
    assert not out.value


def test_null_handle_calls_return_invalid_arg():
    import long_context_prefill_ttt_b200 as T
    assert T.lib.ttt_prefill(None, None, 4, None, 0) == T.TTT_ERR_INVALID_ARG
    assert T.lib.ttt_decode(None, 1, None, None, None, 0) == T.TTT_ERR_INVALID_ARG
    assert T.lib.ttt_reset(None) == T.TTT_ERR_INVALID_ARG
    assert T.lib.ttt_k_gemm_pair(T.TTT_BF16, None, None, None) == T.TTT_ERR_INVALID_ARG
    empty = T.ttt_gemm_desc()          # null operands: rejected before any CUDA call
    assert T.lib.ttt_k_gemm_pair(T.TTT_BF16, ctypes.byref(empty), ctypes.byref(empty), None) == T.TTT_ERR_INVALID_ARG
    assert T.lib.ttt_position(None) == -1
    T.lib.ttt_destroy(None)


def test_binding_refuses_buffers_that_do_not_cover_the_call():
    """The library sees only addresses, so the binding checks element types and extents
    first: nothing undersized or mistyped reaches a kernel."""
    import long_context_prefill_ttt_b200 as T
    bf = torch.bfloat16
    M, N, K = 64, 128, 64
    A, B, D = torch.zeros(M, K, dtype=bf), torch.zeros(N, K, dtype=bf), torch.zeros(M, N)
    with pytest.raises(ValueError, match="A: .* elements"):
        T.ttt_k_gemm(A[:10], B, D, M, N, K)
    with pytest.raises(ValueError, match="D: .* elements"):
        T.ttt_k_gemm(A, B, D[:5], M, N, K)
    with pytest.raises(ValueError, match="X: element type"):
        T.ttt_k_gemm(A, B, D, M, N, K, X=torch.zeros(M, N, dtype=bf), ldx=N, epi=T.EPI_RESID)
    with pytest.raises(ValueError, match="B2: .* elements"):
        T.ttt_k_gemm(A, B, D, M, N, K, batch=2, sA=0, sB=0, B2=B, sB2=N * K, sD=0)
    with pytest.raises(ValueError, match="must be a device buffer"):
        T.ttt_k_gemm(A, B, D, M, N, K)       # right sizes, but host memory
    one = dict(A=A, B=B, D=D, M=M, N=N, K=K)
    with pytest.raises(ValueError, match="D: .* elements"):
        T.ttt_k_gemm_pair(dict(one, D=D[:5]), one)
    with pytest.raises(ValueError, match="same element type"):
        T.ttt_k_gemm_pair(one, dict(one, A=A.float(), B=B.float()))
    with pytest.raises(ValueError, match="must be a device buffer"):
        T.ttt_k_gemm_pair(one, one)
    qkv, out, lse = torch.zeros(4 * 3 * 64, dtype=bf), torch.zeros(4 * 64, dtype=bf), torch.zeros(4)
    with pytest.raises(ValueError, match="ring_k"):
        T.ttt_k_attention_fwd(qkv, out, lse, 1, 1, 64, 4, 128, 64, None, None, 256)
    with pytest.raises(ValueError, match="qkv: .* elements"):
        T.ttt_k_attention_fwd(qkv, out, lse, 1, 2, 64, 4, 0, 64)


def test_binding_checks_prefill_and_create_inputs():
    import long_context_prefill_ttt_b200 as T
    cfg = syn.config("tiny_fp32", T=32)
    h = T.Handle(None, cfg, T.make_config(cfg))   # never reaches the library: inputs are refused first
    toks = syn.make_token_batch(cfg)
    with pytest.raises(ValueError, match="int32"):
        T.ttt_prefill(h, toks.astype(np.int64))
    with pytest.raises(ValueError, match="shape"):
        T.ttt_prefill(h, np.ascontiguousarray(np.concatenate([toks, toks])))
    with pytest.raises(ValueError, match="out_losses"):
        T.ttt_prefill(h, toks, np.zeros((1, 31), dtype=np.float32))
    with pytest.raises(ValueError, match="forced"):
        T.ttt_decode(h, 4, forced=np.zeros((1, 3), dtype=np.int32))
    w = syn.make_weights(cfg)
    w["layers.0.Wq"] = w["layers.0.Wq"][:-1]
    with pytest.raises(ValueError, match="layers.0.Wq"):
        T.ttt_create(cfg, w)
    assert T.weight_shapes(cfg) == [int(np.prod(s)) for _, s in syn.weight_shapes(cfg)]


def test_every_device_allocation_goes_through_the_one_allocation_routine():
    """The allocation-failure hook (include/ttt_testing.h) and the allocation-free entry
    point rely on this: the library calls cudaMalloc in exactly one place."""
    csrc = os.path.join(ROOT, "long_context_prefill_ttt_b200", "csrc")
    sites = []
    for f in sorted(os.listdir(csrc)):
        for i, line in enumerate(open(os.path.join(csrc, f)), 1):
            code = line.split("//")[0]
            if re.search(r"\bcu(da)?Mem(Alloc|alloc)\w*\s*\(|\bcudaMalloc\w*\s*\(", code):
                sites.append((f, i))
    assert len(sites) == 1 and sites[0][0] == "ttt_runtime.cu", sites
    src = open(os.path.join(csrc, "ttt_runtime.cu")).read()
    body = src[src.index("cudaError_t device_alloc("):]
    assert "cudaMalloc(p, bytes)" in body[:body.index("\n}\n")]
