"""CPU-only checks of the C ABI: the library loads and exports every symbol that
include/*.h declares, and argument validation happens before any device call."""
import ctypes
import os
import re

import pytest

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
              "ttt_last_error", "ttt_k_gemm", "ttt_k_attention_fwd", "ttt_k_attention_bwd"):
        assert n in names


def test_library_exports_every_declared_symbol():
    import long_context_prefill_ttt_b200 as T
    lib = ctypes.CDLL(T.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert "sm_100a" in T.ttt_version()


def test_weight_tensor_count_and_order_match_the_generator():
    import long_context_prefill_ttt_b200 as T
    for name in ("tiny_fp32", "small_bf16", "b1_128k_bf16"):
        cfg = syn.config(name)
        c = T.make_config(cfg)
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


def test_null_handle_calls_return_invalid_arg():
    import long_context_prefill_ttt_b200 as T
    assert T.lib.ttt_prefill(None, None, 4, None, 0) == T.TTT_ERR_INVALID_ARG
    assert T.lib.ttt_decode(None, 1, None, None, None, 0) == T.TTT_ERR_INVALID_ARG
    assert T.lib.ttt_reset(None) == T.TTT_ERR_INVALID_ARG
    assert T.lib.ttt_position(None) == -1
    T.lib.ttt_destroy(None)
