"""Python binding of the TTT-E2E inner-loop library (B200, sm_100a).

Argument marshalling only: every step of prefill and decode runs in the CUDA
library libttt_b200.so through its C ABI (include/ttt.h, include/ttt_kernels.h).
PyTorch supplies device memory and the CUDA stream. There is no fallback: if
the library is missing, importing the binding raises.

    h = ttt_create(cfg, weights)            # cfg: object/dict with the ttt_config fields
    losses = ttt_prefill(h, tokens)         # tokens [B][T+1] int32 (torch or numpy)
    toks, losses = ttt_decode(h, n)
    w1, w2 = ttt_get_weights(h, seq, block)
    ttt_destroy(h)
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libttt_b200.so")

TTT_OK, TTT_ERR_INVALID_ARG, TTT_ERR_OOM, TTT_ERR_CUDA = 0, -1, -2, -3
TTT_ERR_TIMEOUT, TTT_ERR_STREAM, TTT_ERR_POISONED, TTT_ERR_UNSUPPORTED = -4, -5, -6, -7
TTT_FP32, TTT_BF16 = 0, 1
TTT_LOSS_E2E, TTT_LOSS_KVB = 0, 1
TTT_PTR_HOST, TTT_PTR_DEVICE = 0, 1
EPI_STORE, EPI_RESID, EPI_GELU, EPI_DGELU, EPI_SGD = 0, 1, 2, 3, 4
ENGINE_AUTO, ENGINE_SIMT, ENGINE_MMA, ENGINE_TC1 = 0, 1, 2, 3

_ERRNAMES = {0: "OK", -1: "INVALID_ARG", -2: "OOM", -3: "CUDA", -4: "TIMEOUT", -5: "STREAM", -6: "POISONED",
             -7: "UNSUPPORTED"}


class TTTError(RuntimeError):
    def __init__(self, code, msg=""):
        super().__init__(f"TTT_ERR_{_ERRNAMES.get(code, code)}: {msg}")
        self.code = code


class ttt_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("vocab", "d", "n_layers", "n_heads", "n_ttt", "mlp_hidden",
                                              "ttt_hidden", "static_hidden", "window_k", "minibatch_b", "batch")] + \
               [("eta", ctypes.c_float), ("rms_eps", ctypes.c_float), ("rope_base", ctypes.c_float),
                ("dtype", ctypes.c_int32), ("max_segment", ctypes.c_int32), ("inner_loss", ctypes.c_int32),
                ("cuda_stream", ctypes.c_void_p)]


class ttt_weights(ctypes.Structure):
    _fields_ = [("tensors", ctypes.POINTER(ctypes.c_void_p)), ("n_tensors", ctypes.c_int32),
                ("values_dtype", ctypes.c_int32), ("ptr_kind", ctypes.c_int32)]


class ttt_gemm_desc(ctypes.Structure):
    """One product of ttt_k_gemm_pair (the arguments of ttt_k_gemm)."""
    _fields_ = [("M", ctypes.c_int32), ("N", ctypes.c_int32), ("K", ctypes.c_int32), ("batch", ctypes.c_int32),
                ("A", ctypes.c_void_p), ("lda", ctypes.c_int64), ("sA", ctypes.c_int64), ("a_mn", ctypes.c_int32),
                ("B", ctypes.c_void_p), ("ldb", ctypes.c_int64), ("sB", ctypes.c_int64), ("b_mn", ctypes.c_int32),
                ("B2", ctypes.c_void_p), ("sB2", ctypes.c_int64),
                ("D", ctypes.c_void_p), ("ldd", ctypes.c_int64), ("sD", ctypes.c_int64), ("d_f32", ctypes.c_int32),
                ("X", ctypes.c_void_p), ("ldx", ctypes.c_int64), ("sX", ctypes.c_int64),
                ("Y", ctypes.c_void_p), ("ldy", ctypes.c_int64), ("sY", ctypes.c_int64),
                ("alpha", ctypes.c_float), ("epi", ctypes.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m long_context_prefill_ttt_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, F, VP = ctypes.POINTER, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p
    sigs = {
        "ttt_num_weight_tensors": (I32, [P(ttt_config)]),
        "ttt_create": (ctypes.c_int, [P(ttt_config), P(ttt_weights), P(VP)]),
        "ttt_prefill": (ctypes.c_int, [VP, VP, I64, VP, I32]),
        "ttt_decode": (ctypes.c_int, [VP, I64, VP, VP, VP, I32]),
        "ttt_get_weights": (ctypes.c_int, [VP, I32, I32, VP, VP, I32]),
        "ttt_reset": (ctypes.c_int, [VP]),
        "ttt_position": (I64, [VP]),
        "ttt_device_bytes": (I64, [VP]),
        "ttt_last_launch_count": (I64, [VP]),
        "ttt_destroy": (None, [VP]),
        "ttt_profile": (ctypes.c_int, [VP, I32]),
        "ttt_profile_read": (ctypes.c_int, [VP, I32, VP, VP, VP, VP]),
        "ttt_last_error": (ctypes.c_char_p, [VP]),
        "ttt_version": (ctypes.c_char_p, []),
        "ttt_k_gemm": (ctypes.c_int, [I32, I32, I32, I32, I32, VP, I64, I64, I32, VP, I64, I64, I32, VP, I64, VP,
                                      I64, I64, I32, VP, I64, I64, VP, I64, I64, F, I32, I32, VP]),
        "ttt_k_gemm_pair": (ctypes.c_int, [I32, P(ttt_gemm_desc), P(ttt_gemm_desc), VP]),
        "ttt_k_attention_fwd": (ctypes.c_int, [I32, I32, I32, I32, I32, I64, I32, VP, VP, VP, I32, VP, VP, I32, VP]),
        "ttt_k_attention_bwd": (ctypes.c_int, [I32, I32, I32, I32, I32, I64, I32, VP, VP, VP, I32, VP, VP, VP, VP,
                                               VP, I32, VP]),
        "ttt_k_attention_bwd_noalloc": (ctypes.c_int, [I32, I32, I32, I32, I32, I64, I32, VP, VP, VP, I32, VP, VP,
                                                       VP, VP, I32, VP]),
        "ttt_k_status": (ctypes.c_int, [VP]),
        "ttt_k_lm_head_ce": (ctypes.c_int, [I32, I32, I32, VP, VP, VP, VP, VP, VP, F, VP]),
        "ttt_test_fail_allocation": (None, [I64]),
        "ttt_test_allocation_count": (I64, []),
        "ttt_test_set_device_status": (ctypes.c_int, [VP, I32]),
        "ttt_k_test_set_status": (ctypes.c_int, [I32]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


# ----------------------------------------------------------------------------- helpers

def _torch():
    import torch
    return torch


def _stream_ptr(stream=None):
    torch = _torch()
    if stream is not None:
        return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))
    if torch.cuda.is_available():
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return ctypes.c_void_p(0)


def _ptr(x):
    """(address, ptr_kind) of a contiguous torch tensor or numpy array."""
    if x is None:
        return None, TTT_PTR_HOST
    if isinstance(x, np.ndarray):
        assert x.flags["C_CONTIGUOUS"], "arrays must be contiguous"
        return x.ctypes.data, TTT_PTR_HOST
    assert x.is_contiguous(), "tensors must be contiguous"
    return x.data_ptr(), (TTT_PTR_DEVICE if x.is_cuda else TTT_PTR_HOST)


def _is_torch(x):
    return not isinstance(x, np.ndarray) and hasattr(x, "data_ptr")


def _elem_name(x):
    if isinstance(x, np.ndarray):
        return str(x.dtype)
    return str(x.dtype).replace("torch.", "")


def _check(x, name, dtypes, min_elems=None, shape=None, cuda=None):
    """Validate a buffer handed to the library, which only sees its address: element
    type in dtypes (names such as "int32", "float32", "bfloat16"), contiguous, and
    covering min_elems elements (or exactly `shape`). cuda=True/False requires a
    device/host buffer. Raises ValueError before anything reaches the device."""
    if x is None:
        raise ValueError(f"{name}: missing buffer")
    if _elem_name(x) not in dtypes:
        raise ValueError(f"{name}: element type {_elem_name(x)}, expected {' or '.join(dtypes)}")
    contiguous = x.flags["C_CONTIGUOUS"] if isinstance(x, np.ndarray) else x.is_contiguous()
    if not contiguous:
        raise ValueError(f"{name}: must be contiguous")
    if shape is not None and tuple(x.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(x.shape)}, expected {tuple(shape)}")
    numel = x.size if isinstance(x, np.ndarray) else x.numel()
    if min_elems is not None and numel < min_elems:
        raise ValueError(f"{name}: {numel} elements, the call reads or writes {min_elems}")
    if cuda is not None:
        on_cuda = _is_torch(x) and x.is_cuda
        if on_cuda != cuda:
            raise ValueError(f"{name}: must be a {'device' if cuda else 'host'} buffer")


def _on_device(**bufs):
    for name, x in bufs.items():
        if x is not None and not (_is_torch(x) and x.is_cuda):
            raise ValueError(f"{name}: must be a device buffer")


def _extent(rows, cols, ld, stride, batch):
    """Elements spanned by `batch` row-major [rows][cols] slices with leading dimension
    ld, `stride` apart (stride 0: one slice shared by all)."""
    if rows <= 0 or cols <= 0:
        return 0
    return (batch - 1) * stride + (rows - 1) * ld + cols


def _get(cfg, name, default=None):
    if isinstance(cfg, dict):
        return cfg.get(name, default)
    return getattr(cfg, name, default)


def make_config(cfg, stream=None, max_segment=0) -> ttt_config:
    """Fill the C struct from any object or dict carrying the fields of ttt_config."""
    c = ttt_config()
    for n in ("vocab", "d", "n_layers", "n_heads", "n_ttt", "mlp_hidden", "ttt_hidden", "static_hidden",
              "window_k", "minibatch_b", "batch"):
        setattr(c, n, int(_get(cfg, n)))
    c.eta = float(_get(cfg, "eta"))
    c.rms_eps = float(_get(cfg, "rms_eps", 1e-6))
    c.rope_base = float(_get(cfg, "rope_base", 10000.0))
    dt = _get(cfg, "dtype", "bf16")
    c.dtype = TTT_BF16 if dt in ("bf16", TTT_BF16) else TTT_FP32
    c.max_segment = int(max_segment or _get(cfg, "max_segment", 0) or 0)
    loss = _get(cfg, "inner_loss", "e2e")
    if loss not in ("e2e", "kvb", TTT_LOSS_E2E, TTT_LOSS_KVB):
        raise ValueError(f"inner_loss must be 'e2e' or 'kvb', not {loss!r}")
    c.inner_loss = TTT_LOSS_KVB if loss in ("kvb", TTT_LOSS_KVB) else TTT_LOSS_E2E
    c.cuda_stream = _stream_ptr(stream).value
    return c


def weight_names(cfg):
    """Tensor order of ttt_weights (include/ttt.h)."""
    names = ["E", "final_norm"]
    L, Lt = int(_get(cfg, "n_layers")), int(_get(cfg, "n_ttt"))
    for l in range(L):
        p = f"layers.{l}."
        names += [p + n for n in ("attn_norm", "Wq", "Wk", "Wv", "Wo")]
        if l >= L - Lt:
            names += [p + n for n in ("ttt_norm", "W1t", "W2t", "static_norm", "W1s", "W2s")]
            if _get(cfg, "inner_loss", "e2e") in ("kvb", TTT_LOSS_KVB):
                names += [p + "theta_K", p + "theta_V"]
        else:
            names += [p + n for n in ("mlp_norm", "W1", "W2")]
    return names


class Handle:
    """Owns a ttt_handle*; keeps the config and stream it was created with."""

    def __init__(self, ptr, cfg, cstruct):
        self.ptr = ptr
        self.cfg = cfg
        self.c = cstruct

    @property
    def batch(self):
        return self.c.batch

    def error(self):
        return lib.ttt_last_error(self.ptr).decode()

    def check(self, rc):
        if rc != TTT_OK:
            raise TTTError(rc, self.error())

    def __del__(self, _lib=lib):
        # _lib is bound at class creation: module globals may already be gone at interpreter exit
        if getattr(self, "ptr", None) and _lib is not None:
            _lib.ttt_destroy(self.ptr)
            self.ptr = None


# ----------------------------------------------------------------------------- C ABI, same names

def weight_shapes(cfg):
    """Element counts of the weight tensors, in weight_names order (include/ttt.h)."""
    V, d = _get(cfg, "vocab"), _get(cfg, "d")
    L, Lt = _get(cfg, "n_layers"), _get(cfg, "n_ttt")
    h, ht, hs = _get(cfg, "mlp_hidden"), _get(cfg, "ttt_hidden"), _get(cfg, "static_hidden")
    out = [V * d, d]
    for l in range(L):
        out += [d, d * d, d * d, d * d, d * d]
        if l >= L - Lt:
            out += [d, ht * d, d * ht, d, hs * d, d * hs]
            if _get(cfg, "inner_loss", "e2e") in ("kvb", TTT_LOSS_KVB):
                out += [d * d, d * d]
        else:
            out += [d, h * d, d * h]
    return out


def ttt_create(cfg, weights, stream=None, max_segment=0) -> Handle:
    """weights: dict name -> float32 array/tensor (values exactly representable in cfg's dtype)."""
    c = make_config(cfg, stream, max_segment)
    names = weight_names(cfg)
    ptrs, kinds, keep = [], set(), []
    for n, numel in zip(names, weight_shapes(cfg)):
        t = weights[n]
        if isinstance(t, np.ndarray):
            t = np.ascontiguousarray(t, dtype=np.float32)
        _check(t, n, ("float32",))
        tn = t.size if isinstance(t, np.ndarray) else t.numel()
        if tn != numel:
            raise ValueError(f"{n}: {tn} elements, the model has {numel}")
        keep.append(t)
        p, k = _ptr(t)
        ptrs.append(p)
        kinds.add(k)
    if len(kinds) != 1:
        raise ValueError("weights must be all host or all device")
    arr = (ctypes.c_void_p * len(ptrs))(*ptrs)
    w = ttt_weights(ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p)), len(ptrs), TTT_FP32, kinds.pop())
    out = ctypes.c_void_p()
    rc = lib.ttt_create(ctypes.byref(c), ctypes.byref(w), ctypes.byref(out))
    if rc != TTT_OK:
        raise TTTError(rc, "ttt_create failed")
    return Handle(out, cfg, c)


def ttt_prefill(h: Handle, tokens, out_losses=None):
    """tokens [B][T+1] int32; returns losses [B][T] (float32, same kind as tokens)."""
    if len(tokens.shape) != 2 or tokens.shape[0] != h.batch or tokens.shape[1] < 2:
        raise ValueError(f"tokens: shape {tuple(tokens.shape)}, expected [B={h.batch}][T+1] with T >= 1")
    B, n1 = tokens.shape
    T = n1 - 1
    on_cuda = _is_torch(tokens) and tokens.is_cuda
    _check(tokens, "tokens", ("int32",))
    if out_losses is None:
        if isinstance(tokens, np.ndarray):
            out_losses = np.empty((B, T), dtype=np.float32)
        else:
            out_losses = _torch().empty((B, T), dtype=_torch().float32, device=tokens.device)
    _check(out_losses, "out_losses", ("float32",), shape=(B, T), cuda=on_cuda)
    tp, kind = _ptr(tokens)
    lp, _ = _ptr(out_losses)
    h.check(lib.ttt_prefill(h.ptr, ctypes.c_void_p(tp), T, ctypes.c_void_p(lp), kind))
    return out_losses


def ttt_decode(h: Handle, n: int, forced=None, device=None):
    """Generate n tokens per sequence; returns (tokens [B][n] int32, losses [B][n] float32)."""
    B = h.batch
    if device is not None and str(device).startswith("cuda"):
        torch = _torch()
        toks = torch.empty((B, n), dtype=torch.int32, device=device)
        losses = torch.empty((B, n), dtype=torch.float32, device=device)
        kind = TTT_PTR_DEVICE
        if forced is not None:
            _check(forced, "forced", ("int32",), shape=(B, n), cuda=True)
        fp = forced.data_ptr() if forced is not None else None
        tp, lp = toks.data_ptr(), losses.data_ptr()
    else:
        toks = np.empty((B, n), dtype=np.int32)
        losses = np.empty((B, n), dtype=np.float32)
        kind = TTT_PTR_HOST
        if forced is not None:
            forced = np.ascontiguousarray(forced, dtype=np.int32)
            _check(forced, "forced", ("int32",), shape=(B, n))
        fp = forced.ctypes.data if forced is not None else None
        tp, lp = toks.ctypes.data, losses.ctypes.data
    h.check(lib.ttt_decode(h.ptr, n, ctypes.c_void_p(fp) if fp else None, ctypes.c_void_p(tp),
                           ctypes.c_void_p(lp), kind))
    return toks, losses


def ttt_get_weights(h: Handle, seq: int, block: int):
    """fp32 fast weights (W1t [h_t][d], W2t [d][h_t]) of sequence seq, adaptive block `block`."""
    d, ht = h.c.d, h.c.ttt_hidden
    w1 = np.empty((ht, d), dtype=np.float32)
    w2 = np.empty((d, ht), dtype=np.float32)
    h.check(lib.ttt_get_weights(h.ptr, seq, block, ctypes.c_void_p(w1.ctypes.data), ctypes.c_void_p(w2.ctypes.data),
                                TTT_PTR_HOST))
    return w1, w2


def ttt_reset(h: Handle):
    h.check(lib.ttt_reset(h.ptr))


def ttt_destroy(h: Handle):
    if h.ptr:
        lib.ttt_destroy(h.ptr)
        h.ptr = None


def ttt_last_error(h: Handle) -> str:
    return h.error()


def ttt_position(h: Handle) -> int:
    return int(lib.ttt_position(h.ptr))


def ttt_device_bytes(h: Handle) -> int:
    return int(lib.ttt_device_bytes(h.ptr))


def ttt_last_launch_count(h: Handle) -> int:
    return int(lib.ttt_last_launch_count(h.ptr))


PROFILE_CLASSES = ("gemm_frozen", "gemm_adaptive", "attention_fwd", "attention_bwd")


def ttt_profile(h: Handle, enable: bool = True):
    h.check(lib.ttt_profile(h.ptr, int(enable)))


def ttt_profile_read(h: Handle):
    """{class: dict(ms, launches, flops, bytes)} accumulated since ttt_profile(h, True)."""
    n = len(PROFILE_CLASSES)
    ms = (ctypes.c_double * n)()
    la = (ctypes.c_int64 * n)()
    fl = (ctypes.c_double * n)()
    by = (ctypes.c_double * n)()
    lib.ttt_profile_read(h.ptr, n, ms, la, fl, by)
    return {c: dict(ms=ms[i], launches=la[i], flops=fl[i], bytes=by[i]) for i, c in enumerate(PROFILE_CLASSES)}


def ttt_version() -> str:
    return lib.ttt_version().decode()


# ----------------------------------------------------------------------------- per-kernel ABI

def _dtype_code(t):
    torch = _torch()
    return TTT_BF16 if t.dtype == torch.bfloat16 else TTT_FP32


def _gemm_desc(A, B, D, M, N, K, *, batch=1, lda=None, sA=0, a_mn=False, ldb=None, sB=0, b_mn=False, B2=None,
               sB2=0, ldd=None, sD=0, X=None, ldx=0, sX=0, Y=None, ldy=0, sY=0, alpha=1.0, epi=EPI_STORE):
    """Checks one product's device tensors against its sizes; returns its ttt_gemm_desc."""
    torch = _torch()
    lda = lda if lda is not None else (M if a_mn else K)
    ldb = ldb if ldb is not None else (N if b_mn else K)
    ldd = ldd if ldd is not None else N
    el = (_elem_name(A),)
    if el[0] not in ("bfloat16", "float32"):
        raise ValueError(f"A: element type {el[0]}, expected bfloat16 or float32")
    a_rows, a_cols = (K, M) if a_mn else (M, K)
    b_rows, b_cols = (K, N) if b_mn else (N, K)
    if lda < a_cols or ldb < b_cols or ldd < N:
        raise ValueError("leading dimensions must cover a row")
    _check(A, "A", el, _extent(a_rows, a_cols, lda, sA, batch))
    _check(B, "B", el, _extent(b_rows, b_cols, ldb, sB, batch))
    if B2 is not None:
        _check(B2, "B2", el, _extent(b_rows, b_cols, ldb, sB2, batch))
    _check(D, "D", ("float32",) + el, _extent(M, N, ldd, sD, batch))
    if X is not None:
        _check(X, "X", ("float32",) if epi == EPI_RESID else el, _extent(M, N, ldx, sX, batch))
    if Y is not None:
        _check(Y, "Y", el, _extent(M, N, ldy, sY, batch))
    _on_device(A=A, B=B, B2=B2, D=D, X=X, Y=Y)
    ptr = lambda x: x.data_ptr() if x is not None else None  # noqa: E731
    return ttt_gemm_desc(M, N, K, batch, A.data_ptr(), lda, sA, int(a_mn), B.data_ptr(), ldb, sB, int(b_mn),
                         ptr(B2), sB2, D.data_ptr(), ldd, sD, int(D.dtype == torch.float32), ptr(X), ldx, sX,
                         ptr(Y), ldy, sY, float(alpha), epi)


def ttt_k_gemm(A, B, D, M, N, K, *, engine=ENGINE_AUTO, stream=None, **kw):
    """Enqueue one contraction on device tensors (see include/ttt_kernels.h); keyword
    arguments as _gemm_desc."""
    g = _gemm_desc(A, B, D, M, N, K, **kw)
    rc = lib.ttt_k_gemm(_dtype_code(A), g.M, g.N, g.K, g.batch, g.A, g.lda, g.sA, g.a_mn, g.B, g.ldb, g.sB, g.b_mn,
                        g.B2, g.sB2, g.D, g.ldd, g.sD, g.d_f32, g.X, g.ldx, g.sX, g.Y, g.ldy, g.sY, g.alpha, g.epi,
                        engine, _stream_ptr(stream))
    if rc != TTT_OK:
        raise TTTError(rc, "ttt_k_gemm")


def ttt_k_gemm_pair(first, second, stream=None):
    """Enqueue two independent contractions, one launch where they can share it.
    first, second: dicts of ttt_k_gemm's arguments (A, B, D, M, N, K and keywords)."""
    if _elem_name(first["A"]) != _elem_name(second["A"]):
        raise ValueError("both products must have the same element type")
    a, b = _gemm_desc(**first), _gemm_desc(**second)
    rc = lib.ttt_k_gemm_pair(_dtype_code(first["A"]), ctypes.byref(a), ctypes.byref(b), _stream_ptr(stream))
    if rc != TTT_OK:
        raise TTTError(rc, "ttt_k_gemm_pair")


def _check_attention(qkv, out, lse, B, H, hd, n, q0, ring_k, ring_v, C, dout=None, dqkv=None, dsum=None):
    el = (_elem_name(qkv),)
    d = H * hd
    _check(qkv, "qkv", el, B * n * 3 * d)
    _check(out, "out", el, B * n * d)
    if lse is not None:
        _check(lse, "lse", ("float32",), B * H * n)
    if q0 > 0:
        _check(ring_k, "ring_k", el, B * C * d)
        _check(ring_v, "ring_v", el, B * C * d)
    if dout is not None:
        _check(dout, "dout", el, B * n * d)
    if dqkv is not None:
        _check(dqkv, "dqkv", el, B * n * 3 * d)
    if dsum is not None:
        _check(dsum, "dsum", ("float32",), B * H * n)
    _on_device(qkv=qkv, out=out, lse=lse, ring_k=ring_k if q0 > 0 else None, ring_v=ring_v if q0 > 0 else None,
               dout=dout, dqkv=dqkv, dsum=dsum)


def ttt_k_attention_fwd(qkv, out, lse, B, H, hd, n, q0, window, ring_k=None, ring_v=None, C=0,
                        engine=ENGINE_AUTO, stream=None):
    _check_attention(qkv, out, lse, B, H, hd, n, q0, ring_k, ring_v, C)
    rc = lib.ttt_k_attention_fwd(_dtype_code(qkv), B, H, hd, n, q0, window, qkv.data_ptr(),
                                 ring_k.data_ptr() if ring_k is not None else None,
                                 ring_v.data_ptr() if ring_v is not None else None, C, out.data_ptr(),
                                 lse.data_ptr() if lse is not None else None, engine, _stream_ptr(stream))
    if rc != TTT_OK:
        raise TTTError(rc, "ttt_k_attention_fwd")


def ttt_k_attention_bwd(qkv, out, lse, dout, dqkv, dsum, B, H, hd, n, q0, window, ring_k=None, ring_v=None, C=0,
                        engine=ENGINE_AUTO, stream=None):
    if lse is None:
        raise ValueError("lse: missing buffer")
    _check_attention(qkv, out, lse, B, H, hd, n, q0, ring_k, ring_v, C, dout=dout, dqkv=dqkv, dsum=dsum)
    rc = lib.ttt_k_attention_bwd(_dtype_code(qkv), B, H, hd, n, q0, window, qkv.data_ptr(),
                                 ring_k.data_ptr() if ring_k is not None else None,
                                 ring_v.data_ptr() if ring_v is not None else None, C, out.data_ptr(),
                                 lse.data_ptr(), dout.data_ptr(), dqkv.data_ptr(), dsum.data_ptr(), engine,
                                 _stream_ptr(stream))
    if rc != TTT_OK:
        raise TTTError(rc, "ttt_k_attention_bwd")


def ttt_k_attention_bwd_noalloc(qkv, out, lse, dout, dqkv, B, H, hd, n, q0, window, ring_k=None, ring_v=None, C=0,
                                engine=ENGINE_AUTO, stream=None):
    """Attention backward that allocates nothing (its scratch is a fixed array inside the library)."""
    if lse is None:
        raise ValueError("lse: missing buffer")
    _check_attention(qkv, out, lse, B, H, hd, n, q0, ring_k, ring_v, C, dout=dout, dqkv=dqkv)
    rc = lib.ttt_k_attention_bwd_noalloc(_dtype_code(qkv), B, H, hd, n, q0, window, qkv.data_ptr(),
                                         ring_k.data_ptr() if ring_k is not None else None,
                                         ring_v.data_ptr() if ring_v is not None else None, C, out.data_ptr(),
                                         lse.data_ptr(), dout.data_ptr(), dqkv.data_ptr(), engine,
                                         _stream_ptr(stream))
    if rc != TTT_OK:
        raise TTTError(rc, "ttt_k_attention_bwd_noalloc")


def ttt_k_lm_head_ce(r, E, targets, z, loss, scratch, M, V, d, grad_scale=0.0, stream=None):
    """Fused LM head + cross-entropy (include/ttt_kernels.h): z [M][V] gets the logits or dz."""
    _check(r, "r", ("bfloat16",), M * d)
    _check(E, "E", ("bfloat16",), V * d)
    _check(targets, "targets", ("int32",), M)
    _check(z, "z", ("bfloat16",), M * V)
    _check(loss, "loss", ("float32",), M)
    _check(scratch, "scratch", ("float32",), 2 * M * (V // 64) + M)
    _on_device(r=r, E=E, targets=targets, z=z, loss=loss, scratch=scratch)
    rc = lib.ttt_k_lm_head_ce(M, V, d, r.data_ptr(), E.data_ptr(), targets.data_ptr(), z.data_ptr(),
                              loss.data_ptr(), scratch.data_ptr(), float(grad_scale), _stream_ptr(stream))
    if rc != TTT_OK:
        raise TTTError(rc, "ttt_k_lm_head_ce")


def ttt_k_status(stream=None):
    rc = lib.ttt_k_status(_stream_ptr(stream))
    if rc != TTT_OK:
        raise TTTError(rc, "device status")


# ----------------------------------------------------------------------------- host-side fault injection (tests)

def ttt_test_fail_allocation(n: int):
    """Make the library's n-th device allocation from now fail (include/ttt_testing.h); n < 0 cancels."""
    lib.ttt_test_fail_allocation(int(n))


def ttt_test_allocation_count() -> int:
    return int(lib.ttt_test_allocation_count())


def ttt_test_set_device_status(h: Handle, code: int):
    h.check(lib.ttt_test_set_device_status(h.ptr, int(code)))


def ttt_k_test_set_status(code: int):
    rc = lib.ttt_k_test_set_status(int(code))
    if rc != TTT_OK:
        raise TTTError(rc, "ttt_k_test_set_status")
