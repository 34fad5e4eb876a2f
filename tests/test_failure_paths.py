"""Failure paths of the library's error contract (include/ttt.h), made on the host.

No GPU is faulted, trapped or hung: an allocation failure is injected into the
library's single allocation routine, and an expired device wait is simulated by
writing its status code into the device status word while no kernel runs
(include/ttt_testing.h).
"""
import numpy as np
import pytest
import torch

import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def T():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import long_context_prefill_ttt_b200 as T
    return T


def _free_bytes():
    torch.cuda.synchronize()
    return torch.cuda.mem_get_info()[0]


def test_create_reports_oom_at_any_allocation_and_leaks_nothing(T):
    cfg = syn.config("small_bf16", T=512)
    w = syn.make_weights(cfg)
    # one successful create: how many allocations does a handle make, and how large is it
    n0 = T.ttt_test_allocation_count()
    h = T.ttt_create(cfg, w)
    n_alloc = T.ttt_test_allocation_count() - n0
    size = T.ttt_device_bytes(h)
    T.ttt_destroy(h)
    assert n_alloc > 10 and size > 100 << 20
    base = _free_bytes()
    # the last request is the weight staging buffer (the weights are host arrays)
    for k in (0, 1, n_alloc // 2, n_alloc - 2, n_alloc - 1):
        T.ttt_test_fail_allocation(k)
        try:
            with pytest.raises(T.TTTError) as e:
                T.ttt_create(cfg, w)
            assert e.value.code == T.TTT_ERR_OOM
        finally:
            T.ttt_test_fail_allocation(-1)
        # everything allocated before the failing request was released
        assert abs(_free_bytes() - base) < 32 << 20, k
    # and the library still works afterwards
    h = T.ttt_create(cfg, w)
    losses = T.ttt_prefill(h, syn.make_token_batch(cfg))
    assert np.all(np.isfinite(losses))
    T.ttt_destroy(h)


@pytest.mark.parametrize("code", [1, 2, 3, 5])
def test_expired_device_wait_reports_timeout_then_poisons_the_handle(T, code):
    cfg = syn.config("tiny_fp32", T=32)
    w = syn.make_weights(cfg)
    h = T.ttt_create(cfg, w)
    T.ttt_prefill(h, syn.make_token_batch(cfg))
    T.ttt_test_set_device_status(h, code)
    # the next call that synchronises sees the status word (this one runs no waiting kernel)
    with pytest.raises(T.TTTError) as e:
        T.ttt_get_weights(h, 0, 0)
    assert e.value.code == T.TTT_ERR_TIMEOUT
    assert "device wait expired" in T.ttt_last_error(h)
    # from now on every call is refused before touching the device
    for call in (lambda: T.ttt_get_weights(h, 0, 0), lambda: T.ttt_reset(h),
                 lambda: T.ttt_prefill(h, syn.make_token_batch(cfg)), lambda: T.ttt_decode(h, 2)):
        with pytest.raises(T.TTTError) as e:
            call()
        assert e.value.code == T.TTT_ERR_POISONED
    T.ttt_destroy(h)


def test_kernel_status_word_reports_timeout_once_and_is_cleared(T):
    assert T.lib.ttt_k_status(None) == T.TTT_OK
    T.ttt_k_test_set_status(1)
    assert T.lib.ttt_k_status(None) == T.TTT_ERR_TIMEOUT
    assert T.lib.ttt_k_status(None) == T.TTT_OK
