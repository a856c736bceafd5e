"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/ckl.h declares, and rejects bad arguments before it
touches the device."""
import ctypes

import pytest

from chunked_kl_loss_logits_b200 import ckl

P = ctypes.c_void_p


@pytest.fixture(scope="module")
def L():
    from chunked_kl_loss_logits_b200 import build
    build.build()
    return ckl.lib()


def test_exports_every_declared_function(L):
    names = ckl.header_functions()
    assert {"ckl_create", "ckl_destroy", "ckl_fwd_bwd", "ckl_forward", "ckl_workspace_bytes",
            "ckl_fwd_bwd_from_host", "ckl_sync_status"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for code in range(10):
        s = L.ckl_status_str(code)
        assert s and s != b"unknown status"
    assert L.ckl_status_str(99) == b"unknown status"


@pytest.mark.parametrize("args,code", [
    ((0, 0, 0, 64, 1, 1), 1),          # V = 0
    ((0, 0, 100, 0, 1, 1), 1),         # d = 0
    ((0, 0, 100, 64, 0, 1), 1),        # K = 0
    ((0, 0, 100, 64, 1, 0), 1),        # max_chunk = 0
    ((-1, 0, 100, 64, 1, 1), 1),       # device < 0
    ((0, 7, 100, 64, 1, 1), 1),        # bad dtype
    ((0, 1, 100, 60, 1, 1), 2),        # d % 8 != 0
    ((0, 1, 100, 64, 1025, 1), 2),     # K > 1024
])
def test_create_rejects_bad_arguments(L, args, code):
    h = P()
    dev, dt, V, d, K, mc = args
    assert L.ckl_create(ctypes.byref(h), dev, dt, V, d, K, mc) == code
    assert not h.value


def test_create_without_a_device_reports_cuda(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    h = P()
    assert L.ckl_create(ctypes.byref(h), 0, 1, 1000, 64, 8, 128) == 5
    assert not h.value


def test_null_handle_calls(L):
    n = ctypes.c_size_t()
    assert L.ckl_workspace_bytes(None, 10, 4, ctypes.byref(n)) == 1
    assert L.ckl_fwd_bwd(None, *([None] * 5), 10, 4, *([None] * 6), 0, None, None) == 1
    assert L.ckl_forward(None, *([None] * 5), 10, 4, *([None] * 4), 0, None, None) == 1
    assert L.ckl_sync_status(None, None) == 1
    assert L.ckl_launch_count(None) == -1
    assert L.ckl_destroy(None) == 0
    assert L.ckl_profile_enable(None, 1, 16) == 1
    assert L.ckl_selftest_wait_bound(None, None, None) == 1
    assert L.ckl_topk_vp_workspace_bytes(None, 2, 10, 4, ctypes.byref(n)) == 1
    assert L.ckl_topk_cache_vocab_parallel(None, None, None, None, 10, 4, None, None, None, 0,
                                           None, 0) == 1
    assert L.ckl_vp_workspace_bytes(None, 2, 10, 4, ctypes.byref(n)) == 1
    assert L.ckl_fwd_bwd_vocab_parallel(None, None, *([None] * 5), 10, 4, *([None] * 6), 0, None,
                                        None) == 1
    assert L.ckl_forward_vocab_parallel(None, None, *([None] * 5), 10, 4, *([None] * 4), 0, None,
                                        None) == 1
