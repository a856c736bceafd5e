"""The allocation-free forward entry point (ckl_forward_static), called through
the C ABI, against the existing ckl_forward on the same inputs.

Callers that may not call cudaMalloc (a host runtime that owns all device memory
through its own allocator, a latency-critical loop that cannot take the
device-wide synchronisation of an allocation) use this variant: its scratch is a
fixed 32 MiB device array inside the library, shared by all calls. The test makes
two calls in a row with different inputs, so state left in the shared array by
the first call would show up in the second. This file is collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from chunked_kl_loss_logits_b200 import build, ckl
from chunked_kl_loss_logits_b200.workloads import small_case
from tests._helpers import rel, rel_fro, upload

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 1e-3, torch.float32: 1e-5}
_P, _I64 = ctypes.c_void_p, ctypes.c_int64


def _entry():
    build.build()
    f = ckl.lib().ckl_forward_static
    f.argtypes = [ctypes.c_int, ctypes.c_int, _I64, _I64, _I64, _P, _P, _P, _P, _P, _I64, _I64,
                  _P, _P, _P, _P, _P]
    f.restype = ctypes.c_int
    return f


def _call_static(f, H, W, idx, logit, mask, chunk):
    T, d = H.shape
    V, K = W.shape[0], idx.shape[1]
    loss = torch.empty((), dtype=torch.float32, device="cuda")
    lse = torch.empty(T, dtype=torch.float32, device="cuda")
    ell = torch.empty(T, dtype=torch.float32, device="cuda")
    host = ctypes.c_float()
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    code = f(torch.cuda.current_device(), 0 if H.dtype == torch.float32 else 1, V, d, K, p(H),
             p(W), p(idx), p(logit), p(mask), T, chunk, p(loss), p(lse), p(ell),
             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream), ctypes.byref(host))
    return code, loss, lse, ell, host.value


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_static_forward_matches_forward_twice(dtype):
    f = _entry()
    dt = "bf16" if dtype == torch.bfloat16 else "f32"
    cases = [small_case(300, 128, 3000, 16, seed=31, dtype=dt, teacher_var=3.0, ids="zipf",
                        packing=True),
             small_case(517, 64, 1777, 12, seed=32, dtype=dt, teacher_var=3.0, ids="zipf")]
    for x, chunk in zip(cases, (128, 200)):
        H, W, idx, logit, mask = upload(x, dtype)
        code, loss, lse, ell, lh = _call_static(f, H, W, idx, logit, mask, chunk)
        assert code == 0, ckl.lib().ckl_status_str(code)
        h = ckl.ChunkedKL(W.shape[0], W.shape[1], idx.shape[1], dtype=dtype, max_chunk=chunk)
        l0, lse0, ell0 = h.forward(H, W, idx, logit, mask, chunk=chunk, token_stats=True)
        assert lh == loss.item()
        assert rel(loss.item(), l0.item()) <= TOL[dtype]
        assert rel_fro(lse.double().cpu().numpy(), lse0.double().cpu().numpy()) <= TOL[dtype]
        assert rel_fro(ell.double().cpu().numpy(), ell0.double().cpu().numpy()) <= TOL[dtype]
        h.close()


def test_static_forward_rejects_sizes_beyond_its_scratch():
    f = _entry()
    V, d, K = 201088, 64, 100
    W = torch.zeros(V, d, dtype=torch.bfloat16, device="cuda")
    T = 8192
    H = torch.zeros(T, d, dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros(T, K, dtype=torch.int32, device="cuda")
    logit = torch.zeros(T, K, dtype=torch.float32, device="cuda")
    code, *_ = _call_static(f, H, W, idx, logit, None, 8192)  # needs ~58 MiB of scratch
    assert code == 3
