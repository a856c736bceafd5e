"""Device-side failure detection, made to fire without a fault: a wait that
nothing will satisfy gives up after its bound, reports CKL_ERR_TIMEOUT through the
status word, and leaves the context usable (a normal call right after it succeeds
and matches the oracle)."""
import numpy as np
import pytest
import torch

import oracle
from chunked_kl_loss_logits_b200 import ckl
from chunked_kl_loss_logits_b200.workloads import small_case

pytestmark = pytest.mark.gpu


def test_wait_bound_fires_and_context_survives():
    dev = torch.device("cuda", 0)
    h = ckl.ChunkedKL(700, 64, 8, max_chunk=64, device=dev)
    code, cycles = h.selftest_wait_bound()
    assert code == 6, ckl._STATUS.get(code, code)  # timed out, as designed
    assert cycles >= 4_000_000_000
    h.sync_status()  # the status word was cleared by the self-test
    x = small_case(100, 64, 700, 8, seed=71, dtype="bf16")
    loss, dH, dW = h.fwd_bwd(torch.from_numpy(x["H"]).to(dev).to(torch.bfloat16),
                             torch.from_numpy(x["W"]).to(dev).to(torch.bfloat16),
                             torch.from_numpy(x["idx"]).to(dev),
                             torch.from_numpy(x["logit"]).to(dev), chunk=64)
    r = oracle.fwd_bwd(x["H"], x["W"], x["idx"], x["logit"])
    assert abs(loss.item() - r["loss"]) <= 1e-3 * abs(r["loss"])
    assert np.linalg.norm(dH.double().cpu().numpy() - r["dH"]) <= 2e-2 * np.linalg.norm(r["dH"])
    h.close()
