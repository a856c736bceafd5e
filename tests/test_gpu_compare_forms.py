"""The pages' two other loss forms, run in plain PyTorch on the GPU in bf16 (the
forms `bench.py --compare` times beside this library), against the fp64 oracle.

"Full Dense KL" rebuilds a dense teacher from the cache and takes PyTorch's KL
divergence on the full log-softmax; "Forward-Chunked Loss" evaluates the sparse
loss chunk by chunk from one full projection. Both are differentiated by autograd
from bf16 logits (the dtype a plain PyTorch model computes them in), so they meet
the bf16 bars of this method against the oracle on the same bf16 inputs, and they
agree with the fused library call. This pins the comparison to the same objective
on the hardware the comparison is measured on.
"""
import pytest
import torch

import bench
import oracle
from chunked_kl_loss_logits_b200 import ckl
from chunked_kl_loss_logits_b200.workloads import WORKLOADS, make_inputs
from tests._helpers import ROW_TOL, TOL, f64, rel, rel_fro, upload, worst_row

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("form", ["dense_kl", "forward_chunked"])
def test_comparison_form_matches_oracle_on_gpu(form):
    w = WORKLOADS["bf16_4k"]
    x = make_inputs(w, T=512)
    r = oracle.fwd_bwd(x["H"], x["W"], x["idx"], x["logit"], x["mask"])
    H, W, idx, logit, _ = upload(x, torch.bfloat16)
    Hp, Wp = H.clone().requires_grad_(True), W.clone().requires_grad_(True)
    loss = bench._dense_kl(Hp, Wp, idx, logit) if form == "dense_kl" else \
        bench._forward_chunked_kl(Hp, Wp, idx, logit, 128)
    loss.backward()
    errs = {"loss": rel(loss.item(), r["loss"]), "dH": rel_fro(f64(Hp.grad), r["dH"]),
            "dW": rel_fro(f64(Wp.grad), r["dW"]), "dH_row": worst_row(f64(Hp.grad), r["dH"]),
            "dW_row": worst_row(f64(Wp.grad), r["dW"])}
    print(form, {k: f"{v:.2e}" for k, v in errs.items()})
    assert errs["loss"] <= TOL["bf16"]["loss"] and errs["dH"] <= TOL["bf16"]["grad"]
    assert errs["dW"] <= TOL["bf16"]["grad"]
    assert errs["dH_row"] <= ROW_TOL["bf16"]["grad_row"]
    assert errs["dW_row"] <= ROW_TOL["bf16"]["grad_row"]
    # the fused call on the same inputs
    h = ckl.ChunkedKL(w.V, w.d, w.K, max_chunk=128)
    l1, dH1, dW1 = h.fwd_bwd(H, W, idx, logit, None, chunk=128)
    h.close()
    assert rel(loss.item(), l1.item()) <= TOL["bf16"]["loss"]
    assert rel_fro(f64(Hp.grad), f64(dH1)) <= TOL["bf16"]["grad"]
    assert rel_fro(f64(Wp.grad), f64(dW1)) <= TOL["bf16"]["grad"]
