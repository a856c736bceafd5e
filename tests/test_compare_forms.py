"""The pages' two other loss forms, as `bench.py --compare` runs them in plain
PyTorch ("Full Dense KL": dense scattered teacher against the dense log-softmax;
"Forward-Chunked Loss": sparse teacher, chunked loss, full logits kept for the
backward), compute the same objective as the oracle: loss, dH and dW agree on a
small fp32 case, so the comparison times the same work."""
import numpy as np
import pytest
import torch

import bench
import oracle
from chunked_kl_loss_logits_b200.workloads import small_case


@pytest.mark.parametrize("form", ["dense", "forward_chunked"])
def test_form_matches_oracle(form):
    x = small_case(50, 32, 700, 10, seed=3)
    r = oracle.fwd_bwd(x["H"], x["W"], x["idx"], x["logit"])
    H = torch.tensor(x["H"], requires_grad=True)
    W = torch.tensor(x["W"], requires_grad=True)
    idx, lg = torch.tensor(x["idx"]), torch.tensor(x["logit"])
    loss = bench._dense_kl(H, W, idx, lg) if form == "dense" else \
        bench._forward_chunked_kl(H, W, idx, lg, 16)
    loss.backward()
    assert abs(loss.item() - r["loss"]) <= 1e-5 * abs(r["loss"])
    for g, ref in ((H.grad, r["dH"]), (W.grad, r["dW"])):
        assert np.abs(g.numpy() - ref).max() <= 1e-5 * np.abs(ref).max()
