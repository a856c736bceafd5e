"""Write tests/golden/tiny_case.json: a tiny seeded case and the oracle's outputs.

Run from the repository root: python tests/golden/make_golden.py
The expected values come from the fp64 oracle only. Before writing, they are
checked against PyTorch's fp64 kl_div on the dense teacher with autograd
gradients (the dense-teacher method, "Full Dense KL", that the README of "Chunked
KL loss, running Knowledge Distillation locally in less <6GB VRAM" uses as its
reference for correctness).
"""
import json
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from chunked_kl_loss_logits_b200.workloads import small_case  # noqa: E402


def main():
    x = small_case(4, 8, 32, 4, seed=2024)
    mask = np.array([1, 0, 1, 1], dtype=np.uint8)
    r = oracle.fwd_bwd(x["H"], x["W"], x["idx"], x["logit"], mask)

    Ht = torch.tensor(x["H"].astype(np.float64), requires_grad=True)
    Wt = torch.tensor(x["W"].astype(np.float64), requires_grad=True)
    lg = torch.tensor(x["logit"].astype(np.float64))
    P = torch.zeros(4, 32, dtype=torch.float64)
    P.scatter_add_(1, torch.tensor(x["idx"], dtype=torch.long), torch.softmax(lg, 1))
    kl = torch.nn.functional.kl_div(torch.log_softmax(Ht @ Wt.T, 1), P, reduction="none").sum(1)
    m = torch.tensor(mask, dtype=torch.float64)
    loss = (m * kl).sum() / m.sum()
    loss.backward()
    assert abs(loss.item() - r["loss"]) < 1e-12
    assert np.abs(Ht.grad.numpy() - r["dH"]).max() < 1e-13
    assert np.abs(Wt.grad.numpy() - r["dW"]).max() < 1e-13

    out = {
        "about": "T=4, d=8, V=32, K=4, token 1 masked; expected values from the fp64 oracle, "
                 "cross-checked against torch kl_div + autograd by make_golden.py",
        "inputs": {"H": x["H"].tolist(), "W": x["W"].tolist(), "idx": x["idx"].tolist(),
                   "logit": x["logit"].tolist(), "mask": mask.tolist()},
        "loss": r["loss"], "dH": r["dH"].tolist(), "dW": r["dW"].tolist(),
    }
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_case.json"), "w") as f:
        json.dump(out, f, indent=0)


if __name__ == "__main__":
    main()
