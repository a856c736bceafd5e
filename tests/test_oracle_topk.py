"""Pins of the oracle's teacher top-K cache builder.

The cache is the offline half of "Efficient Knowledge Distillation for LLMs:
Offline Top-K Logits and a Fused Chunked KL Loss" (abstract; the author's forum
post: each position keeps its 100 largest teacher logits). Pinned to
torch.topk, to closed forms for ties and constant logits, and to the loss: a
student distilled from its own cache has loss -log(the top-K probability mass of
its own softmax), zero when K = V.
"""
import numpy as np
import torch

import oracle
from chunked_kl_loss_logits_b200.workloads import small_case


def test_matches_torch_topk():
    x = small_case(9, 16, 300, 20, seed=41)
    idx, lg = oracle.topk_cache(x["H"], x["W"], 20)
    z = torch.tensor(np.asarray(x["H"], np.float64) @ np.asarray(x["W"], np.float64).T)
    v, i = torch.topk(z, 20, dim=1, largest=True, sorted=True)
    assert np.array_equal(idx, i.numpy())
    np.testing.assert_array_equal(lg, v.numpy())
    assert np.all(np.diff(lg, axis=1) <= 0)


def test_constant_logits_take_the_smallest_ids():
    x = small_case(4, 8, 50, 7, seed=42)
    idx, lg = oracle.topk_cache(x["H"], np.zeros_like(x["W"]), 7)
    assert np.array_equal(idx, np.tile(np.arange(7), (4, 1)))
    assert np.all(lg == 0.0)


def test_ties_break_by_id():
    rng = np.random.default_rng(43)
    W = rng.standard_normal((30, 6))
    W[17] = W[3]          # ids 3 and 17 always tie
    W[25] = W[3]
    H = rng.standard_normal((5, 6))
    idx, lg = oracle.topk_cache(H, W, 30)
    for t in range(5):
        pos = {int(v): k for k, v in enumerate(idx[t])}
        assert pos[3] < pos[17] < pos[25]
        assert pos[17] == pos[3] + 1 and pos[25] == pos[3] + 2


def test_k_not_above_v():
    x = small_case(3, 8, 12, 4, seed=44)
    idx, lg = oracle.topk_cache(x["H"], x["W"], 50)
    assert idx.shape == (3, 12)
    assert sorted(idx[0].tolist()) == list(range(12))


def test_self_distillation_closed_form():
    x = small_case(6, 12, 80, 10, seed=45)
    for K in (10, 80):
        idx, lg = oracle.topk_cache(x["H"], x["W"], K)
        r = oracle.fwd_bwd(x["H"], x["W"], idx, lg)
        z = np.asarray(x["H"], np.float64) @ np.asarray(x["W"], np.float64).T
        q = np.exp(z - z.max(1, keepdims=True))
        q /= q.sum(1, keepdims=True)
        mass = np.take_along_axis(q, idx, 1).sum(1)
        np.testing.assert_allclose(r["ell"], -np.log(mass), rtol=1e-10, atol=1e-12)
        if K == 80:
            assert abs(r["loss"]) < 1e-12
