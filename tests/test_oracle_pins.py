"""Pins of the fp64 oracle against facts it does not compute itself.

The loss is the forward KL of "Chunked KL loss, running Knowledge Distillation
locally in less <6GB VRAM" (README formula section: one forward KL shared by
the three methods; the "Full Dense KL" method rebuilds a dense teacher from the
cache and is the README's reference for correctness). The author's forum post
says the loss equals PyTorch's KL divergence. Each test below pins the oracle to
one of:
  * a dense reconstruction written separately (the pages' own baseline),
  * PyTorch's kl_div / cross_entropy with autograd gradients (fp64),
  * closed forms (K = 1, W = 0, a two-token vocabulary),
  * central finite differences,
  * invariants of the definition (non-negativity, zero at self-distillation,
    shift and permutation invariance, gradient rows summing to zero, masking).
The last test plants mistakes in the oracle and checks that these pins catch them.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import ckl_oracle as O
from chunked_kl_loss_logits_b200.workloads import small_case

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def case(T=6, d=8, V=40, K=5, seed=0, mask=False, var=2.0):
    x = small_case(T, d, V, K, seed, teacher_var=var)
    rng = np.random.default_rng(seed + 99)
    if mask:
        x["mask"] = (rng.random(T) > 0.3).astype(np.uint8)
        x["mask"][0] = 1
    return x


def dense_teacher(idx, logit, V):
    """p scattered into a length-V vector per token (repeated ids add)."""
    T, K = idx.shape
    lg = np.asarray(logit, np.float64)
    mx = lg.max(1, keepdims=True)
    e = np.exp(lg - mx)
    p = e / e.sum(1, keepdims=True)
    P = np.zeros((T, V))
    for t in range(T):
        for k in range(K):
            P[t, idx[t, k]] += p[t, k]
    return P


def dense_kl(H, W, idx, logit, mask=None):
    """Dense forward KL: sum_v P_v (log P_v - log_softmax(z)_v), mean over unmasked tokens."""
    z = np.asarray(H, np.float64) @ np.asarray(W, np.float64).T
    m = z.max(1, keepdims=True)
    logq = z - (m + np.log(np.exp(z - m).sum(1, keepdims=True)))
    P = dense_teacher(idx, logit, W.shape[0])
    kl = np.array([sum(P[t, v] * (np.log(P[t, v]) - logq[t, v])
                       for v in range(W.shape[0]) if P[t, v] > 0) for t in range(H.shape[0])])
    msk = np.ones(H.shape[0]) if mask is None else np.asarray(mask, np.float64)
    return (msk * kl).sum() / msk.sum(), kl


def torch_kl(H, W, idx, logit, mask=None):
    """PyTorch fp64 kl_div on the dense teacher, gradients by autograd."""
    Ht = torch.tensor(np.asarray(H, np.float64), requires_grad=True)
    Wt = torch.tensor(np.asarray(W, np.float64), requires_grad=True)
    P = torch.tensor(dense_teacher(idx, logit, W.shape[0]))
    logq = torch.log_softmax(Ht @ Wt.T, dim=1)
    kl = torch.nn.functional.kl_div(logq, P, reduction="none").sum(1)
    msk = torch.ones(H.shape[0], dtype=torch.float64) if mask is None else \
        torch.tensor(np.asarray(mask, np.float64))
    loss = (msk * kl).sum() / msk.sum()
    loss.backward()
    return loss.item(), Ht.grad.numpy(), Wt.grad.numpy()


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


# ----------------------------------------------------------------------------- pins

@pytest.mark.parametrize("seed,mask", [(0, False), (1, True), (2, False)])
def test_dense_reconstruction(seed, mask):
    x = case(seed=seed, mask=mask)
    r = oracle.fwd_bwd(x["H"], x["W"], x["idx"], x["logit"], x["mask"])
    L, kl = dense_kl(x["H"], x["W"], x["idx"], x["logit"], x["mask"])
    assert abs(r["loss"] - L) <= 1e-12 * abs(L)
    np.testing.assert_allclose(r["ell"], kl, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("seed,mask", [(3, False), (4, True)])
def test_torch_kl_div_autograd(seed, mask):
    x = case(T=7, d=12, V=50, K=6, seed=seed, mask=mask)
    r = oracle.fwd_bwd(x["H"], x["W"], x["idx"], x["logit"], x["mask"])
    L, dH, dW = torch_kl(x["H"], x["W"], x["idx"], x["logit"], x["mask"])
    assert abs(r["loss"] - L) <= 1e-12 * abs(L)
    assert rel(r["dH"], dH) <= 1e-11
    assert rel(r["dW"], dW) <= 1e-11


def test_k1_is_cross_entropy():
    x = case(T=9, d=10, V=30, K=1, seed=5)
    r = oracle.fwd_bwd(x["H"], x["W"], x["idx"], x["logit"])
    z = torch.tensor(np.asarray(x["H"], np.float64) @ np.asarray(x["W"], np.float64).T)
    ce = torch.nn.functional.cross_entropy(z, torch.tensor(x["idx"][:, 0], dtype=torch.long))
    assert abs(r["loss"] - ce.item()) <= 1e-12 * ce.item()


def test_zero_weights_closed_form():
    x = case(T=5, d=6, V=20, K=4, seed=6)
    W = np.zeros_like(x["W"])
    r = oracle.fwd_bwd(x["H"], W, x["idx"], x["logit"])
    V = W.shape[0]
    lg = np.asarray(x["logit"], np.float64)
    p = np.exp(lg - lg.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    ent = (p * np.log(p)).sum(1)
    assert abs(r["loss"] - np.mean(ent + np.log(V))) <= 1e-13
    assert np.abs(r["dH"]).max() == 0.0
    T = x["H"].shape[0]
    P = dense_teacher(x["idx"], x["logit"], V)
    dW = ((1.0 / V - P).T @ np.asarray(x["H"], np.float64)) / T
    assert rel(r["dW"], dW) <= 1e-13


def test_two_word_vocabulary_closed_form():
    # V = 2, d = 1, one token, teacher all on word 0: loss = log(1 + exp((b - a) h)),
    # d/dh = q1 (b - a), d/da = -q1 h, d/db = q1 h with q1 = sigmoid((b - a) h).
    h, a, b = 0.7, 1.3, -0.4
    H = np.array([[h]])
    W = np.array([[a], [b]])
    r = oracle.fwd_bwd(H, W, np.array([[0]]), np.array([[0.25]]))
    q1 = 1.0 / (1.0 + np.exp(-(b - a) * h))
    assert abs(r["loss"] - np.log1p(np.exp((b - a) * h))) <= 1e-15
    assert abs(r["dH"][0, 0] - q1 * (b - a)) <= 1e-15
    np.testing.assert_allclose(r["dW"][:, 0], [-q1 * h, q1 * h], rtol=0, atol=1e-15)


def test_finite_differences():
    x = case(T=4, d=8, V=32, K=4, seed=7, mask=True)
    H = np.asarray(x["H"], np.float64)
    W = np.asarray(x["W"], np.float64)
    r = oracle.fwd_bwd(H, W, x["idx"], x["logit"], x["mask"])
    f = lambda H_, W_: oracle.fwd_bwd(H_, W_, x["idx"], x["logit"], x["mask"])["loss"]
    h = 1e-6
    num_dH = np.zeros_like(H)
    for i in np.ndindex(H.shape):
        Hp, Hm = H.copy(), H.copy()
        Hp[i] += h
        Hm[i] -= h
        num_dH[i] = (f(Hp, W) - f(Hm, W)) / (2 * h)
    num_dW = np.zeros_like(W)
    for i in np.ndindex(W.shape):
        Wp, Wm = W.copy(), W.copy()
        Wp[i] += h
        Wm[i] -= h
        num_dW[i] = (f(H, Wp) - f(H, Wm)) / (2 * h)
    assert rel(r["dH"], num_dH) <= 1e-7
    assert rel(r["dW"], num_dW) <= 1e-7


def test_loss_nonnegative():
    for seed in range(10):
        x = case(T=8, d=6, V=25, K=7, seed=100 + seed, var=8.0)
        r = oracle.fwd_bwd(x["H"], x["W"], x["idx"], x["logit"])
        assert r["loss"] >= 0.0
        assert np.all(r["ell"] >= -1e-12)


def test_self_distillation_is_zero():
    # K = V and the cached logits are the student's own logits (plus a constant):
    # the teacher equals the student, so the loss and every gradient vanish.
    T, d, V = 5, 7, 16
    x = case(T=T, d=d, V=V, K=4, seed=8)
    rng = np.random.default_rng(8)
    idx = np.stack([rng.permutation(V) for _ in range(T)]).astype(np.int32)
    z = np.asarray(x["H"], np.float64) @ np.asarray(x["W"], np.float64).T
    logit = np.take_along_axis(z, idx, 1) + 3.0
    r = oracle.fwd_bwd(x["H"], x["W"], idx, logit)
    assert abs(r["loss"]) <= 1e-12
    assert np.abs(r["dH"]).max() <= 1e-12
    assert np.abs(r["dW"]).max() <= 1e-12


def test_gradient_rows_sum_to_zero():
    x = case(T=6, d=9, V=40, K=5, seed=9, mask=True)
    r = oracle.fwd_bwd(x["H"], x["W"], x["idx"], x["logit"], x["mask"])
    # sum_v G_tv = M - sum p = 0, hence sum_v dW[v] = 0 column-wise.
    assert np.abs(r["dW"].sum(0)).max() <= 1e-14
    # dH_t = (mask_t/N) (softmax - p) W, and its row sum is that times W 1.
    W = np.asarray(x["W"], np.float64)
    z = np.asarray(x["H"], np.float64) @ W.T
    q = np.exp(z - z.max(1, keepdims=True))
    q /= q.sum(1, keepdims=True)
    P = dense_teacher(x["idx"], x["logit"], W.shape[0])
    s = x["mask"] / x["mask"].sum()
    np.testing.assert_allclose(r["dH"].sum(1), s * ((q - P) @ W.sum(1)), rtol=1e-11, atol=1e-15)


def test_invariances():
    x = case(T=6, d=5, V=30, K=6, seed=10)
    base = oracle.fwd_bwd(x["H"], x["W"], x["idx"], x["logit"])
    # teacher logits shifted by a constant per token
    sh = oracle.fwd_bwd(x["H"], x["W"], x["idx"], x["logit"] + np.arange(6)[:, None] * 1.5)
    assert abs(sh["loss"] - base["loss"]) <= 1e-12
    # the same vector added to every row of W shifts all logits of a token equally
    c = np.random.default_rng(10).standard_normal(5)
    W2 = np.asarray(x["W"], np.float64) + c
    sw = oracle.fwd_bwd(x["H"], W2, x["idx"], x["logit"])
    assert abs(sw["loss"] - base["loss"]) <= 1e-12
    # permuting the K slots of every token
    perm = np.random.default_rng(11).permutation(6)
    sp = oracle.fwd_bwd(x["H"], x["W"], x["idx"][:, perm], x["logit"][:, perm])
    assert abs(sp["loss"] - base["loss"]) <= 1e-13
    assert rel(sp["dH"], base["dH"]) <= 1e-13 and rel(sp["dW"], base["dW"]) <= 1e-13


def test_mask_equals_subbatch():
    x = case(T=9, d=6, V=30, K=5, seed=12, mask=True)
    r = oracle.fwd_bwd(x["H"], x["W"], x["idx"], x["logit"], x["mask"])
    keep = x["mask"].astype(bool)
    s = oracle.fwd_bwd(x["H"][keep], x["W"], x["idx"][keep], x["logit"][keep])
    assert abs(r["loss"] - s["loss"]) <= 1e-13
    assert rel(r["dW"], s["dW"]) <= 1e-13
    assert rel(r["dH"][keep], s["dH"]) <= 1e-13
    assert np.abs(r["dH"][~keep]).max() == 0.0
    z = oracle.fwd_bwd(x["H"], x["W"], x["idx"], x["logit"], np.zeros(9, np.uint8))
    assert z["loss"] == 0.0 and np.abs(z["dH"]).max() == 0.0 and np.abs(z["dW"]).max() == 0.0


def test_neg_inf_logits_drop_entries():
    x = case(T=4, d=6, V=30, K=6, seed=13)
    lg = x["logit"].copy()
    lg[:, 4:] = -np.inf
    r = oracle.fwd_bwd(x["H"], x["W"], x["idx"], lg)
    s = oracle.fwd_bwd(x["H"], x["W"], x["idx"][:, :4], x["logit"][:, :4])
    assert abs(r["loss"] - s["loss"]) <= 1e-13
    assert rel(r["dH"], s["dH"]) <= 1e-13 and rel(r["dW"], s["dW"]) <= 1e-13
    # a token whose whole cache is -inf contributes zero loss and zero gradient
    lg[0, :] = -np.inf
    r0 = oracle.fwd_bwd(x["H"], x["W"], x["idx"], lg)
    assert r0["ell"][0] == 0.0 and np.abs(r0["dH"][0]).max() == 0.0


def test_duplicate_ids_are_additive():
    x = case(T=5, d=6, V=20, K=5, seed=14)
    idx = x["idx"].copy()
    idx[:, 3] = idx[:, 1]
    r = oracle.fwd_bwd(x["H"], x["W"], idx, x["logit"])
    L, kl = dense_kl(x["H"], x["W"], idx, x["logit"])
    assert abs(r["loss"] - L) <= 1e-12 * abs(L)
    tl, tdH, tdW = torch_kl(x["H"], x["W"], idx, x["logit"])
    assert rel(r["dH"], tdH) <= 1e-11 and rel(r["dW"], tdW) <= 1e-11


def test_sampled_rows_match_full():
    x = case(T=12, d=7, V=45, K=5, seed=15, mask=True)
    r = oracle.fwd_bwd(x["H"], x["W"], x["idx"], x["logit"], x["mask"])
    rows = np.array([0, 3, 4, 11])
    s = oracle.sampled_rows(x["H"], x["W"], x["idx"], x["logit"], rows, x["mask"], with_dW=True)
    np.testing.assert_allclose(s["lse"], r["lse"][rows], rtol=1e-14)
    np.testing.assert_allclose(s["ell"], r["ell"][rows], rtol=1e-14)
    assert rel(s["dH"], r["dH"][rows]) <= 1e-14
    # the dW shares of all tokens add up to dW
    s_all = oracle.sampled_rows(x["H"], x["W"], x["idx"], x["logit"], np.arange(12), x["mask"],
                                with_dW=True)
    assert rel(s_all["dW_part"], r["dW"]) <= 1e-14


def test_dW_rows_match_full():
    # sampled dW rows over all tokens equal the full computation's rows, and the
    # blockwise log-normaliser equals the one over the whole row (several W blocks)
    x = case(T=40, d=6, V=9000, K=5, seed=16, mask=True)
    x["idx"][3, 2] = x["idx"][3, 0]  # a repeated id
    r = oracle.fwd_bwd(x["H"], x["W"], x["idx"], x["logit"], x["mask"])
    vrows = np.array([0, int(x["idx"][3, 0]), 4095, 4096, 8999])
    dW, lse = oracle.dW_rows(x["H"], x["W"], x["idx"], x["logit"], vrows, x["mask"])
    np.testing.assert_allclose(lse, r["lse"], rtol=1e-14)
    assert rel(dW, r["dW"][vrows]) <= 1e-13


def test_golden_fixture():
    with open(os.path.join(GOLDEN, "tiny_case.json")) as f:
        g = json.load(f)
    inp = {k: np.array(v) for k, v in g["inputs"].items()}
    r = oracle.fwd_bwd(inp["H"], inp["W"], inp["idx"].astype(np.int32), inp["logit"], inp["mask"])
    assert abs(r["loss"] - g["loss"]) <= 1e-13 * abs(g["loss"])
    assert rel(r["dH"], np.array(g["dH"])) <= 1e-13
    assert rel(r["dW"], np.array(g["dW"])) <= 1e-13


# ----------------------------------------------------------- planted mistakes

def _mut_drop_lse(z, idx, p, M):
    ell, lse = _orig_token_loss(z, idx, p, M)
    return ell - M * lse, lse


def _mut_cross_sign(z, idx, p, M):
    ell, lse = _orig_token_loss(z, idx, p, M)
    zk = np.take_along_axis(z, np.asarray(idx, np.int64), 1)
    return ell + 2 * (p * zk).sum(1), lse


def _mut_grad_no_p(z, lse, idx, p, M):
    return M[:, None] * np.exp(z - lse[:, None])


def _mut_grad_shift_idx(z, lse, idx, p, M):
    return _orig_grad_logits(z, lse, (np.asarray(idx) + 1) % z.shape[1], p, M)


def _mut_student_transposed(H_rows, W):
    z = _orig_student_logits(H_rows, W)
    return z[:, ::-1].copy()


def _mut_unpooled(idx, p):
    return np.asarray(p, dtype=np.float64).copy()  # a repeated id keeps only its own slot


def _mut_mask_ignored(mask, T):
    return _orig_token_scale(None, T)


_orig_token_loss = O.token_loss
_orig_grad_logits = O.grad_logits
_orig_student_logits = O.student_logits
_orig_token_scale = O.token_scale


PLANTED = [("token_loss", _mut_drop_lse), ("token_loss", _mut_cross_sign),
           ("grad_logits", _mut_grad_no_p), ("grad_logits", _mut_grad_shift_idx),
           ("student_logits", _mut_student_transposed), ("merged_probs", _mut_unpooled),
           ("token_scale", _mut_mask_ignored)]


@pytest.mark.parametrize("name,fn", PLANTED)
def test_brute_force_pin_catches_every_planted_mistake(monkeypatch, name, fn):
    monkeypatch.setattr(O, name, fn)
    with pytest.raises(AssertionError):
        test_brute_force_loops()


@pytest.mark.parametrize("name,fn", PLANTED[:5])
def test_pins_catch_planted_mistakes(monkeypatch, name, fn):
    monkeypatch.setattr(O, name, fn)
    pins = [lambda: test_dense_reconstruction(1, True), lambda: test_torch_kl_div_autograd(3, False),
            test_finite_differences, test_gradient_rows_sum_to_zero, test_brute_force_loops]
    failed = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed >= 1


def _brute_force(H, W, idx, logit, mask):
    """The definition written out with Python floats and loops only (no NumPy, no
    BLAS): per token, z = H_t . W_v for every v, lse, p = softmax of the cached
    logits (-inf -> 0), P = p pooled per id, l_t = sum_k p_k log P_{id_k} -
    sum_k p_k z_{id_k} + M lse; loss = mean over unmasked tokens; G = (mask/N)(M
    softmax(z) - P); dH = G W; dW = G^T H."""
    import math
    T, d, V, K = len(H), len(H[0]), len(W), len(idx[0])
    N = sum(1 for t in range(T) if mask[t])
    loss, ell, lse_all = 0.0, [], []
    dH = [[0.0] * d for _ in range(T)]
    dW = [[0.0] * d for _ in range(V)]
    for t in range(T):
        z = [sum(H[t][j] * W[v][j] for j in range(d)) for v in range(V)]
        m = max(z)
        lse = m + math.log(sum(math.exp(zv - m) for zv in z))
        lm = max(logit[t])
        if lm == -math.inf:
            p = [0.0] * K
        else:
            e = [0.0 if l == -math.inf else math.exp(l - lm) for l in logit[t]]
            p = [x / sum(e) for x in e]
        P = {}
        for k in range(K):
            P[idx[t][k]] = P.get(idx[t][k], 0.0) + p[k]
        M = sum(p)
        l_t = sum(p[k] * math.log(P[idx[t][k]]) for k in range(K) if p[k] > 0)
        l_t -= sum(p[k] * z[idx[t][k]] for k in range(K))
        l_t += M * lse
        ell.append(l_t)
        lse_all.append(lse)
        s = (1.0 / N) if (mask[t] and N) else 0.0
        loss += s * l_t
        for v in range(V):
            g = s * (M * math.exp(z[v] - lse) - P.get(v, 0.0))
            for j in range(d):
                dH[t][j] += g * W[v][j]
                dW[v][j] += g * H[t][j]
    return loss, ell, lse_all, dH, dW


def test_brute_force_loops():
    rng = np.random.default_rng(97)
    T, d, V, K = 5, 3, 7, 4
    H = rng.standard_normal((T, d))
    W = rng.standard_normal((V, d)) * 0.7
    idx = rng.integers(0, V, (T, K)).astype(np.int32)
    idx[1, 3] = idx[1, 0]            # a repeated id
    logit = rng.standard_normal((T, K)) * 1.5
    logit[2, 1] = -np.inf            # a dropped entry
    mask = np.array([1, 1, 0, 1, 1], dtype=np.uint8)
    bl, bell, blse, bdH, bdW = _brute_force(H.tolist(), W.tolist(), idx.tolist(),
                                            logit.tolist(), mask.tolist())
    r = oracle.fwd_bwd(H, W, idx, logit, mask)
    assert abs(r["loss"] - bl) <= 1e-12 * max(1.0, abs(bl))
    np.testing.assert_allclose(r["ell"], bell, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r["lse"], blse, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r["dH"], bdH, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(r["dW"], bdW, rtol=1e-11, atol=1e-13)
