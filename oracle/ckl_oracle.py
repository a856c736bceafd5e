"""fp64 CPU oracle of the fused top-K forward-KL distillation loss.

TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the CPU-baseline leg
of the benchmark may import or call this module; the library never does, and it
shares no code with the CUDA path.

What it computes follows "Chunked KL loss, running Knowledge Distillation locally
in less <6GB VRAM" (the README section stating that all three methods evaluate the
same forward KL against cached top-K teacher probabilities). For a token with
student logits z = H_t W^T over the whole vocabulary and a teacher support S (the
K cached ids), the per-token loss is

    l_t = sum_{v in S} p_v log p_v  -  sum_{v in S} p_v z_v  +  M * logsumexp(z)

with p the teacher probabilities on S and M = sum_{v in S} p_v. Only the
log-normaliser spans the vocabulary. The pages drop the definitions of S, p, M,
the closed-form gradient and the reduction (the extracted text is cut at those
formulas), so this module takes these readings:

  * p = softmax of the K cached teacher logits (the README and the forum post:
    the cache keeps each position's 100 largest teacher logits); M = sum p, i.e. 1 unless every cached
    logit is -inf, in which case p = 0, M = 0 and the token contributes nothing.
    A -inf logit gives p = 0 and 0 log 0 := 0.
  * Repeated ids within one token's K entries add their probabilities
    (scatter-add reading of the dense teacher that the README's "Full Dense KL"
    method rebuilds from the cache).
  * Temperature 1; no bias on the LM head.
  * The loss is the mean of l_t over unmasked tokens, N = sum(mask); if N = 0
    the loss and both gradients are 0.
  * Gradient: d l_t / d z_v = M softmax(z)_v - p_v (p_v = 0 off S), the closed
    form that follows from differentiating l_t (the README's equation itself is
    lost in extraction). dH = (mask/N) G W and dW = sum_t (mask_t/N) G_t^T H_t,
    the chain rule through z = H W^T.

Everything is evaluated in float64 from the exact input values (bf16 inputs are
widened exactly). The matrix products are numpy matmuls (a library primitive);
products over the vocabulary are taken in row blocks of W only to bound host
memory, which changes nothing but the rounding order of fp64 sums.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64
_VBLOCK = 16384  # vocabulary rows of W widened to fp64 at a time


def teacher_probs(logit):
    """p (R, K) = softmax over each row of cached teacher logits; M (R,) = sum p.

    Rows whose logits are all -inf get p = 0 and M = 0.
    """
    logit = np.asarray(logit, dtype=F64)
    mx = logit.max(axis=1, keepdims=True)
    live = np.isfinite(mx)
    e = np.exp(logit - np.where(live, mx, 0.0))
    e = np.where(live, e, 0.0)
    s = e.sum(axis=1, keepdims=True)
    p = np.divide(e, s, out=np.zeros_like(e), where=s > 0)
    return p, p.sum(axis=1)


def student_logits(H_rows, W):
    """z (R, V) = H_rows W^T in float64."""
    H_rows = np.asarray(H_rows, dtype=F64)
    V = W.shape[0]
    z = np.empty((H_rows.shape[0], V), dtype=F64)
    for v0 in range(0, V, _VBLOCK):
        v1 = min(V, v0 + _VBLOCK)
        z[:, v0:v1] = H_rows @ np.asarray(W[v0:v1], dtype=F64).T
    return z


def logsumexp(z):
    """log sum_v exp(z_v) per row, shifted by the row maximum."""
    m = z.max(axis=1)
    return m + np.log(np.exp(z - m[:, None]).sum(axis=1))


def merged_probs(idx, p):
    """P (R, K): for each slot, the total teacher probability of its id.

    The README's sums run over the support S, a set of vocabulary ids; when an id
    is cached in several slots its probability is the sum over those slots. With
    distinct ids P = p.
    """
    idx = np.asarray(idx, dtype=np.int64)
    same = idx[:, :, None] == idx[:, None, :]
    return (same * p[:, None, :]).sum(axis=2)


def token_loss(z, idx, p, M):
    """Per-token loss l_t and log-normaliser lse_t from the full-vocabulary logits.

    sum_{v in S} P_v log P_v is taken as sum_k p_k log P_k (P_k = merged_probs),
    which groups the slots of each distinct id.
    """
    P = merged_probs(idx, p)
    ent = np.where(p > 0, p * np.log(np.where(p > 0, P, 1.0)), 0.0).sum(axis=1)
    zk = np.take_along_axis(z, np.asarray(idx, dtype=np.int64), axis=1)
    cross = np.where(p > 0, p * zk, 0.0).sum(axis=1)
    lse = logsumexp(z)
    return ent - cross + M * lse, lse


def grad_logits(z, lse, idx, p, M):
    """G (R, V) = M softmax(z) - p scattered onto the cached ids (repeated ids add)."""
    G = M[:, None] * np.exp(z - lse[:, None])
    rows = np.repeat(np.arange(z.shape[0]), idx.shape[1])
    np.add.at(G, (rows, np.asarray(idx, dtype=np.int64).ravel()), -p.ravel())
    return G


def token_scale(mask, T):
    """mask_t / N with N = sum(mask); all zeros when N = 0. Also returns N."""
    m = np.ones(T, dtype=F64) if mask is None else np.asarray(mask, dtype=F64)
    N = m.sum()
    return (m / N if N > 0 else np.zeros(T, dtype=F64)), N


def fwd_bwd(H, W, idx, logit, mask=None):
    """Mean loss, dH (T, d), dW (V, d), per-token lse and l over all tokens (small sizes).

    Returns a dict with float64 arrays.
    """
    T = H.shape[0]
    p, M = teacher_probs(logit)
    z = student_logits(H, W)
    ell, lse = token_loss(z, idx, p, M)
    s, N = token_scale(mask, T)
    loss = float((s * ell).sum())
    Gs = s[:, None] * grad_logits(z, lse, idx, p, M)
    W64 = np.asarray(W, dtype=F64)
    dH = Gs @ W64
    dW = Gs.T @ np.asarray(H, dtype=F64)
    return {"loss": loss, "dH": dH, "dW": dW, "lse": lse, "ell": ell, "N": N}


def sampled_rows(H, W, idx, logit, rows, mask=None, with_dW=False):
    """lse, l and dH for the token positions `rows` only (optionally their dW share).

    N comes from the full mask, so dH rows equal those of the full computation.
    Costs O(len(rows) * V * d); this is how the 32K-256K workloads are checked.
    With `with_dW`, also returns dW_part = sum over the sampled tokens of their
    rank-1 contributions (mask_t/N) G_t^T H_t, so that the whole per-token path is
    done for each sampled token (this is what the CPU baseline times).
    """
    rows = np.asarray(rows, dtype=np.int64)
    T = H.shape[0]
    s_all, N = token_scale(mask, T)
    s = s_all[rows]
    p, M = teacher_probs(np.asarray(logit)[rows])
    Hr = np.asarray(H)[rows]
    z = student_logits(Hr, W)
    ir = np.asarray(idx)[rows]
    ell, lse = token_loss(z, ir, p, M)
    Gs = s[:, None] * grad_logits(z, lse, ir, p, M)
    V = W.shape[0]
    dH = np.zeros((rows.size, W.shape[1]), dtype=F64)
    for v0 in range(0, V, _VBLOCK):
        v1 = min(V, v0 + _VBLOCK)
        dH += Gs[:, v0:v1] @ np.asarray(W[v0:v1], dtype=F64)
    out = {"lse": lse, "ell": ell, "dH": dH, "N": N}
    if with_dW:
        out["dW_part"] = Gs.T @ np.asarray(Hr, dtype=F64)
    return out


def dW_rows(H, W, idx, logit, vrows, mask=None):
    """dW rows of the vocabulary ids `vrows`, and lse of every token (large sizes).

    dW[v] = sum_t (mask_t/N) G_tv H_t with G_tv = M_t softmax(z_t)_v - P_tv (the
    closed-form gradient of the README formula, as in fwd_bwd). Every token's
    log-normaliser enters, so lse_t is taken over the whole vocabulary first: the
    log-sum-exp of the log-sum-exps of blocks of W's rows (the same quantity as
    logsumexp over all of z_t, summed in another order); G is then formed at the
    sampled columns only. Costs O(T V d) multiply-adds and O(T) memory per block.
    Returns (dW rows (len(vrows), d), lse (T,)).
    """
    H64 = np.asarray(H, dtype=F64)
    T, V = H64.shape[0], W.shape[0]
    block = _VBLOCK // 4
    lse_b = []
    for v0 in range(0, V, block):
        lse_b.append(logsumexp(H64 @ np.asarray(W[v0:min(V, v0 + block)], dtype=F64).T))
    lse = np.logaddexp.reduce(np.stack(lse_b, axis=1), axis=1)
    vrows = np.asarray(vrows, dtype=np.int64)
    p, M = teacher_probs(logit)
    ids = np.asarray(idx, dtype=np.int64)
    zv = H64 @ np.asarray(W[vrows], dtype=F64).T                      # T x n
    Pv = np.stack([np.where(ids == v, p, 0.0).sum(axis=1) for v in vrows], axis=1)
    G = M[:, None] * np.exp(zv - lse[:, None]) - Pv
    s, _ = token_scale(mask, T)
    return (s[:, None] * G).T @ H64, lse


def topk_cache(H, W, K):
    """Teacher top-K cache: per token, the K largest logits of z = H W^T and their ids.

    The offline distillation of "Efficient Knowledge Distillation for LLMs:
    Offline Top-K Logits and a Fused Chunked KL Loss" (abstract) and the author's
    forum post: the teacher's forward pass runs once and each position keeps only
    its largest logits (100 of them), which the loss above then reads. Order:
    descending logit; equal logits in ascending id order. Returns (idx int64
    (T, K), logit float64 (T, K)). Computed in float64 from the exact inputs.
    """
    z = student_logits(H, W)
    T, V = z.shape
    K = min(K, V)
    ids = np.broadcast_to(np.arange(V), z.shape)
    order = np.lexsort((ids, -z), axis=1)[:, :K]   # primary key -z, then id
    return order.astype(np.int64), np.take_along_axis(z, order, axis=1)
