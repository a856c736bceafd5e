"""GPU teacher top-K cache builder vs the fp64 oracle, through the C ABI.

Where the K-th and (K+1)-th logits of a row are separated by more than the
fp32-accumulation error, the ids must equal the oracle's exactly (index work);
elsewhere the selected set must be a valid top-K (every selected logit at least
as large as every unselected one, up to that error) and the logits must equal
the oracle's at the selected ids within the error. Constant logits and tied
rows check the id tie-break exactly.
"""
import numpy as np
import pytest
import torch

import oracle
from chunked_kl_loss_logits_b200 import ckl
from chunked_kl_loss_logits_b200.workloads import WORKLOADS, make_inputs, small_case, sample_rows

pytestmark = pytest.mark.gpu

TOL = 1e-4  # absolute, on O(1) logits accumulated in fp32 from bf16 inputs


def check_rows(ids, logits, H, W, K, rows=None):
    """ids/logits: GPU result rows (host numpy); H, W: the exact inputs (host)."""
    rows = np.arange(ids.shape[0]) if rows is None else rows
    z = np.asarray(H, np.float64)[rows] @ np.asarray(W, np.float64).T
    o_idx, o_lg = oracle.topk_cache(np.asarray(H)[rows], W, K + 1)
    exact_rows = 0
    for r in range(len(rows)):
        gi, gl = ids[r], logits[r]
        assert len(set(gi.tolist())) == K and gi.min() >= 0 and gi.max() < W.shape[0]
        assert np.all(np.diff(gl) <= 0)                         # descending
        np.testing.assert_allclose(gl, z[r, gi], rtol=0, atol=TOL)  # logits at the ids
        kth = o_lg[r, K - 1]
        assert z[r, gi].min() >= kth - TOL                        # a valid top-K
        if o_lg[r, K - 1] - o_lg[r, K] > 2 * TOL:                 # unique top-K: ids exact
            assert np.array_equal(gi, o_idx[r, :K]) or \
                np.array_equal(np.sort(gi), np.sort(o_idx[r, :K]))
            exact_rows += 1
    return exact_rows


def run(x, K, chunk):
    T, d = x["H"].shape
    V = x["W"].shape[0]
    H = torch.from_numpy(x["H"]).cuda().to(torch.bfloat16)
    W = torch.from_numpy(x["W"]).cuda().to(torch.bfloat16)
    h = ckl.ChunkedKL(V, d, K, max_chunk=chunk)
    ids, lg = h.topk_cache(H, W, chunk=chunk)
    return ids.cpu().numpy(), lg.cpu().numpy()


@pytest.mark.parametrize("T,d,V,K,chunk", [
    (300, 128, 3000, 16, 128),    # ragged tokens and vocabulary, 12 tiles <= K: take-all path
    (257, 64, 20000, 20, 100),    # 79 tiles > K: threshold path
    (64, 2880, 50000, 100, 64),   # the headline hidden size and K
])
def test_cache_matches_oracle(T, d, V, K, chunk):
    x = small_case(T, d, V, K, seed=T + V, dtype="bf16")
    ids, lg = run(x, K, chunk)
    exact = check_rows(ids, lg, x["H"], x["W"], K)
    assert exact >= T // 2


def test_constant_logits_take_the_smallest_ids():
    x = small_case(40, 64, 5000, 12, seed=7, dtype="bf16")
    x["W"] = np.zeros_like(x["W"])
    ids, lg = run(x, 12, 32)
    assert np.array_equal(ids, np.tile(np.arange(12, dtype=np.int32), (40, 1)))
    assert np.all(lg == 0.0)


def test_ties_break_by_id():
    x = small_case(50, 64, 4000, 30, seed=8, dtype="bf16")
    W = x["W"].copy()
    z = np.asarray(x["H"], np.float64) @ W.T.astype(np.float64)
    top = int(np.argmax(z[0]))
    for dup in (3000, 1234, 3999):
        W[dup] = W[top]
    x["W"] = W
    ids, lg = run(x, 30, 64)
    pos = {int(v): k for k, v in enumerate(ids[0])}
    group = sorted([top, 1234, 3000, 3999])
    assert all(g in pos for g in group)
    assert [pos[g] for g in group] == list(range(pos[group[0]], pos[group[0]] + 4))


def test_headline_teacher_shape_sampled():
    w = WORKLOADS["bf16_32k"]
    x = make_inputs(w, T=2048)
    ids, lg = run(x, w.K, 2048)
    rows = sample_rows(2048, 48, seed=9)
    exact = check_rows(ids[rows], lg[rows], x["H"], x["W"], w.K, rows=rows)
    assert exact >= len(rows) // 2


def test_cache_feeds_the_loss():
    # a student distilled from a cache built from itself: loss = -log(top-K mass)
    x = small_case(200, 128, 6000, 32, seed=10, dtype="bf16")
    H = torch.from_numpy(x["H"]).cuda().to(torch.bfloat16)
    W = torch.from_numpy(x["W"]).cuda().to(torch.bfloat16)
    h = ckl.ChunkedKL(6000, 128, 32, max_chunk=128)
    ids, lg = h.topk_cache(H, W, chunk=128)
    loss, lse, ell = h.forward(H, W, ids, lg, chunk=128, token_stats=True)
    z = np.asarray(x["H"], np.float64) @ np.asarray(x["W"], np.float64).T
    q = np.exp(z - z.max(1, keepdims=True))
    q /= q.sum(1, keepdims=True)
    mass = np.take_along_axis(q, ids.cpu().numpy().astype(np.int64), 1).sum(1)
    np.testing.assert_allclose(ell.cpu().numpy(), -np.log(mass), rtol=1e-4, atol=1e-5)


def test_k_equal_to_v_keeps_every_id_sorted():
    x = small_case(50, 64, 200, 20, seed=11, dtype="bf16")
    ids, lg = run(x, 200, 32)  # one vocabulary tile, K = V
    z = np.asarray(x["H"], np.float64) @ np.asarray(x["W"], np.float64).T
    for r in range(50):
        assert sorted(ids[r].tolist()) == list(range(200))
        assert np.all(np.diff(lg[r]) <= 0)
        np.testing.assert_allclose(lg[r], z[r, ids[r]], rtol=0, atol=TOL)


def test_cache_is_chunk_invariant():
    x = small_case(300, 128, 5000, 24, seed=12, dtype="bf16")
    a = run(x, 24, 300)
    for chunk in (1, 77, 128):
        b = run(x, 24, chunk)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def run_cache_group(x, K, chunk, world):
    """The cache built by `world` ranks (threads) holding vocab_shards of W."""
    import threading

    from tests.test_gpu_vocab_parallel import ThreadGroup
    T, d = x["H"].shape
    V = x["W"].shape[0]
    dev = torch.device("cuda", 0)
    H = torch.from_numpy(x["H"]).to(dev).to(torch.bfloat16)
    W = torch.from_numpy(x["W"]).to(dev).to(torch.bfloat16)
    torch.cuda.synchronize(dev)
    shards = ckl.vocab_shards(V, world)
    tg = ThreadGroup(world)
    out, errs = [None] * world, []

    def rank_main(r):
        try:
            torch.cuda.set_device(dev)
            v0, n = shards[r]
            h = ckl.ChunkedKL(n, d, K, max_chunk=chunk, device=dev)
            s = torch.cuda.Stream(dev)
            with torch.cuda.stream(s):
                W_r = W[v0:v0 + n].contiguous()
                s.synchronize()
                ids, lg = h.topk_cache_vocab_parallel(tg.member(r, V, v0), H, W_r, chunk=chunk)
                s.synchronize()
            out[r] = (ids.cpu(), lg.cpu())
            h.close()
        except Exception as e:
            errs.append(e)
            tg.barrier.abort()

    th = [threading.Thread(target=rank_main, args=(r,)) for r in range(world)]
    for t in th:
        t.start()
    for t in th:
        t.join(300)
    assert not errs, errs
    return out, tg


@pytest.mark.parametrize("world,T,d,V,K,chunk", [
    (2, 300, 128, 5000, 24, 128),
    (3, 257, 64, 5000, 24, 100),    # uneven shards (1792, 1792, 1416 rows)
])
def test_vocab_parallel_cache_equals_single_rank(world, T, d, V, K, chunk):
    x = small_case(T, d, V, K, seed=world + T, dtype="bf16")
    out, tg = run_cache_group(x, K, chunk, world)
    ref_ids, ref_lg = run(x, K, chunk)
    for ids, lg in out:
        assert np.array_equal(ids.numpy(), ref_ids) and np.array_equal(lg.numpy(), ref_lg)
    n_chunks = (T + chunk - 1) // chunk
    for calls in tg.calls:
        assert [c[0] for c in calls] == ["gather"] * n_chunks


def test_vocab_parallel_cache_headline_shape():
    w = WORKLOADS["bf16_32k"]
    x = make_inputs(w, T=512)
    out, _ = run_cache_group(x, w.K, 256, 2)
    ref_ids, ref_lg = run(x, w.K, 256)
    for ids, lg in out:
        assert np.array_equal(ids.numpy(), ref_ids) and np.array_equal(lg.numpy(), ref_lg)
