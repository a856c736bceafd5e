"""Vocabulary-parallel loss through the C ABI, against the fp64 oracle.

The ranks of a group run as threads of this process on one GPU, each with its
own handle and stream; the group's collectives meet on the host (each rank's
stream is synchronised before its buffer is shared and after the result is
written back), so no kernel ever waits for another. Checked: loss, dH, lse and
per-token loss identical bit for bit on every rank; loss, lse, dH and the
concatenated dW shards equal to the oracle within the bf16 tolerances; a group
of one equal to the single-rank call; a failing collective reported as
CKL_ERR_COLLECTIVE with no further collective called.
"""
import threading

import numpy as np
import pytest
import torch

import oracle
from chunked_kl_loss_logits_b200 import ckl
from chunked_kl_loss_logits_b200.workloads import small_case

pytestmark = pytest.mark.gpu


class ThreadGroup:
    """`world` ranks as threads; collectives exchange device tensors through the host side."""

    def __init__(self, world):
        self.world = world
        self.barrier = threading.Barrier(world, timeout=120)
        self.slots = [None] * world
        self.calls = [[] for _ in range(world)]

    def member(self, rank, V_total, v0):
        def all_gather(send, recv):
            self.calls[rank].append(("gather", send.numel()))
            torch.cuda.current_stream().synchronize()
            self.slots[rank] = send.clone()
            torch.cuda.current_stream().synchronize()
            self.barrier.wait()
            n = send.numel()
            for r in range(self.world):
                recv[r * n:(r + 1) * n].copy_(self.slots[r])
            torch.cuda.current_stream().synchronize()
            self.barrier.wait()

        def all_reduce_sum(buf):
            self.calls[rank].append(("reduce", buf.numel()))
            torch.cuda.current_stream().synchronize()
            self.slots[rank] = buf.clone()
            torch.cuda.current_stream().synchronize()
            self.barrier.wait()
            acc = self.slots[0].clone()
            for r in range(1, self.world):  # rank order: the same sum on every rank
                acc += self.slots[r]
            buf.copy_(acc)
            torch.cuda.current_stream().synchronize()
            self.barrier.wait()

        return ckl.VocabGroup(self.world, rank, V_total, v0, all_gather, all_reduce_sum)


def run_group(x, world, chunk, shards=None, forward_only=False):
    T, d = x["H"].shape
    V = x["W"].shape[0]
    K = x["idx"].shape[1]
    shards = shards or ckl.vocab_shards(V, world)
    dev = torch.device("cuda", 0)
    H = torch.from_numpy(x["H"]).to(dev).to(torch.bfloat16)
    W = torch.from_numpy(x["W"]).to(dev).to(torch.bfloat16)
    idx = torch.from_numpy(x["idx"]).to(dev)
    lg = torch.from_numpy(x["logit"]).to(dev)
    mask = torch.from_numpy(x["mask"]).to(dev) if x.get("mask") is not None else None
    torch.cuda.synchronize(dev)  # inputs ready before the ranks' streams read them
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
                fn = h.forward_vocab_parallel if forward_only else h.fwd_bwd_vocab_parallel
                res = fn(tg.member(r, V, v0), H, W_r, idx, lg, mask, chunk=chunk,
                         token_stats=True)
                s.synchronize()
            out[r] = [t.cpu() for t in res]
            h.close()
        except Exception as e:  # surfaced by the test
            errs.append(e)
            tg.barrier.abort()

    th = [threading.Thread(target=rank_main, args=(r,)) for r in range(world)]
    for t in th:
        t.start()
    for t in th:
        t.join(300)
    assert not errs, errs
    return out, tg, shards


def check_against_oracle(x, out, shards):
    r = oracle.fwd_bwd(x["H"], x["W"], x["idx"], x["logit"], x.get("mask"))
    loss, dH, _, lse, ell = out[0]
    for o in out[1:]:  # identical on every rank
        for a, b in ((loss, o[0]), (dH, o[1]), (lse, o[3]), (ell, o[4])):
            assert torch.equal(a, b)
    assert abs(float(loss) - r["loss"]) <= 1e-3 * max(1.0, abs(r["loss"]))
    np.testing.assert_allclose(lse.numpy(), r["lse"], rtol=0, atol=2e-6 * np.abs(r["lse"]).max() + 1e-5)
    scale = np.abs(r["dH"]).max()
    assert np.abs(dH.float().numpy() - r["dH"]).max() <= 1e-2 * scale
    dW = torch.cat([o[2] for o in out]).numpy()
    assert dW.shape == r["dW"].shape
    assert np.abs(dW - r["dW"]).max() <= 1e-2 * np.abs(r["dW"]).max()


@pytest.mark.parametrize("world,T,d,V,K,chunk", [
    (2, 300, 128, 3000, 16, 128),    # two shards, ragged chunks
    (3, 257, 64, 1000, 12, 100),     # uneven shards (512, 256, 232 rows)
    (4, 129, 2880, 3001, 100, 129),  # the headline hidden size and K
])
def test_group_matches_oracle(world, T, d, V, K, chunk):
    x = small_case(T, d, V, K, seed=world * 100 + T, dtype="bf16", teacher_var=3.0, ids="zipf")
    out, tg, shards = run_group(x, world, chunk)
    check_against_oracle(x, out, shards)
    n_chunks = (T + chunk - 1) // chunk
    for calls in tg.calls:  # one gather and one reduce per chunk, the same on every rank
        assert [c[0] for c in calls] == ["gather", "reduce"] * n_chunks
    assert tg.calls[0] == tg.calls[-1]


def test_group_with_mask():
    x = small_case(300, 64, 1500, 16, seed=31, dtype="bf16", packing=True)
    out, _, shards = run_group(x, 2, 128)
    check_against_oracle(x, out, shards)


@pytest.mark.parametrize("rows", ["all", "half"])
def test_group_rows_far_above_their_reference(rows):
    # each rank keeps its exps against a reference logit of its own rows; hidden
    # states scaled 40x put the largest logits ~100 nats above it, so the ranks'
    # tiles fall back to their own maxima and those rows take the repair path
    # (and rows whose cached ids all lie on other ranks take it anyway)
    from chunked_kl_loss_logits_b200.workloads import round_to_bf16
    x = small_case(260, 64, 2600, 12, seed=37, dtype="bf16", teacher_var=3.0, ids="zipf")
    sel = slice(None) if rows == "all" else slice(1, None, 2)
    x["H"][sel] *= 40.0
    x["H"] = round_to_bf16(x["H"])
    out, _, shards = run_group(x, 3, 100)
    check_against_oracle(x, out, shards)


def test_group_of_one_equals_single_rank_call():
    x = small_case(200, 128, 2000, 16, seed=32, dtype="bf16")
    out, _, _ = run_group(x, 1, 64)
    dev = torch.device("cuda", 0)
    h = ckl.ChunkedKL(2000, 128, 16, max_chunk=64, device=dev)
    H = torch.from_numpy(x["H"]).to(dev).to(torch.bfloat16)
    W = torch.from_numpy(x["W"]).to(dev).to(torch.bfloat16)
    loss, dH, dW, lse, ell = h.fwd_bwd(H, W, torch.from_numpy(x["idx"]).to(dev),
                                       torch.from_numpy(x["logit"]).to(dev), chunk=64,
                                       token_stats=True)
    assert torch.equal(dH.cpu(), out[0][1]) and torch.equal(dW.cpu(), out[0][2])
    torch.testing.assert_close(lse.cpu(), out[0][3], rtol=1e-6, atol=1e-6)
    torch.testing.assert_close(loss.cpu(), out[0][0], rtol=1e-6, atol=1e-7)


def test_failing_collective_is_reported():
    x = small_case(100, 64, 500, 8, seed=33, dtype="bf16")
    dev = torch.device("cuda", 0)
    calls = []

    def bad_gather(send, recv):
        calls.append("gather")
        raise RuntimeError("peer lost")

    def reduce(buf):
        calls.append("reduce")

    g = ckl.VocabGroup(1, 0, 500, 0, bad_gather, reduce)
    h = ckl.ChunkedKL(500, 64, 8, max_chunk=32, device=dev)
    H = torch.from_numpy(x["H"]).to(dev).to(torch.bfloat16)
    W = torch.from_numpy(x["W"]).to(dev).to(torch.bfloat16)
    with pytest.raises(ckl.CKLError) as ei:
        h.fwd_bwd_vocab_parallel(g, H, W, torch.from_numpy(x["idx"]).to(dev),
                                 torch.from_numpy(x["logit"]).to(dev), chunk=32)
    assert ei.value.code == 9 and isinstance(ei.value.__cause__, RuntimeError)
    assert calls == ["gather"]  # no collective after the failed one
    torch.cuda.synchronize()


def test_ids_outside_the_full_vocabulary_are_reported():
    x = small_case(64, 64, 600, 8, seed=34, dtype="bf16")
    x["idx"][3, 2] = 600
    with pytest.raises(AssertionError) as ei:
        run_group(x, 2, 32)
    assert "top-K index out of range" in str(ei.value)


def test_group_in_recompute_mode():
    # the backward forms the logits again from the merged lse
    x = small_case(260, 64, 2000, 10, seed=35, dtype="bf16", teacher_var=3.0, ids="zipf")
    orig = ckl.ChunkedKL.fwd_bwd_vocab_parallel

    def with_recompute(self, *a, **k):
        self.set_recompute(True)
        return orig(self, *a, **k)

    ckl.ChunkedKL.fwd_bwd_vocab_parallel = with_recompute
    try:
        out, _, shards = run_group(x, 2, 100)
    finally:
        ckl.ChunkedKL.fwd_bwd_vocab_parallel = orig
    check_against_oracle(x, out, shards)


def test_group_ragged_k_and_chunks():
    x = small_case(77, 136, 1301, 7, seed=36, dtype="bf16")  # K % 4 != 0, d % 64 != 0
    out, _, shards = run_group(x, 3, 32)
    check_against_oracle(x, out, shards)


@pytest.mark.parametrize("bad", ["rank", "v0", "world", "callback", "f32"])
def test_group_arguments_are_checked(bad):
    import ctypes
    dev = torch.device("cuda", 0)
    V, d, K = 512, 64, 8
    dt = torch.float32 if bad == "f32" else torch.bfloat16
    h = ckl.ChunkedKL(V, d, K, dtype=dt, max_chunk=32, device=dev)
    calls = []
    g = ckl.VocabGroup(2, 0, 1024, 0, lambda s, r: calls.append(1), lambda b: calls.append(2))
    if bad == "rank":
        g.rank = 2
    elif bad == "v0":
        g.v0 = 600  # 600 + 512 > 1024
    elif bad == "world":
        g.world = 0
    H = torch.zeros((16, d), dtype=dt, device=dev)
    W = torch.zeros((V, d), dtype=dt, device=dev)
    idx = torch.zeros((16, K), dtype=torch.int32, device=dev)
    lg = torch.zeros((16, K), dtype=torch.float32, device=dev)
    if bad == "callback":
        c, keep = g._c(dev)
        c.all_gather = ckl._GatherFn()  # null function pointer
        n = ctypes.c_size_t()
        ckl.lib().ckl_vp_workspace_bytes(h._h, 2, 16, 32, ctypes.byref(n))
        ws = torch.empty(n.value, dtype=torch.uint8, device=dev)
        out = [torch.empty((), device=dev), torch.empty_like(H), torch.empty((V, d), device=dev)]
        code = ckl.lib().ckl_fwd_bwd_vocab_parallel(
            h._h, ctypes.byref(c), ckl._ptr(H), ckl._ptr(W), ckl._ptr(idx), ckl._ptr(lg), None, 16,
            32, ckl._ptr(out[0]), ckl._ptr(out[1]), ckl._ptr(out[2]), None, None, ckl._ptr(ws),
            ws.numel(), None, None)
        assert code == 1
    else:
        with pytest.raises(ckl.CKLError) as ei:
            h.fwd_bwd_vocab_parallel(g, H, W, idx, lg, chunk=32)
        assert ei.value.code == (2 if bad == "f32" else 1)
    assert calls == []  # argument errors come before any collective


def test_empty_input_makes_no_collective_call():
    dev = torch.device("cuda", 0)
    calls = []
    g = ckl.VocabGroup(1, 0, 512, 0, lambda s, r: calls.append(1), lambda b: calls.append(2))
    h = ckl.ChunkedKL(512, 64, 8, max_chunk=32, device=dev)
    H = torch.zeros((0, 64), dtype=torch.bfloat16, device=dev)
    W = torch.randn((512, 64), device=dev).to(torch.bfloat16)
    loss, dH, dW = h.fwd_bwd_vocab_parallel(g, H, W, torch.zeros((0, 8), dtype=torch.int32,
                                                                   device=dev),
                                            torch.zeros((0, 8), device=dev), chunk=32)
    assert calls == [] and float(loss) == 0.0 and torch.count_nonzero(dW) == 0


def test_forward_only_group():
    x = small_case(300, 128, 3000, 16, seed=37, dtype="bf16", teacher_var=3.0, ids="zipf",
                   packing=True)
    full, _, _ = run_group(x, 2, 128)
    fwd, tg, _ = run_group(x, 2, 128, forward_only=True)
    for r in range(2):
        loss, lse, ell = fwd[r]
        assert torch.equal(loss, full[r][0]) and torch.equal(lse, full[r][3])
        assert torch.equal(ell, full[r][4])
        assert [c[0] for c in tg.calls[r]] == ["gather"] * 3  # no all-reduce without a backward


def test_autograd_with_a_group_of_one():
    # the autograd wrapper routes through the vocabulary-parallel call
    dev = torch.device("cuda", 0)
    x = small_case(150, 64, 900, 8, seed=38, dtype="bf16")
    H = torch.from_numpy(x["H"]).to(dev).to(torch.bfloat16).requires_grad_(True)
    W = torch.from_numpy(x["W"]).to(dev).to(torch.bfloat16).requires_grad_(True)
    idx, lg = torch.from_numpy(x["idx"]).to(dev), torch.from_numpy(x["logit"]).to(dev)
    calls = []
    g = ckl.VocabGroup(1, 0, 900, 0, lambda s, r: (calls.append(1), r.copy_(s)),
                       lambda b: calls.append(2))
    loss = ckl.chunked_kl_loss(H, W, idx, lg, chunk=64, group=g)
    (2.0 * loss).backward()
    r = oracle.fwd_bwd(x["H"], x["W"], x["idx"], x["logit"])
    assert abs(loss.item() - r["loss"]) <= 1e-3 * abs(r["loss"])
    assert np.abs(H.grad.float().cpu().numpy() - 2 * r["dH"]).max() <= 2e-2 * np.abs(2 * r["dH"]).max()
    assert np.abs(W.grad.float().cpu().numpy() - 2 * r["dW"]).max() <= 2e-2 * np.abs(2 * r["dW"]).max()
    assert calls.count(1) == 3 and calls.count(2) == 3


def test_nccl_group_of_one():
    # the torch.distributed adapter on NCCL: collectives on device buffers wrapped
    # from the library's pointers, ordered on the library's stream
    import socket

    import torch.distributed as dist
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    dev = torch.device("cuda", 0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=dev)
    try:
        x = small_case(300, 128, 3000, 16, seed=39, dtype="bf16", teacher_var=3.0, ids="zipf")
        H = torch.from_numpy(x["H"]).to(dev).to(torch.bfloat16)
        W = torch.from_numpy(x["W"]).to(dev).to(torch.bfloat16)
        idx, lg = torch.from_numpy(x["idx"]).to(dev), torch.from_numpy(x["logit"]).to(dev)
        g = ckl.torch_vocab_group(3000)
        assert (g.world, g.rank, g.v0) == (1, 0, 0)
        h = ckl.ChunkedKL(3000, 128, 16, max_chunk=128, device=dev)
        s = torch.cuda.Stream(dev)
        with torch.cuda.stream(s):
            loss, dH, dW = h.fwd_bwd_vocab_parallel(g, H, W, idx, lg, chunk=128)
        ref = h.fwd_bwd(H, W, idx, lg, chunk=128)
        assert torch.equal(dH, ref[1]) and torch.equal(dW, ref[2])
        torch.testing.assert_close(loss, ref[0], rtol=1e-6, atol=1e-7)
        h.close()
    finally:
        dist.destroy_process_group()
