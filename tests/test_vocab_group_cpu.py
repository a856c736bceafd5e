"""Host side of the vocabulary-parallel path, on CPU: the row split of the LM
head, and the torch.distributed collectives of `torch_vocab_group` on a gloo
group of two processes (rank-major gather, element-wise sum)."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from chunked_kl_loss_logits_b200 import ckl


@pytest.mark.parametrize("V,world", [(201088, 2), (201088, 8), (1000, 3), (300, 2), (256, 1)])
def test_vocab_shards_cover_the_vocabulary(V, world):
    sh = ckl.vocab_shards(V, world)
    assert len(sh) == world and sh[0][0] == 0
    for (a, n), (b, _) in zip(sh, sh[1:]):
        assert a + n == b and a % 256 == 0
    assert sh[-1][0] + sh[-1][1] == V and all(n > 0 for _, n in sh)
    assert max(n for _, n in sh) - min(n for _, n in sh) < 2 * 256  # one block, plus a partial last one


def test_vocab_shards_reject_empty_ranks():
    with pytest.raises(ValueError):
        ckl.vocab_shards(300, 3)  # two 256-row blocks cannot feed three ranks


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = ckl.torch_vocab_group(1000, None)
        send = torch.arange(6, dtype=torch.float32) + 10 * rank
        recv = torch.empty(6 * world)
        g.all_gather(send, recv)
        buf = torch.full((5,), float(rank + 1))
        g.all_reduce_sum(buf)
        out[rank] = (g.world, g.rank, g.v0, recv.tolist(), buf.tolist())
    finally:
        dist.destroy_process_group()


def test_torch_group_collectives_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(120)
    assert all(p.exitcode == 0 for p in ps)
    shards = ckl.vocab_shards(1000, world)
    for r in range(world):
        w, rk, v0, recv, buf = out[r]
        assert (w, rk, v0) == (world, r, shards[r][0])
        assert recv == [float(i + 10 * q) for q in range(world) for i in range(6)]
        assert buf == [float(sum(range(1, world + 1)))] * 5
