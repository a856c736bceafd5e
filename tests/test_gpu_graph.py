"""A fused forward+backward call captured in a CUDA graph and replayed.

`ChunkedKL.fwd_bwd(..., sync=False)` with a caller-provided workspace enqueues
only kernel launches, memsets and device-to-device copies (no allocation, no
host synchronisation), so it can be captured once and replayed: the replay must
give the eager call's loss, dH and dW bit for bit, also after new inputs are
copied into the captured buffers.
"""
import pytest
import torch

from chunked_kl_loss_logits_b200 import ckl
from chunked_kl_loss_logits_b200.workloads import small_case

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("recompute", [False, True], ids=["stored", "recompute"])
def test_graph_replay_matches_eager(recompute):
    dev = torch.device("cuda", 0)
    xs = [small_case(300, 128, 3000, 16, seed=s, dtype="bf16", teacher_var=3.0, ids="zipf",
                     packing=True) for s in (51, 52)]

    def dev_inputs(x):
        return (torch.from_numpy(x["H"]).to(dev).to(torch.bfloat16),
                torch.from_numpy(x["W"]).to(dev).to(torch.bfloat16),
                torch.from_numpy(x["idx"]).to(dev), torch.from_numpy(x["logit"]).to(dev),
                torch.from_numpy(x["mask"]).to(dev))

    h = ckl.ChunkedKL(3000, 128, 16, max_chunk=128, device=dev)
    h.set_recompute(recompute)
    ws = h.workspace(300, 128)
    bufs = [t.clone() for t in dev_inputs(xs[0])]
    out = (torch.empty((), device=dev), torch.empty_like(bufs[0]),
           torch.empty((3000, 128), dtype=torch.float32, device=dev))

    def call():
        h.fwd_bwd(*bufs, chunk=128, out=out, workspace=ws, sync=False)

    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        call()  # warm-up outside the capture (first-use setup of the kernels)
    torch.cuda.current_stream(dev).wait_stream(s)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    for x in xs:
        for b, t in zip(bufs, dev_inputs(x)):
            b.copy_(t)
        g.replay()
        torch.cuda.synchronize(dev)
        got = [t.clone() for t in out]
        h.sync_status()
        ref = h.fwd_bwd(*dev_inputs(x), chunk=128)
        for a, b in zip(got, ref):
            assert torch.equal(a, b)
    h.close()
