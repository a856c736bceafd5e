"""One rank of the two-GPU vocabulary-parallel check (launched by torch.distributed.run
from tests/test_gpu_vp_nccl.py; not collected by pytest).

Every rank draws the same seeded inputs, keeps its rows of the LM head
(vocab_shards), runs the autograd wrapper with an NCCL group, and writes its loss,
dH and dW shard to <out>/rank<r>.npz for the parent test to check against the
oracle.
"""
import datetime
import os
import sys

import numpy as np
import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from chunked_kl_loss_logits_b200 import ckl  # noqa: E402
from chunked_kl_loss_logits_b200.workloads import small_case  # noqa: E402


def main(out_dir):
    rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    dev = torch.device("cuda", int(os.environ["LOCAL_RANK"]))
    torch.cuda.set_device(dev)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    try:
        x = small_case(600, 256, 5000, 32, seed=71, dtype="bf16", teacher_var=3.0, ids="zipf",
                       packing=True)
        V = x["W"].shape[0]
        v0, Vr = ckl.vocab_shards(V, world)[rank]
        H = torch.from_numpy(x["H"]).to(dev).to(torch.bfloat16).requires_grad_(True)
        W = torch.from_numpy(x["W"][v0:v0 + Vr]).to(dev).to(torch.bfloat16).requires_grad_(True)
        idx = torch.from_numpy(x["idx"]).to(dev)
        lg = torch.from_numpy(x["logit"]).to(dev)
        mask = torch.from_numpy(x["mask"]).to(dev)
        g = ckl.torch_vocab_group(V)
        loss = ckl.chunked_kl_loss(H, W, idx, lg, mask, chunk=256, group=g)
        loss.backward()
        torch.cuda.synchronize(dev)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), loss=loss.item(), v0=v0,
                 dH=H.grad.float().cpu().numpy(), dW=W.grad.float().cpu().numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


if __name__ == "__main__":
    main(sys.argv[1])
