"""The vocabulary-parallel loss over NCCL on two GPUs: two processes launched with
torch.distributed.run, the LM head split by vocabulary rows, the autograd wrapper
with torch_vocab_group. The loss and dH (identical on both ranks) and the two dW
shards (concatenated) are checked against the fp64 oracle on the full head.
Skipped where fewer than two GPUs are visible.
"""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
from chunked_kl_loss_logits_b200.workloads import small_case
from tests._helpers import TOL, rel, rel_fro

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(torch.cuda.device_count() < 2, reason="needs two GPUs")
def test_vocab_parallel_autograd_on_two_gpus(tmp_path):
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    env = dict(os.environ, NCCL_NVLS_ENABLE="0")
    cmd = ["timeout", "-k", "30", "240", sys.executable, "-m", "torch.distributed.run",
           "--nnodes=1", "--nproc-per-node=2", "--master-addr=127.0.0.1",
           f"--master-port={port}", os.path.join(ROOT, "tests", "vp_nccl_worker.py"),
           str(tmp_path)]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    out = [np.load(tmp_path / f"rank{k}.npz") for k in range(2)]
    x = small_case(600, 256, 5000, 32, seed=71, dtype="bf16", teacher_var=3.0, ids="zipf",
                   packing=True)
    ref = oracle.fwd_bwd(x["H"], x["W"], x["idx"], x["logit"], x["mask"])
    assert float(out[0]["loss"]) == float(out[1]["loss"])
    assert np.array_equal(out[0]["dH"], out[1]["dH"])
    assert rel(float(out[0]["loss"]), ref["loss"]) <= TOL["bf16"]["loss"]
    assert rel_fro(out[0]["dH"], ref["dH"]) <= TOL["bf16"]["grad"]
    dW = np.concatenate([o["dW"] for o in out])
    assert int(out[1]["v0"]) == out[0]["dW"].shape[0]
    assert rel_fro(dW, ref["dW"]) <= TOL["bf16"]["grad"]
