"""Shared helpers of the GPU parity tests: upload seeded inputs, error measures."""
import numpy as np
import torch


def rel_fro(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / nb) if nb > 0 else float(np.linalg.norm(a))


def worst_row(a, b) -> float:
    """Largest per-row relative error max_r |a_r - b_r| / |b_r| (Frobenius norms of rows).

    A row where b is exactly zero counts as 0 if a is zero there too, else as inf,
    so a defect confined to a few rows or one tile cannot hide under a whole-tensor
    norm.
    """
    a = np.asarray(a, np.float64).reshape(len(a), -1)
    b = np.asarray(b, np.float64).reshape(len(b), -1)
    nb = np.linalg.norm(b, axis=1)
    na = np.linalg.norm(a - b, axis=1)
    zero = nb == 0
    if np.any(zero & (na > 0)):
        return float("inf")
    return float(np.max(na[~zero] / nb[~zero])) if np.any(~zero) else 0.0


def rel(a, b) -> float:
    return abs(float(a) - float(b)) / max(abs(float(b)), 1e-30)


def upload(x, dtype, device="cuda"):
    """Host arrays from workloads.make_inputs -> device tensors (bf16 values are exact)."""
    dev = torch.device(device)
    H = torch.from_numpy(x["H"]).to(dev).to(dtype).contiguous()
    W = torch.from_numpy(x["W"]).to(dev).to(dtype).contiguous()
    idx = torch.from_numpy(np.ascontiguousarray(x["idx"], dtype=np.int32)).to(dev)
    logit = torch.from_numpy(np.ascontiguousarray(x["logit"], dtype=np.float32)).to(dev)
    mask = None if x.get("mask") is None else torch.from_numpy(
        np.ascontiguousarray(x["mask"], dtype=np.uint8)).to(dev)
    return H, W, idx, logit, mask


def f64(t):
    return t.detach().to(torch.float64).cpu().numpy()


# Tolerances stated for the method's parity: fp32 inputs computed in fp32, bf16
# inputs with fp32 accumulation against the oracle on the same bf16 values.
TOL = {
    "f32": {"loss": 1e-5, "grad": 1e-4},
    "bf16": {"loss": 1e-3, "grad": 2e-2},
}

# Worst single row (a token's dH row, a vocabulary id's dW row) and worst single
# token (absolute error of lse_t and l_t, in nats). Rounding spreads evenly over
# rows, so these sit a few times above the whole-tensor errors; a wrong tile or a
# wrong token shows up as an error of order one.
ROW_TOL = {
    "f32": {"grad_row": 1e-3, "tok_abs": 1e-4},
    "bf16": {"grad_row": 5e-2, "tok_abs": 2e-3},
}
