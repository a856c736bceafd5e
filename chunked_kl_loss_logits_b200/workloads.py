"""Seeded synthetic inputs for the chunked top-K forward-KL loss.

This module only draws inputs. It holds none of the loss arithmetic, so both the
CUDA path's callers and the fp64 oracle's callers can take their inputs from it
without sharing any of the method's computation.

The workloads follow the toy benchmark of "Chunked KL loss, running Knowledge
Distillation locally in less <6GB VRAM" (section "Synthetic hidden states,
output weights, and sparse teacher targets are generated deterministically"):
hidden states H (T x d), output weights W (V x d) and a cached top-K teacher
(K token ids plus K logits per position). The shapes are the gpt-oss-120b LM head
(V = 201,088) at the context lengths the pages benchmark (4K .. 256K tokens).

Distributions (all draws from numpy's PCG64, one child stream per tensor):
  * H ~ N(0, 1); W ~ N(0, 1/d) (variance 1/d, so student logits are O(1)).
  * teacher ids: K distinct ids per position. "uniform": uniform without
    replacement. "zipf": each draw comes with probability 0.8 from a Zipf(1.1)
    ranking of the vocabulary (rank r has weight r^-1.1, ranks mapped to ids by a
    seeded permutation) and otherwise uniformly; repeated ids are rejected until
    K distinct ones are held, in draw order.
  * teacher logits ~ N(0, var), sorted in descending order along K (slot 0 holds
    the largest logit).
  * packing mask: 64 segments with random cut points summing to T; the last token
    of each segment is masked (it has no next-token target), plus uniformly drawn
    positions until round(0.05 * T) positions are masked in total.
bf16 workloads round H and W to bf16 (round to nearest even) on the host, so the
float32 arrays returned here hold exactly the values the GPU sees.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    V: int
    K: int
    chunk: int
    dtype: str  # "f32" or "bf16"
    teacher_var: float
    ids: str  # "uniform" or "zipf"
    packing: bool = False
    chunk_sweep: tuple = field(default_factory=tuple)
    seed: int = 0

    @property
    def useful_flops(self) -> float:
        """6*T*V*d: the forward contraction plus the dH and dW contractions."""
        return 6.0 * self.T * self.V * self.d

    @property
    def executed_flops(self) -> float:
        """8*T*V*d: as above plus the recomputation of the logits in the backward pass."""
        return 8.0 * self.T * self.V * self.d


# The five workloads: a tiny fp32 case, a 4K bf16 case, the 32K-context headline
# case, a packed 128K case and a 256K case with a chunk-size sweep.
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 256, 128, 4096, 16, 64, "f32", 2.0, "uniform", seed=1001),
    "bf16_4k": Workload("bf16_4k", 4096, 2048, 32000, 100, 1024, "bf16", 3.0, "zipf", seed=1002),
    "bf16_32k": Workload("bf16_32k", 32768, 2880, 201088, 100, 2048, "bf16", 3.0, "zipf", seed=1003),
    "bf16_128k_packed": Workload("bf16_128k_packed", 131072, 2880, 201088, 100, 4096, "bf16", 3.0,
                                 "zipf", packing=True, seed=1004),
    "bf16_256k": Workload("bf16_256k", 262144, 2880, 201088, 100, 2048, "bf16", 3.0, "zipf",
                          chunk_sweep=(512, 1024, 2048, 4096, 8192), seed=1005),
    # Profiling case: one 2048-token chunk of the headline shapes (d, K, chunk) with
    # a 32000-word vocabulary, so W (184 MB) still exceeds L2 while the whole
    # footprint stays under 1 GB for multi-pass counter captures.
    "prof_2k": Workload("prof_2k", 2048, 2880, 32000, 100, 2048, "bf16", 3.0, "zipf", seed=1099),
    # Two chunks of the same shapes: the second dW contraction adds into the dW the
    # first one stored, as every chunk after the first does at full size (dW, 368 MB
    # fp32, still exceeds L2).
    "prof_2x2k": Workload("prof_2x2k", 4096, 2880, 32000, 100, 2048, "bf16", 3.0, "zipf",
                          seed=1098),
}

_STREAMS = ("perm", "ids", "logits", "H", "W", "mask")


def round_to_bf16(x: np.ndarray, block: int = 1 << 22) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even), in place; return x.

    Works block by block on the raw bits: add 0x7FFF plus the lowest kept bit,
    then clear the 16 dropped bits. Inputs here are finite and far from the
    float32 range limit, so the addition cannot carry into the sign bit.
    """
    if x.dtype != np.float32 or not x.flags.c_contiguous:
        x = np.ascontiguousarray(x, dtype=np.float32)
    flat = x.reshape(-1).view(np.uint32)
    tmp = np.empty(min(block, flat.size), dtype=np.uint32)
    for i in range(0, flat.size, block):
        b = flat[i:i + block]
        t = tmp[:b.size]
        np.right_shift(b, 16, out=t)
        np.bitwise_and(t, 1, out=t)
        np.add(t, 0x7FFF, out=t)
        np.add(b, t, out=b)
        np.bitwise_and(b, np.uint32(0xFFFF0000), out=b)
    return x


def _rngs(seed: int) -> dict:
    children = np.random.SeedSequence(seed).spawn(len(_STREAMS))
    return {n: np.random.Generator(np.random.PCG64(c)) for n, c in zip(_STREAMS, children)}


def _normal(rng, shape, std, bf16, block_rows=4096):
    """N(0, std^2) float32 draws, generated, scaled and (optionally) bf16-rounded per block."""
    out = np.empty(shape, dtype=np.float32)
    for r0 in range(0, shape[0], block_rows):
        blk = out[r0:min(shape[0], r0 + block_rows)]
        rng.standard_normal(blk.shape, dtype=np.float32, out=blk)
        if std != 1.0:
            blk *= np.float32(std)
        if bf16:
            round_to_bf16(blk)
    return out


def _first_k_distinct(cand: np.ndarray, K: int):
    """Per row, the first K distinct values of `cand` in draw order, and which rows had K."""
    order = np.argsort(cand, axis=1, kind="stable")
    srt = np.take_along_axis(cand, order, axis=1)
    dup = np.zeros(srt.shape, dtype=bool)
    dup[:, 1:] = srt[:, 1:] == srt[:, :-1]
    first = np.empty_like(dup)
    np.put_along_axis(first, order, ~dup, axis=1)
    cnt = np.cumsum(first, axis=1)
    ok = cnt[:, -1] >= K
    sel = first & (cnt <= K)
    out = np.zeros((cand.shape[0], K), dtype=np.int64)
    out[ok] = cand[ok][sel[ok]].reshape(-1, K)
    return out, ok


def teacher_ids(rng, perm, T, V, K, kind, block=8192) -> np.ndarray:
    """K distinct teacher token ids per position, int32 (T, K)."""
    if K > V:
        raise ValueError("K must not exceed V")
    out = np.empty((T, K), dtype=np.int32)
    if kind == "zipf":
        w = np.arange(1, V + 1, dtype=np.float64) ** -1.1
        cdf = np.cumsum(w)
        cdf /= cdf[-1]

    def draw(n):
        if kind == "uniform":
            return rng.integers(0, V, n)
        from_zipf = rng.random(n) < 0.8
        rank = np.minimum(np.searchsorted(cdf, rng.random(n), side="right"), V - 1)
        return np.where(from_zipf, perm[rank], rng.integers(0, V, n))

    for t0 in range(0, T, block):
        t1 = min(T, t0 + block)
        rows = np.arange(t0, t1)
        C = 4 * K
        while rows.size:
            cand = draw(rows.size * C).reshape(rows.size, C)
            got, ok = _first_k_distinct(cand, K)
            out[rows[ok]] = got[ok]
            rows = rows[~ok]
            C *= 2
    return out


def teacher_logits(rng, T, K, var) -> np.ndarray:
    x = rng.standard_normal((T, K), dtype=np.float32) * np.float32(np.sqrt(var))
    return -np.sort(-x, axis=1)


def packing_mask(rng, T, segments=64, frac=0.05) -> np.ndarray:
    """uint8 (T,): 0 at each segment's last token and at random positions, 1 elsewhere."""
    mask = np.ones(T, dtype=np.uint8)
    segments = max(1, min(segments, T))
    cuts = np.sort(rng.choice(np.arange(1, T), size=segments - 1, replace=False))
    ends = np.concatenate([cuts - 1, [T - 1]])
    mask[ends] = 0
    target = int(round(frac * T))
    free = np.flatnonzero(mask)
    extra = max(0, target - (T - free.size))
    if extra:
        mask[rng.choice(free, size=extra, replace=False)] = 0
    return mask


def make_inputs(w: Workload, T: int | None = None, seed: int | None = None) -> dict:
    """Draw one workload's inputs as host arrays.

    Returns H (T, d) and W (V, d) as float32 (bf16-representable for bf16
    workloads), idx int32 (T, K), logit float32 (T, K) and mask uint8 (T,) or None.
    `T` overrides the token count (the peak-memory sweep draws shorter sequences).
    """
    T = w.T if T is None else T
    r = _rngs(w.seed if seed is None else seed)
    perm = r["perm"].permutation(w.V)
    idx = teacher_ids(r["ids"], perm, T, w.V, w.K, w.ids)
    logit = teacher_logits(r["logits"], T, w.K, w.teacher_var)
    bf16 = w.dtype == "bf16"
    H = _normal(r["H"], (T, w.d), 1.0, bf16)
    W = _normal(r["W"], (w.V, w.d), 1.0 / np.sqrt(w.d), bf16)
    mask = packing_mask(r["mask"], T) if w.packing else None
    return {"H": H, "W": W, "idx": idx, "logit": logit, "mask": mask}


def small_case(T, d, V, K, seed, dtype="f32", teacher_var=2.0, ids="uniform", packing=False):
    """A workload-shaped draw at arbitrary (small) sizes, for parity and edge-case tests."""
    w = Workload(f"case_{T}x{d}x{V}x{K}", T, d, V, K, max(1, T), dtype, teacher_var, ids,
                 packing=packing, seed=seed)
    return make_inputs(w)


def sample_rows(T: int, n: int, seed: int) -> np.ndarray:
    """A seeded, sorted sample of n distinct token positions (always including 0 and T-1)."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 77])))
    n = min(n, T)
    inner = rng.choice(np.arange(1, T - 1), size=max(0, n - 2), replace=False) if T > 2 else []
    rows = np.unique(np.concatenate([[0, T - 1], inner]).astype(np.int64))
    return rows
