"""Python binding of libckl.so (argument marshalling only).

Every step of the loss runs in the library's CUDA kernels; this module only
allocates outputs and the workspace with PyTorch, passes raw pointers and the
current CUDA stream, and turns status codes into exceptions. If the library has
not been built the import of `lib()` raises: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# The in-tree build; CKL_LIBRARY names another build of the same library.
LIB_PATH = os.environ.get("CKL_LIBRARY") or os.path.join(_PKG, "lib", "libckl.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "ckl.h")

F32, BF16 = 0, 1
_STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported size", 3: "workspace",
           4: "top-K index out of range", 5: "CUDA error", 6: "device wait timed out",
           7: "pointer misaligned", 8: "internal consistency check failed",
           9: "a caller-supplied collective failed"}


class CKLError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {_STATUS.get(code, code)} (status {code})")
        self.code = code


_GatherFn = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                             ctypes.c_int64, ctypes.c_void_p)
_ReduceFn = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                             ctypes.c_void_p)


class _VocabGroupC(ctypes.Structure):
    """Mirror of ckl_vocab_group."""
    _fields_ = [("world", ctypes.c_int32), ("rank", ctypes.c_int32), ("V_total", ctypes.c_int64),
                ("v0", ctypes.c_int64), ("all_gather", _GatherFn), ("all_reduce_sum", _ReduceFn),
                ("user", ctypes.c_void_p)]


class KernelStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int64),
                ("total_ms", ctypes.c_double), ("flops", ctypes.c_double),
                ("bytes", ctypes.c_double)]


_lib = None
_P, _I64, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t


def lib() -> ctypes.CDLL:
    """Load libckl.so (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m chunked_kl_loss_logits_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    sig = {
        "ckl_create": ([ctypes.POINTER(_P), ctypes.c_int, ctypes.c_int, _I64, _I64, _I64, _I64],
                       ctypes.c_int),
        "ckl_destroy": ([_P], ctypes.c_int),
        "ckl_status_str": ([ctypes.c_int], ctypes.c_char_p),
        "ckl_workspace_bytes": ([_P, _I64, _I64, ctypes.POINTER(_SZ)], ctypes.c_int),
        "ckl_fwd_bwd": ([_P, _P, _P, _P, _P, _P, _I64, _I64, _P, _P, _P, _P, _P, _P, _SZ, _P, _P],
                        ctypes.c_int),
        "ckl_forward": ([_P, _P, _P, _P, _P, _P, _I64, _I64, _P, _P, _P, _P, _SZ, _P, _P],
                        ctypes.c_int),
        "ckl_fwd_bwd_from_host": ([_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _P, _P, _P,
                                   _P, _SZ, _P, _P], ctypes.c_int),
        "ckl_sync_status": ([_P, _P], ctypes.c_int),
        "ckl_launch_count": ([_P], ctypes.c_int64),
        "ckl_set_recompute": ([_P, ctypes.c_int], ctypes.c_int),
        "ckl_topk_workspace_bytes": ([_P, _I64, _I64, ctypes.POINTER(_SZ)], ctypes.c_int),
        "ckl_topk_cache": ([_P, _P, _P, _I64, _I64, _P, _P, _P, _SZ, _P, ctypes.c_int], ctypes.c_int),
        "ckl_vp_workspace_bytes": ([_P, ctypes.c_int32, _I64, _I64, ctypes.POINTER(_SZ)],
                                   ctypes.c_int),
        "ckl_fwd_bwd_vocab_parallel": ([_P, ctypes.POINTER(_VocabGroupC), _P, _P, _P, _P, _P, _I64,
                                        _I64, _P, _P, _P, _P, _P, _P, _SZ, _P, _P], ctypes.c_int),
        "ckl_forward_vocab_parallel": ([_P, ctypes.POINTER(_VocabGroupC), _P, _P, _P, _P, _P, _I64,
                                        _I64, _P, _P, _P, _P, _SZ, _P, _P], ctypes.c_int),
        "ckl_selftest_wait_bound": ([_P, _P, ctypes.POINTER(_I64)], ctypes.c_int),
        "ckl_topk_vp_workspace_bytes": ([_P, ctypes.c_int32, _I64, _I64, ctypes.POINTER(_SZ)],
                                        ctypes.c_int),
        "ckl_topk_cache_vocab_parallel": ([_P, ctypes.POINTER(_VocabGroupC), _P, _P, _I64, _I64,
                                           _P, _P, _P, _SZ, _P, ctypes.c_int], ctypes.c_int),
        "ckl_profile_enable": ([_P, ctypes.c_int, ctypes.c_int], ctypes.c_int),
        "ckl_profile_collect": ([_P, ctypes.POINTER(KernelStat), ctypes.c_int,
                                 ctypes.POINTER(ctypes.c_int)], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    _lib = L
    return L


def header_functions() -> list:
    """Names of the functions include/ckl.h declares."""
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"\b(ckl_[a-z_0-9]+)\s*\(", text)))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(code: int, what: str):
    if code != 0:
        raise CKLError(code, what)


class _DevArray:
    """A raw device pointer seen as a float32 vector (CUDA array interface, no copy)."""

    def __init__(self, ptr: int, count: int):
        self.__cuda_array_interface__ = {"shape": (count,), "typestr": "<f4",
                                         "data": (ptr, False), "version": 3, "stream": None}


def vocab_shards(V_total: int, world: int, align: int = 256) -> list:
    """(v0, V_r) of each rank: contiguous row ranges of the LM head, as equal as
    possible in whole `align`-row blocks (the last rank takes the remainder)."""
    if world < 1 or V_total < world:
        raise ValueError("need 1 <= world <= V_total")
    blocks = (V_total + align - 1) // align
    out, v0 = [], 0
    for r in range(world):
        nb = blocks // world + (1 if r < blocks % world else 0)
        v1 = min(V_total, v0 + nb * align) if r < world - 1 else V_total
        out.append((v0, v1 - v0))
        v0 = v1
    if any(n <= 0 for _, n in out):
        raise ValueError("a rank would hold no rows")
    return out


class VocabGroup:
    """This rank's place in a vocabulary-parallel group and the group's two collectives.

    all_gather(send, recv): send is a float32 vector of n entries, recv one of
    world * n entries to fill rank-major; all_reduce_sum(buf): in place. Both
    get device tensors and must be ordered on the current CUDA stream (the
    library's stream is made current around each call) and return None.
    """

    def __init__(self, world: int, rank: int, V_total: int, v0: int, all_gather, all_reduce_sum):
        self.world, self.rank, self.V_total, self.v0 = world, rank, V_total, v0
        self.all_gather, self.all_reduce_sum = all_gather, all_reduce_sum
        self.error = None

    def _c(self, device):
        def as_stream(ptr):
            return torch.cuda.ExternalStream(ptr, device=device) if ptr else \
                torch.cuda.default_stream(device)

        def gather(_user, send, recv, count, stream):
            try:
                with torch.cuda.stream(as_stream(stream)):
                    a = torch.as_tensor(_DevArray(send, count), device=device)
                    b = torch.as_tensor(_DevArray(recv, count * self.world), device=device)
                    self.all_gather(a, b)
                return 0
            except Exception as e:  # reported as CKL_ERR_COLLECTIVE; kept for the caller
                self.error = e
                return 1

        def reduce(_user, buf, count, stream):
            try:
                with torch.cuda.stream(as_stream(stream)):
                    self.all_reduce_sum(torch.as_tensor(_DevArray(buf, count), device=device))
                return 0
            except Exception as e:
                self.error = e
                return 1

        fns = (_GatherFn(gather), _ReduceFn(reduce))  # kept alive by the caller for the call
        return _VocabGroupC(self.world, self.rank, self.V_total, self.v0, fns[0], fns[1], None), fns


def torch_vocab_group(V_total: int, group=None) -> VocabGroup:
    """A VocabGroup over a torch.distributed process group (NCCL on GPUs): this
    rank's rows come from vocab_shards(V_total, world)."""
    import torch.distributed as dist
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    v0, _ = vocab_shards(V_total, world)[rank]
    return VocabGroup(world, rank, V_total, v0,
                      lambda send, recv: dist.all_gather_into_tensor(recv, send, group=group),
                      lambda buf: dist.all_reduce(buf, group=group))


class ChunkedKL:
    """A handle for one LM-head shape (V x d, K cached teacher entries) on one device."""

    def __init__(self, V: int, d: int, K: int, dtype=torch.bfloat16, max_chunk: int = 8192,
                 device=None):
        if dtype not in (torch.float32, torch.bfloat16):
            raise ValueError("dtype must be torch.float32 or torch.bfloat16")
        self.V, self.d, self.K, self.dtype, self.max_chunk = V, d, K, dtype, max_chunk
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        self.device = dev
        h = _P()
        _check(lib().ckl_create(ctypes.byref(h), dev.index or 0,
                                F32 if dtype == torch.float32 else BF16, V, d, K, max_chunk),
               "ckl_create")
        self._h = h

    def close(self):
        if getattr(self, "_h", None):
            lib().ckl_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ------------------------------------------------------------------ helpers
    def workspace_bytes(self, T: int, chunk: int) -> int:
        n = _SZ()
        _check(lib().ckl_workspace_bytes(self._h, T, chunk, ctypes.byref(n)), "ckl_workspace_bytes")
        return n.value

    def workspace(self, T: int, chunk: int) -> torch.Tensor:
        return torch.empty(max(1, self.workspace_bytes(T, chunk)), dtype=torch.uint8,
                           device=self.device)

    def set_recompute(self, on: bool):
        """bf16 only: form the logits again in the backward (True) or keep exp(z) (False)."""
        _check(lib().ckl_set_recompute(self._h, int(on)), "ckl_set_recompute")

    def launch_count(self) -> int:
        return int(lib().ckl_launch_count(self._h))

    def profile_enable(self, on: bool = True, max_launches: int = 8192):
        _check(lib().ckl_profile_enable(self._h, int(on), max_launches), "ckl_profile_enable")

    def profile_collect(self) -> list:
        arr = (KernelStat * 32)()
        n = ctypes.c_int()
        _check(lib().ckl_profile_collect(self._h, arr, 32, ctypes.byref(n)), "ckl_profile_collect")
        return [{"name": arr[i].name.decode(), "launches": arr[i].launches,
                 "total_ms": arr[i].total_ms, "flops": arr[i].flops, "bytes": arr[i].bytes}
                for i in range(min(n.value, 32))]

    def selftest_wait_bound(self, stream=None):
        """(status code, SM cycles waited) of the bounded-wait self-test; 6 (timeout) is a pass."""
        s = stream or torch.cuda.current_stream(self.device)
        cyc = _I64()
        code = lib().ckl_selftest_wait_bound(self._h, ctypes.c_void_p(s.cuda_stream),
                                             ctypes.byref(cyc))
        return code, cyc.value

    def sync_status(self, stream=None):
        s = stream or torch.cuda.current_stream(self.device)
        _check(lib().ckl_sync_status(self._h, ctypes.c_void_p(s.cuda_stream)), "ckl_sync_status")

    def _inputs(self, H, W, idx, logit, mask):
        T = H.shape[0]
        if H.dtype != self.dtype or W.dtype != self.dtype:
            raise TypeError(f"H and W must be {self.dtype}")
        if tuple(W.shape) != (self.V, self.d) or H.shape[1] != self.d:
            raise ValueError("H must be T x d and W must be V x d")
        if tuple(idx.shape) != (T, self.K) or tuple(logit.shape) != (T, self.K):
            raise ValueError("topk_idx and topk_logit must be T x K")
        if idx.dtype != torch.int32 or logit.dtype != torch.float32:
            raise TypeError("topk_idx must be int32 and topk_logit float32")
        if mask is not None and (mask.dtype != torch.uint8 or mask.numel() != T):
            raise TypeError("mask must be a uint8 tensor of T entries")
        for t in (H, W, idx, logit) + ((mask,) if mask is not None else ()):
            if not t.is_contiguous() or t.device != self.device:
                raise ValueError("inputs must be contiguous tensors on the handle's device")
        return T

    # ------------------------------------------------------------------ calls
    def fwd_bwd(self, H, W, idx, logit, mask=None, chunk: int | None = None, out=None,
                workspace=None, token_stats: bool = False, sync: bool = True, stream=None):
        """Loss (0-d float32 tensor), dH (T x d, dtype), dW (V x d, float32).

        With token_stats=True also returns per-token logsumexp and loss (float32, T).
        With sync=True the call waits and raises on a device-detected error.
        """
        T = self._inputs(H, W, idx, logit, mask)
        chunk = min(chunk or self.max_chunk, self.max_chunk)
        if out is None:
            out = (torch.empty((), dtype=torch.float32, device=self.device),
                   torch.empty_like(H), torch.empty((self.V, self.d), dtype=torch.float32,
                                                    device=self.device))
        loss, dH, dW = out
        ws = workspace if workspace is not None else self.workspace(T, chunk)
        lse = ell = None
        if token_stats:
            lse = torch.empty(T, dtype=torch.float32, device=self.device)
            ell = torch.empty(T, dtype=torch.float32, device=self.device)
        s = stream or torch.cuda.current_stream(self.device)
        host = ctypes.c_float() if sync else None
        code = lib().ckl_fwd_bwd(self._h, _ptr(H), _ptr(W), _ptr(idx), _ptr(logit), _ptr(mask), T,
                                 chunk, _ptr(loss), _ptr(dH), _ptr(dW), _ptr(lse), _ptr(ell),
                                 _ptr(ws), ws.numel(), ctypes.c_void_p(s.cuda_stream),
                                 ctypes.byref(host) if sync else None)
        _check(code, "ckl_fwd_bwd")
        return (loss, dH, dW, lse, ell) if token_stats else (loss, dH, dW)

    def forward(self, H, W, idx, logit, mask=None, chunk: int | None = None, workspace=None,
                token_stats: bool = False, sync: bool = True, stream=None):
        """Loss only (no gradients); optionally per-token logsumexp and loss."""
        T = self._inputs(H, W, idx, logit, mask)
        chunk = min(chunk or self.max_chunk, self.max_chunk)
        loss = torch.empty((), dtype=torch.float32, device=self.device)
        ws = workspace if workspace is not None else self.workspace(T, chunk)
        lse = ell = None
        if token_stats:
            lse = torch.empty(T, dtype=torch.float32, device=self.device)
            ell = torch.empty(T, dtype=torch.float32, device=self.device)
        s = stream or torch.cuda.current_stream(self.device)
        host = ctypes.c_float()
        _check(lib().ckl_forward(self._h, _ptr(H), _ptr(W), _ptr(idx), _ptr(logit), _ptr(mask), T,
                                 chunk, _ptr(loss), _ptr(lse), _ptr(ell), _ptr(ws), ws.numel(),
                                 ctypes.c_void_p(s.cuda_stream),
                                 ctypes.byref(host) if sync else None), "ckl_forward")
        return (loss, lse, ell) if token_stats else loss

    def fwd_bwd_vocab_parallel(self, group: VocabGroup, H, W_shard, idx, logit, mask=None,
                               chunk: int | None = None, token_stats: bool = False,
                               sync: bool = True, stream=None):
        """Loss, dH (full, identical on every rank) and dW_shard (this rank's V x d rows).

        The handle's V is this rank's row count; ids are global in [0, group.V_total).
        """
        T = self._inputs(H, W_shard, idx, logit, mask)
        chunk = min(chunk or self.max_chunk, self.max_chunk)
        n = _SZ()
        _check(lib().ckl_vp_workspace_bytes(self._h, group.world, T, chunk, ctypes.byref(n)),
               "ckl_vp_workspace_bytes")
        ws = torch.empty(max(1, n.value), dtype=torch.uint8, device=self.device)
        loss = torch.empty((), dtype=torch.float32, device=self.device)
        dH = torch.empty_like(H)
        dW = torch.empty((self.V, self.d), dtype=torch.float32, device=self.device)
        lse = ell = None
        if token_stats:
            lse = torch.empty(T, dtype=torch.float32, device=self.device)
            ell = torch.empty(T, dtype=torch.float32, device=self.device)
        s = stream or torch.cuda.current_stream(self.device)
        g, keep = group._c(self.device)
        host = ctypes.c_float() if sync else None
        group.error = None
        code = lib().ckl_fwd_bwd_vocab_parallel(
            self._h, ctypes.byref(g), _ptr(H), _ptr(W_shard), _ptr(idx), _ptr(logit), _ptr(mask),
            T, chunk, _ptr(loss), _ptr(dH), _ptr(dW), _ptr(lse), _ptr(ell), _ptr(ws), ws.numel(),
            ctypes.c_void_p(s.cuda_stream), ctypes.byref(host) if sync else None)
        del keep
        if code == 9 and group.error is not None:
            raise CKLError(code, "ckl_fwd_bwd_vocab_parallel") from group.error
        _check(code, "ckl_fwd_bwd_vocab_parallel")
        return (loss, dH, dW, lse, ell) if token_stats else (loss, dH, dW)

    def forward_vocab_parallel(self, group: VocabGroup, H, W_shard, idx, logit, mask=None,
                               chunk: int | None = None, token_stats: bool = False,
                               sync: bool = True, stream=None):
        """Loss only (identical on every rank); the handle's V is this rank's row count."""
        T = self._inputs(H, W_shard, idx, logit, mask)
        chunk = min(chunk or self.max_chunk, self.max_chunk)
        n = _SZ()
        _check(lib().ckl_vp_workspace_bytes(self._h, group.world, T, chunk, ctypes.byref(n)),
               "ckl_vp_workspace_bytes")
        ws = torch.empty(max(1, n.value), dtype=torch.uint8, device=self.device)
        loss = torch.empty((), dtype=torch.float32, device=self.device)
        lse = ell = None
        if token_stats:
            lse = torch.empty(T, dtype=torch.float32, device=self.device)
            ell = torch.empty(T, dtype=torch.float32, device=self.device)
        s = stream or torch.cuda.current_stream(self.device)
        g, keep = group._c(self.device)
        host = ctypes.c_float() if sync else None
        group.error = None
        code = lib().ckl_forward_vocab_parallel(
            self._h, ctypes.byref(g), _ptr(H), _ptr(W_shard), _ptr(idx), _ptr(logit), _ptr(mask),
            T, chunk, _ptr(loss), _ptr(lse), _ptr(ell), _ptr(ws), ws.numel(),
            ctypes.c_void_p(s.cuda_stream), ctypes.byref(host) if sync else None)
        del keep
        if code == 9 and group.error is not None:
            raise CKLError(code, "ckl_forward_vocab_parallel") from group.error
        _check(code, "ckl_forward_vocab_parallel")
        return (loss, lse, ell) if token_stats else loss

    def topk_cache(self, H, W, chunk: int | None = None, workspace=None, sync: bool = True,
                   stream=None):
        """Teacher top-K cache: (ids int32 T x K, logits float32 T x K), descending.

        The handle must have the teacher's shape (V, d = teacher hidden size, K).
        """
        T = H.shape[0]
        if H.dtype != self.dtype or W.dtype != self.dtype or H.shape[1] != self.d or \
                tuple(W.shape) != (self.V, self.d):
            raise ValueError("H must be T x d and W must be V x d, in the handle's dtype")
        chunk = min(chunk or self.max_chunk, self.max_chunk)
        idx = torch.empty((T, self.K), dtype=torch.int32, device=self.device)
        logit = torch.empty((T, self.K), dtype=torch.float32, device=self.device)
        if workspace is None:
            n = _SZ()
            _check(lib().ckl_topk_workspace_bytes(self._h, T, chunk, ctypes.byref(n)),
                   "ckl_topk_workspace_bytes")
            workspace = torch.empty(max(1, n.value), dtype=torch.uint8, device=self.device)
        s = stream or torch.cuda.current_stream(self.device)
        _check(lib().ckl_topk_cache(self._h, _ptr(H), _ptr(W), T, chunk, _ptr(idx), _ptr(logit),
                                    _ptr(workspace), workspace.numel(),
                                    ctypes.c_void_p(s.cuda_stream), int(sync)), "ckl_topk_cache")
        return idx, logit

    def topk_cache_vocab_parallel(self, group: VocabGroup, H, W_shard, chunk: int | None = None,
                                  sync: bool = True, stream=None):
        """Teacher top-K cache with the teacher's LM head split by vocabulary rows over
        `group`: (ids int32 T x K, global; logits float32 T x K), the same on every
        rank and the same as topk_cache with all of W on one rank."""
        T = H.shape[0]
        if H.dtype != self.dtype or W_shard.dtype != self.dtype or H.shape[1] != self.d or \
                tuple(W_shard.shape) != (self.V, self.d):
            raise ValueError("H must be T x d and W_shard V x d, in the handle's dtype")
        chunk = min(chunk or self.max_chunk, self.max_chunk)
        n = _SZ()
        _check(lib().ckl_topk_vp_workspace_bytes(self._h, group.world, T, chunk, ctypes.byref(n)),
               "ckl_topk_vp_workspace_bytes")
        ws = torch.empty(max(1, n.value), dtype=torch.uint8, device=self.device)
        idx = torch.empty((T, self.K), dtype=torch.int32, device=self.device)
        logit = torch.empty((T, self.K), dtype=torch.float32, device=self.device)
        s = stream or torch.cuda.current_stream(self.device)
        g, keep = group._c(self.device)
        group.error = None
        code = lib().ckl_topk_cache_vocab_parallel(
            self._h, ctypes.byref(g), _ptr(H), _ptr(W_shard), T, chunk, _ptr(idx), _ptr(logit),
            _ptr(ws), ws.numel(), ctypes.c_void_p(s.cuda_stream), int(sync))
        del keep
        if code == 9 and group.error is not None:
            raise CKLError(code, "ckl_topk_cache_vocab_parallel") from group.error
        _check(code, "ckl_topk_cache_vocab_parallel")
        return idx, logit

    def fwd_bwd_from_host(self, H_host, idx_host, logit_host, mask_host, staging, W, chunk,
                          out, workspace, stream=None) -> float:
        """Fused loss with the per-step inputs in (pinned) host memory; returns the loss.

        `staging` = (H_dev, idx_dev, logit_dev, mask_dev or None): device buffers
        the inputs are copied into. `out` = (loss, dH, dW) device tensors.
        """
        H_dev, idx_dev, logit_dev, mask_dev = staging
        loss, dH, dW = out
        T = H_host.shape[0]
        s = stream or torch.cuda.current_stream(self.device)
        host = ctypes.c_float()
        _check(lib().ckl_fwd_bwd_from_host(
            self._h, _ptr(H_host), _ptr(idx_host), _ptr(logit_host), _ptr(mask_host),
            _ptr(H_dev), _ptr(idx_dev), _ptr(logit_dev), _ptr(mask_dev), _ptr(W), T, chunk,
            _ptr(loss), _ptr(dH), _ptr(dW), _ptr(workspace), workspace.numel(),
            ctypes.c_void_p(s.cuda_stream), ctypes.byref(host)), "ckl_fwd_bwd_from_host")
        return host.value


class _ChunkedKLFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, H, W, idx, logit, mask, handle, chunk, check):
        loss, dH, dW = handle.fwd_bwd(H.detach(), W.detach(), idx, logit, mask, chunk=chunk,
                                      sync=False)
        ctx.save_for_backward(dH, dW)
        ctx.w_dtype = W.dtype
        ctx.handle, ctx.check = handle, check
        return loss

    @staticmethod
    def backward(ctx, g):
        if ctx.check:
            ctx.handle.sync_status()  # raises CKLError on a device-detected error
        dH, dW = ctx.saved_tensors
        return (dH * g.to(dH.dtype), (dW * g).to(ctx.w_dtype), None, None, None, None, None, None)


class _VocabParallelKLFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, H, W_shard, idx, logit, mask, handle, chunk, group, check):
        loss, dH, dW = handle.fwd_bwd_vocab_parallel(group, H.detach(), W_shard.detach(), idx,
                                                     logit, mask, chunk=chunk, sync=False)
        ctx.save_for_backward(dH, dW)
        ctx.w_dtype = W_shard.dtype
        ctx.handle, ctx.check = handle, check
        return loss

    @staticmethod
    def backward(ctx, g):
        if ctx.check:
            ctx.handle.sync_status()
        dH, dW = ctx.saved_tensors
        return (dH * g.to(dH.dtype), (dW * g).to(ctx.w_dtype), None, None, None, None, None, None,
                None)


_HANDLES = {}


def handle_for(W, K: int, chunk: int | None = None) -> ChunkedKL:
    """The cached handle for W's device, dtype and shape with K cached entries.

    chunked_kl_loss calls this when it is given no handle, so a training loop
    creates one handle per LM-head shape (ckl_create allocates and synchronises
    the device) instead of one per step. The handle is replaced by one with a
    larger max_chunk when a call asks for a chunk above the cached one's.
    """
    dev = W.device
    key = (dev.type, dev.index, W.dtype, W.shape[0], W.shape[1], K)
    h = _HANDLES.get(key)
    need = max(chunk or 4096, 1)
    if h is None or h.max_chunk < need:
        if h is not None:
            h.close()
        h = ChunkedKL(W.shape[0], W.shape[1], K, dtype=W.dtype, max_chunk=need, device=dev)
        _HANDLES[key] = h
    return h


def chunked_kl_loss(H, W, idx, logit, mask=None, chunk=None, handle: ChunkedKL | None = None,
                    group: VocabGroup | None = None, check: bool = True):
    """Autograd-friendly mean top-K forward KL; the gradients come from the fused call.

    With `group`, W is this rank's vocabulary rows (vocab_shards) and the loss is the
    full-vocabulary one, identical on every rank; H's gradient is the full dH on
    every rank and W's is this rank's rows. Without `handle` the handle cached for
    W's shape (handle_for) is used.

    check=True: backward() waits for the call's stream and raises CKLError if the
    device reported an error (a teacher id outside [0, V), a pipeline timeout);
    the outputs of such a call are undefined. check=False: nothing waits; the
    device status stays set in the handle (errors of later calls add to it) until
    the caller reads it with handle.sync_status() (handle_for(W, K) gives the
    cached handle), which raises and clears it.
    """
    if handle is None:
        handle = handle_for(W, idx.shape[1], chunk)
    if group is not None:
        return _VocabParallelKLFn.apply(H, W, idx, logit, mask, handle, chunk, group, check)
    return _ChunkedKLFn.apply(H, W, idx, logit, mask, handle, chunk, check)


def forward_static(H, W, idx, logit, mask=None, chunk: int = 2048, stream=None,
                   token_stats: bool = False):
    """Forward-only loss through ckl_forward_static: no device allocation by the library.

    For callers that may not allocate device memory: the library's scratch is a
    fixed 32 MiB device array shared by all calls (overlapping calls race). The
    outputs here are allocated by torch on the caller's side; pass your own
    buffers to the C entry point if that is not allowed either. Returns the loss
    (0-d float32 tensor), plus per-token logsumexp and loss when token_stats.
    """
    f = lib().ckl_forward_static
    f.argtypes = [ctypes.c_int, ctypes.c_int, _I64, _I64, _I64, _P, _P, _P, _P, _P, _I64, _I64,
                  _P, _P, _P, _P, _P]
    f.restype = ctypes.c_int
    T, d = H.shape
    V, K = W.shape[0], idx.shape[1]
    dev = H.device
    loss = torch.empty((), dtype=torch.float32, device=dev)
    lse = ell = None
    if token_stats:
        lse = torch.empty(T, dtype=torch.float32, device=dev)
        ell = torch.empty(T, dtype=torch.float32, device=dev)
    s = stream or torch.cuda.current_stream(dev)
    host = ctypes.c_float()
    _check(f(dev.index or 0, F32 if H.dtype == torch.float32 else BF16, V, d, K, _ptr(H), _ptr(W),
             _ptr(idx), _ptr(logit), _ptr(mask), T, chunk, _ptr(loss), _ptr(lse), _ptr(ell),
             ctypes.c_void_p(s.cuda_stream), ctypes.byref(host)), "ckl_forward_static")
    return (loss, lse, ell) if token_stats else loss
