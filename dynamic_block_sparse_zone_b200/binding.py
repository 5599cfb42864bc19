"""Thin Python binding of libprism.so (the C ABI in include/prism.h).

Argument marshalling only: torch tensors provide device memory and the
current CUDA stream; every step of the computation runs in the library's
kernels.  There is no fallback: if the library is missing or a call fails, an
exception is raised.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Tuple

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libprism.so")

PRISM_OK = 0
_STATUS = {0: "PRISM_OK", 1: "PRISM_ERR_INVALID_ARG", 2: "PRISM_ERR_UNSUPPORTED", 3: "PRISM_ERR_CUDA",
           4: "PRISM_ERR_TIMEOUT", 5: "PRISM_ERR_NOMEM", 6: "PRISM_ERR_STATE"}

EXPORTED = ("prism_plan_create", "prism_plan_bytes", "prism_plan_build", "prism_attn_fwd", "prism_attn_bwd",
            "prism_plan_view_get", "prism_plan_check", "prism_plan_destroy", "prism_last_error",
            "prism_plan_set_timing", "prism_plan_read_timing", "prism_timer_name", "prism_zone_shapes_noalloc",
            "prism_plan_selftest_timeout", "prism_plan_update_qkv", "prism_step_host", "prism_step_join",
            "prism_step_wait", "prism_audio_norms", "prism_plan_build_stats", "prism_plan_stats_slice",
            "prism_plan_build_finish", "prism_attn_fwd_taylor", "prism_plan_build_with_zones")
NUM_TIMERS = 12


class PrismError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_STATUS.get(status, status)}: {msg}")
        self.status = status


class prism_params(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
                ("heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("top_k", ctypes.c_int),
                ("top_p", ctypes.c_float), ("max_frac", ctypes.c_float), ("fixed_shape", ctypes.c_int * 3),
                ("eps", ctypes.c_double), ("heads_total", ctypes.c_int), ("head_offset", ctypes.c_int),
                ("hilbert_block", ctypes.c_int)]


class prism_plan_view(ctypes.Structure):
    _fields_ = [("zone_B", ctypes.c_void_p), ("zone_shape", ctypes.c_void_p), ("perm", ctypes.c_void_p),
                ("blk_off", ctypes.c_void_p), ("row_ptr", ctypes.c_void_p), ("col_idx", ctypes.c_void_p),
                ("nbmax", ctypes.c_int), ("nnz", ctypes.c_longlong), ("n_blocks", ctypes.c_int * 64)]


_lib = None


class prism_host_io(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("Q", "K", "V", "a_norm", "dO", "O", "lse", "dQ", "dK", "dV")] + [
        ("taylor", ctypes.c_int)]


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libprism.so; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libprism.so not built ({path}); run python -m dynamic_block_sparse_zone_b200.build")
    lib = ctypes.CDLL(path)
    P, V = ctypes.c_void_p, ctypes.c_void_p
    lib.prism_plan_create.argtypes = [ctypes.POINTER(prism_params), ctypes.POINTER(V)]
    lib.prism_plan_bytes.argtypes = [ctypes.POINTER(prism_params)]
    lib.prism_plan_bytes.restype = ctypes.c_size_t
    lib.prism_plan_build.argtypes = [V, P, P, P, P, P]
    lib.prism_attn_fwd.argtypes = [V, P, P, P]
    lib.prism_attn_fwd_taylor.argtypes = [V, P, P, P]
    lib.prism_attn_fwd_taylor.restype = ctypes.c_int
    lib.prism_plan_update_qkv.argtypes = [V, P, P, P, P]
    lib.prism_plan_update_qkv.restype = ctypes.c_int
    lib.prism_attn_bwd.argtypes = [V, P, P, P, P, P, P]
    lib.prism_plan_view_get.argtypes = [V, ctypes.POINTER(prism_plan_view), P]
    lib.prism_plan_check.argtypes = [V, P]
    lib.prism_plan_selftest_timeout.argtypes = [V, P]
    lib.prism_plan_selftest_timeout.restype = ctypes.c_int
    lib.prism_step_host.argtypes = [V, ctypes.POINTER(prism_host_io), P, ctypes.POINTER(ctypes.c_ulonglong)]
    lib.prism_step_host.restype = ctypes.c_int
    lib.prism_step_join.argtypes = [V, ctypes.c_ulonglong, P]
    lib.prism_step_join.restype = ctypes.c_int
    lib.prism_step_wait.argtypes = [V, ctypes.c_ulonglong]
    lib.prism_step_wait.restype = ctypes.c_int
    lib.prism_plan_build_stats.argtypes = [V, P, P, P]
    lib.prism_plan_build_stats.restype = ctypes.c_int
    S = ctypes.POINTER(ctypes.c_size_t)
    lib.prism_plan_stats_slice.argtypes = [V, ctypes.POINTER(ctypes.c_void_p), S, S, S]
    lib.prism_plan_stats_slice.restype = ctypes.c_int
    lib.prism_plan_build_finish.argtypes = [V, P, P, P, P]
    lib.prism_plan_build_finish.restype = ctypes.c_int
    lib.prism_plan_build_with_zones.argtypes = [V, P, P, P, P, P, P]
    lib.prism_plan_build_with_zones.restype = ctypes.c_int
    lib.prism_audio_norms.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, P]
    lib.prism_audio_norms.restype = ctypes.c_int
    lib.prism_plan_destroy.argtypes = [V]
    lib.prism_plan_destroy.restype = None
    lib.prism_last_error.restype = ctypes.c_char_p
    lib.prism_plan_set_timing.argtypes = [V, ctypes.c_int]
    lib.prism_plan_read_timing.argtypes = [V, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int)]
    lib.prism_zone_shapes_noalloc.argtypes = [ctypes.POINTER(prism_params), P, P, P, P, P]
    lib.prism_zone_shapes_noalloc.restype = ctypes.c_int
    lib.prism_timer_name.argtypes = [ctypes.c_int]
    lib.prism_timer_name.restype = ctypes.c_char_p
    for name in ("prism_plan_create", "prism_plan_build", "prism_attn_fwd", "prism_attn_bwd",
                 "prism_plan_view_get", "prism_plan_check", "prism_plan_set_timing", "prism_plan_read_timing"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def _check(status: int):
    if status != PRISM_OK:
        raise PrismError(status, load_library().prism_last_error().decode())


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype, shape):
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous() or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor of shape {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}")


class _DevArray:
    """Zero-copy view of device memory via __cuda_array_interface__."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr, "data": (ptr, False),
                                         "version": 3, "strides": None}


def _dev_tensor(ptr: int, shape, dtype=torch.int32) -> torch.Tensor:
    return _dev_view(ptr, shape, dtype).clone()


def _dev_view(ptr: int, shape, dtype) -> torch.Tensor:
    """Zero-copy tensor over device memory the plan owns (valid while the plan lives)."""
    ts = {torch.int32: "<i4", torch.float64: "<f8"}[dtype]
    return torch.as_tensor(_DevArray(ptr, shape, ts), device="cuda")


@dataclass
class Params:
    batch: int
    T: int
    H: int
    W: int
    heads: int
    head_dim: int
    top_k: int
    top_p: float
    max_frac: float = 0.0
    fixed_shape: Tuple[int, int, int] = (0, 0, 0)
    eps: float = 1e-6
    heads_total: int = 0  # head sharding: this plan holds heads [head_offset, head_offset + heads)
    head_offset: int = 0
    hilbert_block: int = 0  # 64/128/256: Hilbert-order fixed-block plan (DFSAttn-style baseline)

    def to_c(self) -> prism_params:
        return prism_params(self.batch, self.T, self.H, self.W, self.heads, self.head_dim, self.top_k,
                            float(self.top_p), float(self.max_frac), (ctypes.c_int * 3)(*self.fixed_shape),
                            float(self.eps), int(self.heads_total), int(self.head_offset),
                            int(self.hilbert_block))

    @property
    def N(self) -> int:
        return self.T * self.H * self.W


def prism_plan_bytes(params: Params) -> int:
    c = params.to_c()
    return int(load_library().prism_plan_bytes(ctypes.byref(c)))


class PrismPlan:
    """Owns one prism_plan (C handle) and its device buffers."""

    def __init__(self, params: Params):
        self.params = params
        self._c = params.to_c()
        h = ctypes.c_void_p()
        _check(load_library().prism_plan_create(ctypes.byref(self._c), ctypes.byref(h)))
        self._h = h
        self._held = {}  # ticket -> host tensors a queued step reads or writes

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            load_library().prism_plan_destroy(self._h)  # waits for queued host steps
            self._h = None
        self._held = {}

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- shapes -------------------------------------------------------------
    def _qkv_shape(self):
        p = self.params
        return (p.batch, p.N, p.heads, p.head_dim)

    # -- the three hot-path calls ---------------------------------------------
    def build(self, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, a_norm: Optional[torch.Tensor]):
        """a_norm may be None for a Hilbert-order plan (no zone statistics)."""
        p = self.params
        for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
            _need(t, n, torch.bfloat16, self._qkv_shape())
        if a_norm is not None or not p.hilbert_block:
            _need(a_norm, "a_norm", torch.float32, (p.batch, p.T, p.H, p.W))
        _check(load_library().prism_plan_build(self._h, _ptr(Q), _ptr(K), _ptr(V), _ptr(a_norm), _stream()))
        return self

    # -- the build in two halves (head-sharded plans) --------------------------
    def build_stats(self, V: torch.Tensor, a_norm: torch.Tensor):
        p = self.params
        _need(V, "V", torch.bfloat16, self._qkv_shape())
        _need(a_norm, "a_norm", torch.float32, (p.batch, p.T, p.H, p.W))
        _check(load_library().prism_plan_build_stats(self._h, _ptr(V), _ptr(a_norm), _stream()))
        return self

    def stats_slice(self):
        """(whole-layer zone-statistics buffer as a float64 device tensor, this plan's
        slice of it as a view): the tensors alias the plan's memory."""
        buf, off, n, tot = ctypes.c_void_p(), ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
        _check(load_library().prism_plan_stats_slice(self._h, ctypes.byref(buf), ctypes.byref(off), ctypes.byref(n),
                                                     ctypes.byref(tot)))
        whole = _dev_view(buf.value, (tot.value // 8,), torch.float64)
        return whole, whole[off.value // 8:(off.value + n.value) // 8]

    def build_finish(self, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor):
        for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
            _need(t, n, torch.bfloat16, self._qkv_shape())
        _check(load_library().prism_plan_build_finish(self._h, _ptr(Q), _ptr(K), _ptr(V), _stream()))
        return self

    def build_sharded(self, Q, K, V, a_norm, group=None):
        """Head-sharded build: zone statistics of this rank's heads, one all-gather
        of every rank's slice (torch.distributed, ranks holding equal consecutive
        head ranges in rank order), then the rest of the plan."""
        self.build_stats(V, a_norm)
        whole, mine = self.stats_slice()
        exchange_zone_stats(whole, mine, group)
        return self.build_finish(Q, K, V)

    def build_with_zones(self, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, zone_B, zone_shape):
        """The plan from given zone decisions (int arrays [batch, N/512]: volumes
        64/128/256 and candidate-table indices) instead of the zone statistics."""
        p = self.params
        for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
            _need(t, n, torch.bfloat16, self._qkv_shape())
        zB = np.ascontiguousarray(np.asarray(zone_B, dtype=np.int32).reshape(p.batch, p.N // 512))
        zs = np.ascontiguousarray(np.asarray(zone_shape, dtype=np.int32).reshape(p.batch, p.N // 512))
        _check(load_library().prism_plan_build_with_zones(self._h, _ptr(Q), _ptr(K), _ptr(V),
                                                         zB.ctypes.data_as(ctypes.c_void_p),
                                                         zs.ctypes.data_as(ctypes.c_void_p), _stream()))
        return self

    def update_qkv(self, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor):
        """Reuse the plan (zones, shapes, permutation, selection) for new Q, K, V."""
        for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
            _need(t, n, torch.bfloat16, self._qkv_shape())
        _check(load_library().prism_plan_update_qkv(self._h, _ptr(Q), _ptr(K), _ptr(V), _stream()))
        return self

    def fwd(self, O: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, want_lse: bool = True,
            taylor: bool = False):
        """Sparse forward over S_i; with taylor=True the blocks outside S_i are
        added through their pooled keys and mean values (prism_attn_fwd_taylor)."""
        p = self.params
        if O is None:
            O = torch.empty(self._qkv_shape(), dtype=torch.bfloat16, device="cuda")
        _need(O, "O", torch.bfloat16, self._qkv_shape())
        if lse is None and want_lse:
            lse = torch.empty((p.batch, p.heads, p.N), dtype=torch.float32, device="cuda")
        if lse is not None:
            _need(lse, "lse", torch.float32, (p.batch, p.heads, p.N))
        fn = load_library().prism_attn_fwd_taylor if taylor else load_library().prism_attn_fwd
        _check(fn(self._h, _ptr(O), _ptr(lse), _stream()))
        return O, lse

    def bwd(self, O: torch.Tensor, dO: torch.Tensor, dQ=None, dK=None, dV=None):
        shp = self._qkv_shape()
        _need(O, "O", torch.bfloat16, shp)
        _need(dO, "dO", torch.bfloat16, shp)
        dQ = torch.empty(shp, dtype=torch.bfloat16, device="cuda") if dQ is None else dQ
        dK = torch.empty(shp, dtype=torch.bfloat16, device="cuda") if dK is None else dK
        dV = torch.empty(shp, dtype=torch.bfloat16, device="cuda") if dV is None else dV
        for t, n in ((dQ, "dQ"), (dK, "dK"), (dV, "dV")):
            _need(t, n, torch.bfloat16, shp)
        _check(load_library().prism_attn_bwd(self._h, _ptr(O), _ptr(dO), _ptr(dQ), _ptr(dK), _ptr(dV), _stream()))
        return dQ, dK, dV

    # -- steps from host memory (pipelined across calls) ---------------------
    def step_host(self, Q, K, V, a_norm, O, lse=None, dO=None, dQ=None, dK=None, dV=None, taylor=False) -> int:
        """Enqueues one layer step on host tensors (page-locked for overlap) and
        returns its ticket; the tensors are kept alive until step_wait covers it."""
        p = self.params
        shp = self._qkv_shape()
        host = [(Q, "Q", torch.bfloat16, shp), (K, "K", torch.bfloat16, shp), (V, "V", torch.bfloat16, shp),
                (O, "O", torch.bfloat16, shp)]
        if a_norm is not None or not p.hilbert_block:  # a Hilbert-order plan does not read a_norm
            host.append((a_norm, "a_norm", torch.float32, (p.batch, p.T, p.H, p.W)))
        if lse is not None:
            host.append((lse, "lse", torch.float32, (p.batch, p.heads, p.N)))
        if dO is not None:
            if dQ is None or dK is None or dV is None:
                raise ValueError("a step with dO needs dQ, dK and dV")
            host += [(t, n, torch.bfloat16, shp) for t, n in ((dO, "dO"), (dQ, "dQ"), (dK, "dK"), (dV, "dV"))]
        for t, n, dt, sh in host:
            if t.is_cuda or t.dtype != dt or tuple(t.shape) != tuple(sh) or not t.is_contiguous():
                raise ValueError(f"{n}: expected a contiguous host tensor {dt} {tuple(sh)}")
        io = prism_host_io(*(None if t is None else t.data_ptr() for t in (Q, K, V, a_norm, dO, O, lse, dQ, dK, dV)),
                           int(bool(taylor)))
        tk = ctypes.c_ulonglong()
        _check(load_library().prism_step_host(self._h, ctypes.byref(io), _stream(), ctypes.byref(tk)))
        self._held[tk.value] = [t for t, *_ in host]
        return tk.value

    def step_join(self, ticket: int):
        """The current CUDA stream waits (on the device) for step `ticket`."""
        _check(load_library().prism_step_join(self._h, ticket, _stream()))

    def step_wait(self, ticket: int):
        """Blocks until step `ticket` (and every earlier one) has its outputs in host memory."""
        _check(load_library().prism_step_wait(self._h, ticket))
        for t in [t for t in self._held if t <= ticket]:
            del self._held[t]

    # -- per-kernel event timing ---------------------------------------------
    def set_timing(self, enable: bool = True):
        _check(load_library().prism_plan_set_timing(self._h, int(bool(enable))))

    def read_timing(self) -> dict:
        """{kernel name: (total ms, launches)} since the previous read (waits for the events)."""
        lib = load_library()
        ms = (ctypes.c_float * NUM_TIMERS)()
        n = (ctypes.c_int * NUM_TIMERS)()
        _check(lib.prism_plan_read_timing(self._h, ms, n))
        return {lib.prism_timer_name(k).decode(): (float(ms[k]), int(n[k])) for k in range(NUM_TIMERS)}

    # -- inspection ----------------------------------------------------------
    def check(self):
        _check(load_library().prism_plan_check(self._h, _stream()))

    def selftest_timeout(self):
        """Enqueues the bounded-wait diagnostic (the next check() raises PRISM_ERR_TIMEOUT)."""
        _check(load_library().prism_plan_selftest_timeout(self._h, _stream()))

    def view(self) -> dict:
        """Copies of the plan's arrays (syncs the current stream)."""
        v = prism_plan_view()
        _check(load_library().prism_plan_view_get(self._h, ctypes.byref(v), _stream()))
        p = self.params
        M = p.N // 512
        nbmax = v.nbmax
        rows = p.batch * p.heads * nbmax
        return dict(
            zone_B=_dev_tensor(v.zone_B, (p.batch, M)),
            zone_shape=_dev_tensor(v.zone_shape, (p.batch, M)),
            perm=_dev_tensor(v.perm, (p.batch, p.N)),
            blk_off=_dev_tensor(v.blk_off, (p.batch, nbmax + 1)),
            row_ptr=_dev_tensor(v.row_ptr, (rows + 1,)),
            col_idx=_dev_tensor(v.col_idx, (max(int(v.nnz), 1),))[: int(v.nnz)],
            n_blocks=[int(v.n_blocks[b]) for b in range(p.batch)],
            nbmax=nbmax,
        )


def prism_zone_shapes_noalloc(params: Params, V: torch.Tensor, a_norm: torch.Tensor,
                              zone_B: torch.Tensor, zone_shape: torch.Tensor):
    """Zone volumes and shapes without any device allocation inside the call
    (the library's fixed scratch array is used); outputs are caller-owned
    int32 CUDA tensors of shape [batch, N/512]."""
    M = params.N // 512
    _need(V, "V", torch.bfloat16, (params.batch, params.N, params.heads, params.head_dim))
    _need(a_norm, "a_norm", torch.float32, (params.batch, params.T, params.H, params.W))
    _need(zone_B, "zone_B", torch.int32, (params.batch, M))
    _need(zone_shape, "zone_shape", torch.int32, (params.batch, M))
    if not (V.device == a_norm.device == zone_B.device == zone_shape.device):
        raise ValueError("V, a_norm, zone_B and zone_shape must be on one GPU")
    c = params.to_c()
    # the library launches on the current device with that device's copy of
    # its scratch array: make the tensors' GPU current for the call
    with torch.cuda.device(V.device):
        _check(load_library().prism_zone_shapes_noalloc(ctypes.byref(c), _ptr(V), _ptr(a_norm), _ptr(zone_B),
                                                        _ptr(zone_shape), _stream()))
    return zone_B, zone_shape


# Module-level names that mirror the C ABI.
def _through_host(t: torch.Tensor, group) -> bool:
    """gloo moves host tensors only: device tensors then go through host copies
    (NCCL takes them as they are)."""
    import torch.distributed as dist
    return t.is_cuda and dist.get_backend(group) == "gloo"


def exchange_zone_stats(whole: torch.Tensor, mine: torch.Tensor, group=None):
    """All-gather of the ranks' zone-statistics slices into `whole` (rank order =
    slice order).  Single process: nothing to exchange."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return whole
    if _through_host(whole, group):
        host = torch.empty(whole.shape, dtype=whole.dtype)
        dist.all_gather_into_tensor(host, mine.cpu(), group=group)
        whole.copy_(host)
        return whole
    dist.all_gather_into_tensor(whole, mine.clone(), group=group)
    return whole


def _all_to_all(send: torch.Tensor, group) -> torch.Tensor:
    import torch.distributed as dist
    if _through_host(send, group):
        host = send.cpu()
        recv = torch.empty_like(host)
        dist.all_to_all_single(recv, host, group=group)
        return recv.to(send.device)
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    return recv


def sequence_to_heads(x: torch.Tensor, group=None) -> torch.Tensor:
    """Sequence-sharded activations to head-sharded ones for a head-sharded plan:
    x [B, N/R, heads, D] on rank r (tokens [r N/R, (r+1) N/R) of every head)
    becomes [B, N, heads/R, D] (heads [r heads/R, (r+1) heads/R) of every token),
    with one all-to-all (NCCL over NVLink on GPUs).  R = 1: x unchanged."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return x
    R = dist.get_world_size(group)
    B, n, Hn, D = x.shape
    if Hn % R:
        raise ValueError("heads must divide evenly among the ranks")
    h = Hn // R
    send = x.reshape(B, n, R, h, D).permute(2, 0, 1, 3, 4).contiguous()  # [dest rank][B][n][h][D]
    recv = _all_to_all(send, group)                                       # [source rank][B][n][h][D]
    return recv.permute(1, 0, 2, 3, 4).reshape(B, R * n, h, D)


def heads_to_sequence(y: torch.Tensor, group=None) -> torch.Tensor:
    """The inverse of sequence_to_heads (for O and the gradients): y [B, N,
    heads/R, D] on rank r becomes [B, N/R, heads, D]."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return y
    R = dist.get_world_size(group)
    B, N, h, D = y.shape
    if N % R:
        raise ValueError("tokens must divide evenly among the ranks")
    n = N // R
    send = y.reshape(B, R, n, h, D).permute(1, 0, 2, 3, 4).contiguous()  # [dest rank][B][n][h][D]
    recv = _all_to_all(send, group)                                       # [source rank][B][n][h][D]
    return recv.permute(1, 2, 0, 3, 4).reshape(B, n, R * h, D)


def gather_sequence(t: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather of token shards along axis 1 ([B, N/R, ...] -> [B, N, ...]),
    e.g. the audio norms a plan needs for every token."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return t
    R = dist.get_world_size(group)
    host = _through_host(t, group)
    src = t.contiguous().cpu() if host else t.contiguous()
    parts = torch.empty((R * t.shape[0],) + tuple(t.shape[1:]), dtype=t.dtype, device=src.device)
    dist.all_gather_into_tensor(parts, src, group=group)  # rank-major concatenation
    if host:
        parts = parts.to(t.device)
    parts = parts.view((R,) + tuple(t.shape))
    return parts.movedim(0, 1).reshape((t.shape[0], R * t.shape[1]) + tuple(t.shape[2:]))


def prism_audio_norms(h: torch.Tensor, T: int, H: int, W: int, a: Optional[torch.Tensor] = None) -> torch.Tensor:
    """a_{t,h,w} = ||h^_{t,h,w}||_2 for h [batch, T*H*W, channels] bf16 on the current device."""
    if h.dtype != torch.bfloat16 or not h.is_cuda or h.dim() != 3 or not h.is_contiguous():
        raise ValueError("h must be a contiguous [batch, N, channels] bf16 CUDA tensor")
    batch, n, ch = h.shape
    if n != T * H * W:
        raise ValueError("h's token axis must be T*H*W")
    if a is None:
        a = torch.empty((batch, T, H, W), dtype=torch.float32, device=h.device)
    _need(a, "a", torch.float32, (batch, T, H, W))
    _check(load_library().prism_audio_norms(_ptr(h), _ptr(a), batch, T, H, W, ch, _stream()))
    return a


def prism_plan_create(params: Params) -> PrismPlan:
    return PrismPlan(params)


def prism_plan_build(plan: PrismPlan, Q, K, V, a_norm) -> PrismPlan:
    return plan.build(Q, K, V, a_norm)


def prism_attn_fwd(plan: PrismPlan, O=None, lse=None):
    return plan.fwd(O, lse)


def prism_attn_fwd_taylor(plan: PrismPlan, O=None, lse=None):
    return plan.fwd(O, lse, taylor=True)


def prism_attn_bwd(plan: PrismPlan, O, dO, dQ=None, dK=None, dV=None):
    return plan.bwd(O, dO, dQ, dK, dV)


def prism_plan_destroy(plan: PrismPlan):
    plan.close()


def params_for(w, batch: Optional[int] = None, hilbert_block: int = 0) -> Params:
    """Params of a synth.Workload (hilbert_block: the Hilbert-order fixed-block
    plan with blocks of that many tokens instead of Prism's zone plan)."""
    return Params(batch=batch or w.batch, T=w.T, H=w.H, W=w.W, heads=w.heads, head_dim=w.head_dim,
                  top_k=w.top_k, top_p=w.top_p, max_frac=w.max_frac,
                  fixed_shape=(0, 0, 0) if hilbert_block else tuple(w.fixed_shape), hilbert_block=hilbert_block)
