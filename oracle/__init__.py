"""fp64 CPU oracle of Prism's dynamic sparse video self-attention hot path.

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the
benchmark's CPU-baseline / reference arm may import this module; the product
path never does.  It shares no code with the CUDA library.

The arithmetic lives in ``prism_oracle.c`` (plain C, fp64, OpenMP over
independent outer loops); this module compiles it with gcc on first use and
marshals numpy arrays.  ``plan()`` strings the steps together in the order of
the paper guide "Prism: Dynamic Sparse Attention cho Huan luyen Mo hinh Tao
Video-Am thanh Dong thoi Do phan giai Goc 2K", Method sections 1-3.

Parity status: see the header of ``prism_oracle.c``.  The density rho(m), the
audio normalisation and the block order are readings (the pages print no
formula); they are pinned only on special cases.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "prism_oracle.c")
_LIB = os.path.join(_HERE, "_build", "liboracle.so")
_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_D = ctypes.c_double


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, IEEE arithmetic, OpenMP)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        sigs = {
            "orc_shape_table": (_I, [_P]),
            "orc_lstar": (None, [_P, _I, _P]),
            "orc_pick_shape": (_I, [_P, _I, _P]),
            "orc_zone_stats": (None, [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P]),
            "orc_zone_decide": (None, [_I, _P, _P, _P, _D, _D, _I, _P, _P, _P, _P, _P, _P, _P]),
            "orc_blocks": (_I, [_I, _I, _I, _P, _P]),
            "orc_perm": (None, [_I, _I, _I, _I, _P, _P]),
            "orc_pool": (None, [_P, _I, _I, _I, _I, _I, _I, _P, _P]),
            "orc_select_row": (_I, [_P, _I, _I, _D, _I, _P, _P]),
            "orc_cap": (_I, [_I, _I, _D]),
            "orc_select": (None, [_P, _P, _I, _I, _I, _I, _D, _D, _I, _P, _P, _P]),
            "orc_attn_fwd_rows": (None, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _I,
                                         _I, _P, _P, _P, _P]),
            "orc_attn_fwd_taylor_rows": (None, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _I,
                                                _I, _P, _P, _P, _P]),
            "orc_attn_bwd_dq_rows": (None, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P,
                                            _I, _I, _P, _P, _P]),
            "orc_attn_bwd_dkv_rows": (None, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P,
                                             _I, _I, _P, _P, _P, _P]),
            "orc_pool_blocks": (None, [_P, _I, _I, _I, _P, _P, _P]),
            "orc_hilbert_index": (ctypes.c_uint64, [_I, _I, _I, _I]),
            "orc_hilbert_indices": (None, [_P, ctypes.c_longlong, _I, _P]),
            "orc_hilbert_perm": (None, [_I, _I, _I, _P]),
            "orc_audio_norms": (None, [_P, _P, ctypes.c_longlong, _I]),
            "orc_num_threads": (_I, []),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(_load().orc_num_threads())


# --------------------------------------------------------------------------
# Single steps
# --------------------------------------------------------------------------
def shape_table() -> np.ndarray:
    """The 16 candidate shapes as edge exponents, [16, 3] (volumes 64,128,256)."""
    e = np.zeros((16, 3), np.int32)
    n = _load().orc_shape_table(_ptr(e))
    return e[:n]


def lstar(g, S: int) -> np.ndarray:
    g = _c(g, np.float64)
    out = np.zeros(3, np.float64)
    _load().orc_lstar(_ptr(g), S, _ptr(out))
    return out


def pick_shape(l, S: int):
    """Returns (table index, distance^2 margin to the runner-up)."""
    l = _c(l, np.float64)
    gap = np.zeros(1, np.float64)
    idx = _load().orc_pick_shape(_ptr(l), S, _ptr(gap))
    return int(idx), float(gap[0])


def zone_stats(V_bits: np.ndarray, a: np.ndarray, T: int, H: int, W: int):
    """V_bits: [N, C] uint16 (bf16 bits, raster tokens); a: [N] float32."""
    N = T * H * W
    V_bits = _c(V_bits.reshape(N, -1), np.uint16)
    a = _c(a.reshape(N), np.float32)
    C = V_bits.shape[1]
    M = N // 512
    sv = np.zeros((M, 3)); sa = np.zeros((M, 3)); am = np.zeros(M); amax = np.zeros(1)
    _load().orc_zone_stats(_ptr(V_bits), _ptr(a), T, H, W, C, _ptr(sv), _ptr(sa), _ptr(am), _ptr(amax))
    return sv, sa, am, float(amax[0])


def zone_decide(sig_v, sig_a, a_mean, a_max: float, eps: float, fixed: int = -1):
    sig_v = _c(sig_v, np.float64); sig_a = _c(sig_a, np.float64); a_mean = _c(a_mean, np.float64)
    M = a_mean.shape[0]
    g = np.zeros((M, 3)); rho = np.zeros(M); ls = np.zeros((M, 3))
    zB = np.zeros(M, np.int32); zs = np.zeros(M, np.int32)
    gs = np.zeros(M); gr = np.zeros(M)
    _load().orc_zone_decide(M, _ptr(sig_v), _ptr(sig_a), _ptr(a_mean), float(a_max), float(eps),
                            int(fixed), _ptr(g), _ptr(rho), _ptr(ls), _ptr(zB), _ptr(zs),
                            _ptr(gs), _ptr(gr))
    return dict(g=g, rho=rho, lstar=ls, zone_B=zB, zone_shape=zs, gap_shape=gs, gap_rho=gr)


def blocks(T: int, H: int, W: int, zone_shape) -> np.ndarray:
    zs = _c(zone_shape, np.int32)
    box = np.zeros((T * H * W // 64, 6), np.int32)
    nb = _load().orc_blocks(T, H, W, _ptr(zs), _ptr(box))
    return box[:nb].copy()


def perm(T: int, H: int, W: int, box) -> np.ndarray:
    box = _c(box, np.int32)
    p = np.zeros(T * H * W, np.int32)
    _load().orc_perm(T, H, W, box.shape[0], _ptr(box), _ptr(p))
    return p


def pool(X_bits: np.ndarray, T: int, H: int, W: int, heads: int, D: int, box) -> np.ndarray:
    X_bits = _c(X_bits, np.uint16)
    box = _c(box, np.int32)
    nb = box.shape[0]
    out = np.zeros((heads, nb, D))
    _load().orc_pool(_ptr(X_bits), T, H, W, heads, D, nb, _ptr(box), _ptr(out))
    return out


def cap(nb: int, k: int, max_frac: float) -> int:
    return int(_load().orc_cap(nb, k, float(max_frac)))


def select_row(z, k: int, p: float, cap_: int):
    z = _c(z, np.float64)
    nb = z.shape[0]
    sel = np.zeros(nb, np.int32)
    diag = np.zeros(3)
    n = _load().orc_select_row(_ptr(z), nb, k, float(p), cap_, _ptr(sel), _ptr(diag))
    return sel[:n].copy(), diag


def select(Qbar, Kbar, k: int, p: float, max_frac: float):
    """Returns (cnt [h, nb], cols [h, nb, stride] (padded with -1), diag [h, nb, 3])."""
    Qbar = _c(Qbar, np.float64); Kbar = _c(Kbar, np.float64)
    heads, nb, D = Qbar.shape
    stride = cap(nb, k, max_frac)
    cnt = np.zeros((heads, nb), np.int32)
    cols = np.full((heads, nb, stride), -1, np.int32)
    diag = np.zeros((heads, nb, 3))
    _load().orc_select(_ptr(Qbar), _ptr(Kbar), heads, nb, D, k, float(p), float(max_frac),
                       stride, _ptr(cnt), _ptr(cols), _ptr(diag))
    return cnt, cols, diag


# --------------------------------------------------------------------------
# Whole plan
# --------------------------------------------------------------------------
@dataclass
class OraclePlan:
    T: int
    H: int
    W: int
    heads: int
    D: int
    sig_v: np.ndarray
    sig_a: np.ndarray
    a_mean: np.ndarray
    a_max: float
    g: np.ndarray
    rho: np.ndarray
    lstar: np.ndarray
    zone_B: np.ndarray
    zone_shape: np.ndarray
    gap_shape: np.ndarray
    gap_rho: np.ndarray
    box: np.ndarray
    perm: np.ndarray
    Qbar: np.ndarray
    Kbar: np.ndarray
    cnt: np.ndarray
    cols: np.ndarray
    diag: np.ndarray

    @property
    def nb(self) -> int:
        return int(self.box.shape[0])

    def blk_off(self) -> np.ndarray:
        sizes = self.box[:, 3] * self.box[:, 4] * self.box[:, 5]
        return np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)

    def row_sets(self, h: int):
        return [self.cols[h, i, : self.cnt[h, i]] for i in range(self.nb)]


def plan(Q_bits, K_bits, V_bits, a, T, H, W, heads, D, k, p, max_frac=0.0,
         eps=1e-6, fixed_shape=None, with_select=True, zone_decisions=None) -> OraclePlan:
    """Full oracle plan for one sample.  *_bits: [N, heads, D] uint16 (bf16).

    zone_decisions: optional (zone_B, zone_shape) per zone that replace the
    volumes and shapes Method sections 1-2 derive from the statistics; the
    block table, permutation, pooling and selection (Method sections 2-3)
    then follow from them, so the later steps can be checked on their own.
    The statistics are still computed and returned; the tie gaps are +inf."""
    N = T * H * W
    sv, sa, am, amax = zone_stats(V_bits.reshape(N, heads * D), a, T, H, W)
    fixed = -1
    if fixed_shape is not None and any(fixed_shape):
        ex = tuple(int(np.log2(e)) for e in fixed_shape)
        table = [tuple(r) for r in shape_table()]
        fixed = table.index(ex)
    dec = zone_decide(sv, sa, am, amax, eps, fixed)
    if zone_decisions is not None:
        zB = np.asarray(zone_decisions[0], np.int32).reshape(-1)
        zs = np.asarray(zone_decisions[1], np.int32).reshape(-1)
        table = shape_table()
        if zB.shape != dec["zone_B"].shape or zs.shape != zB.shape:
            raise ValueError("zone_decisions: one volume and one shape per zone")
        if np.any((zs < 0) | (zs >= len(table))):
            raise ValueError("zone_decisions: shape index outside the candidate table")
        if np.any(zB != (1 << table[zs].sum(axis=1))):
            raise ValueError("zone_decisions: a volume differs from its shape's")
        dec = dict(dec, zone_B=zB.copy(), zone_shape=zs.copy(),
                   gap_shape=np.full(zB.shape, np.inf), gap_rho=np.full(zB.shape, np.inf))
    box = blocks(T, H, W, dec["zone_shape"])
    pm = perm(T, H, W, box)
    Qb = pool(Q_bits.reshape(N, heads, D), T, H, W, heads, D, box)
    Kb = pool(K_bits.reshape(N, heads, D), T, H, W, heads, D, box)
    if with_select:
        cnt, cols, diag = select(Qb, Kb, k, p, max_frac)
    else:
        cnt = cols = diag = None
    return OraclePlan(T, H, W, heads, D, sv, sa, am, amax, dec["g"], dec["rho"], dec["lstar"],
                      dec["zone_B"], dec["zone_shape"], dec["gap_shape"], dec["gap_rho"], box, pm,
                      Qb, Kb, cnt, cols, diag)


def pool_blocks(X_bits: np.ndarray, heads: int, D: int, perm, blk_off) -> np.ndarray:
    """fp64 means of blocks given as perm runs: [heads, nb, D]."""
    X_bits = _c(X_bits, np.uint16)
    perm = _c(perm, np.int32)
    off = _c(blk_off, np.int32)
    nb = off.shape[0] - 1
    out = np.zeros((heads, nb, D))
    _load().orc_pool_blocks(_ptr(X_bits), heads, D, nb, _ptr(perm), _ptr(off), _ptr(out))
    return out


def hilbert_indices(pts, k: int) -> np.ndarray:
    """Hilbert index of each point (t, h, w) of the 2^k cube ([n, 3] ints)."""
    pts = _c(pts, np.int32).reshape(-1, 3)
    out = np.zeros(pts.shape[0], np.uint64)
    _load().orc_hilbert_indices(_ptr(pts), ctypes.c_longlong(pts.shape[0]), k, _ptr(out))
    return out


def hilbert_perm(T: int, H: int, W: int) -> np.ndarray:
    """Raster indices of the grid's tokens in the order of the Hilbert curve of
    the smallest enclosing 2^k cube [DFSAttn page, first component]."""
    p = np.zeros(T * H * W, np.int32)
    _load().orc_hilbert_perm(T, H, W, _ptr(p))
    return p


@dataclass
class HilbertPlan:
    """Hilbert-order fixed-block plan: blocks are runs of `bsize` tokens of the
    curve's order; pooling, selection and attention as in Prism's plan."""
    T: int
    H: int
    W: int
    heads: int
    D: int
    bsize: int
    perm: np.ndarray
    Qbar: np.ndarray
    Kbar: np.ndarray
    cnt: np.ndarray
    cols: np.ndarray
    diag: np.ndarray

    @property
    def nb(self) -> int:
        return self.T * self.H * self.W // self.bsize

    def blk_off(self) -> np.ndarray:
        return np.arange(0, self.T * self.H * self.W + 1, self.bsize, dtype=np.int64)

    def row_sets(self, h: int):
        return [self.cols[h, i, : self.cnt[h, i]] for i in range(self.nb)]


def plan_hilbert(Q_bits, K_bits, V_bits, T, H, W, heads, D, bsize, k, p, max_frac=0.0,
                 with_select=True) -> HilbertPlan:
    """Hilbert-order fixed-block plan for one sample (V is not needed: there are
    no zone statistics).  *_bits: [N, heads, D] uint16 (bf16)."""
    N = T * H * W
    assert N % bsize == 0
    pm = hilbert_perm(T, H, W)
    off = np.arange(0, N + 1, bsize)
    Qb = pool_blocks(Q_bits.reshape(N, heads, D), heads, D, pm, off)
    Kb = pool_blocks(K_bits.reshape(N, heads, D), heads, D, pm, off)
    if with_select:
        cnt, cols, diag = select(Qb, Kb, k, p, max_frac)
    else:
        cnt = cols = diag = None
    return HilbertPlan(T, H, W, heads, D, bsize, pm, Qb, Kb, cnt, cols, diag)


def audio_norms(h_bits: np.ndarray) -> np.ndarray:
    """a_{t,h,w} = ||h^_{t,h,w}||_2 over the last axis of bf16 bits h_bits [..., C]
    (fp64, channel order) [Prism guide, Method section 1]."""
    C = h_bits.shape[-1]
    hb = _c(h_bits.reshape(-1, C), np.uint16)
    out = np.empty(hb.shape[0], np.float64)
    lib = _load()
    lib.orc_audio_norms(_ptr(hb), _ptr(out), ctypes.c_longlong(hb.shape[0]), _I(C))
    return out.reshape(h_bits.shape[:-1])


# --------------------------------------------------------------------------
# Attention on requested outputs
# --------------------------------------------------------------------------
def _attn_args(pl):
    """Blocks as perm / blk_off runs, and the selection arrays, of a plan
    (OraclePlan, HilbertPlan or any object with the same fields)."""
    perm = _c(pl.perm, np.int32)
    off = _c(pl.blk_off(), np.int32)
    cnt = _c(pl.cnt, np.int32)
    cols = _c(np.where(pl.cols < 0, 0, pl.cols), np.int32)
    return perm, off, cnt, cols, cols.shape[-1]


def attn_fwd_rows(pl: OraclePlan, Q_bits, K_bits, V_bits, req_h, req_tok):
    """O [n, D] and LSE [n] of query tokens req_tok (raster index) of heads req_h."""
    perm, off, cnt, cols, stride = _attn_args(pl)
    req_h = _c(req_h, np.int32); req_tok = _c(req_tok, np.int32)
    n = req_h.shape[0]
    O = np.zeros((n, pl.D)); lse = np.zeros(n)
    Qb = _c(Q_bits, np.uint16); Kb = _c(K_bits, np.uint16); Vb = _c(V_bits, np.uint16)
    _load().orc_attn_fwd_rows(_ptr(Qb), _ptr(Kb), _ptr(Vb), pl.T, pl.H, pl.W, pl.heads, pl.D, pl.nb,
                              _ptr(perm), _ptr(off), _ptr(cnt), _ptr(cols), stride, n, _ptr(req_h),
                              _ptr(req_tok), _ptr(O), _ptr(lse))
    return O, lse


def attn_fwd_taylor_rows(pl: OraclePlan, Q_bits, K_bits, V_bits, req_h, req_tok):
    """O [n, D] and LSE [n] with the blocks outside each S_i added through a
    zeroth-order Taylor term (pooled key, mean value, weight |B_j|)
    [In-Context Sparse Attention article, grouped computation]."""
    perm, off, cnt, cols, stride = _attn_args(pl)
    req_h = _c(req_h, np.int32); req_tok = _c(req_tok, np.int32)
    n = req_h.shape[0]
    O = np.zeros((n, pl.D)); lse = np.zeros(n)
    Qb = _c(Q_bits, np.uint16); Kb = _c(K_bits, np.uint16); Vb = _c(V_bits, np.uint16)
    _load().orc_attn_fwd_taylor_rows(_ptr(Qb), _ptr(Kb), _ptr(Vb), pl.T, pl.H, pl.W, pl.heads, pl.D,
                                     pl.nb, _ptr(perm), _ptr(off), _ptr(cnt), _ptr(cols), stride, n, _ptr(req_h),
                                     _ptr(req_tok), _ptr(O), _ptr(lse))
    return O, lse


def attn_bwd_dq_rows(pl: OraclePlan, Q_bits, K_bits, V_bits, dO_bits, req_h, req_tok):
    perm, off, cnt, cols, stride = _attn_args(pl)
    req_h = _c(req_h, np.int32); req_tok = _c(req_tok, np.int32)
    n = req_h.shape[0]
    dQ = np.zeros((n, pl.D))
    arrs = [_c(x, np.uint16) for x in (Q_bits, K_bits, V_bits, dO_bits)]
    _load().orc_attn_bwd_dq_rows(*[_ptr(x) for x in arrs], pl.T, pl.H, pl.W, pl.heads, pl.D, pl.nb,
                                 _ptr(perm), _ptr(off), _ptr(cnt), _ptr(cols), stride, n, _ptr(req_h),
                                 _ptr(req_tok), _ptr(dQ))
    return dQ


def attn_bwd_dkv_rows(pl: OraclePlan, Q_bits, K_bits, V_bits, dO_bits, req_h, req_tok):
    perm, off, cnt, cols, stride = _attn_args(pl)
    req_h = _c(req_h, np.int32); req_tok = _c(req_tok, np.int32)
    n = req_h.shape[0]
    dK = np.zeros((n, pl.D)); dV = np.zeros((n, pl.D))
    arrs = [_c(x, np.uint16) for x in (Q_bits, K_bits, V_bits, dO_bits)]
    _load().orc_attn_bwd_dkv_rows(*[_ptr(x) for x in arrs], pl.T, pl.H, pl.W, pl.heads, pl.D, pl.nb,
                                  _ptr(perm), _ptr(off), _ptr(cnt), _ptr(cols), stride, n, _ptr(req_h),
                                  _ptr(req_tok), _ptr(dK), _ptr(dV))
    return dK, dV
