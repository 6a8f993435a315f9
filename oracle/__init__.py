"""fp64 CPU oracle for the activation-sparse gated FFN (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports it, and it imports nothing from the product.

The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP over independent
rows); this module is argument marshalling (ctypes) plus ``build()``.  What
each function computes, and which passage of "Sparser, Faster, Lighter
Transformer Language Models" it follows, is stated in ``oracle.c``.

Pins (tests/test_oracle_*.py) tie every function to something other than
itself: brute force on tiny inputs, numpy float64 matmul, torch float64
autograd, central finite differences, torch's dtype casts, closed-form special
cases (zero density, full density) and the format invariants.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

VAL_F64, VAL_F32, VAL_BF16, VAL_F16 = 0, 1, 2, 3

_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, -O2 -fopenmp)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(_LIB)
        P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        sig = {
            "oracle_round_value": (ctypes.c_double, [ctypes.c_double, I]),
            "oracle_round_array": (None, [P, I64, I, P]),
            "oracle_gate_preact": (None, [P, P, I64, I64, I64, P]),
            "oracle_twell_pack": (I64, [P, I64, I64, I, I, I, P, P, P]),
            "oracle_twell_unpack": (None, [P, P, P, I64, I64, I, I, P]),
            "oracle_fused_up_down": (None, [P, P, P, P, P, P, I64, I64, I64, I, I, P]),
            "oracle_dense_ffn": (None, [P, P, P, P, I64, I64, I64, P]),
            "oracle_hybrid_pack": (I64, [P, P, P, I64, I64, I, I, I, I, P, P, P, P, P, P]),
            "oracle_hybrid_fwd": (None, [P, P, P, P, P, P, P, P, I64, I64, I64, I, P, P, P]),
            "oracle_hybrid_bwd": (None, [P, P, P, P, P, P, P, P, P, P, P, P, I64, I64, I64, I,
                                         P, P, P, P, P, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(_lib, name)
            fn.restype = res
            fn.argtypes = args
    return _lib


def _f64(a) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def round_value(v: float, kind: int) -> float:
    return _load().oracle_round_value(float(v), int(kind))


def round_array(v, kind: int) -> np.ndarray:
    v = _f64(v)
    out = np.empty_like(v)
    _load().oracle_round_array(_p(v), v.size, kind, _p(out))
    return out


def gate_preact(x, wg_t) -> np.ndarray:
    """G = x W_gate, [N][F] fp64."""
    x, wg_t = _f64(x), _f64(wg_t)
    n, d = x.shape
    f = wg_t.shape[0]
    assert wg_t.shape[1] == d
    g = np.empty((n, f), np.float64)
    _load().oracle_gate_preact(_p(x), _p(wg_t), n, d, f, _p(g))
    return g


class TwELL:
    """Host TwELL buffers: count [N][F/T], idx [N][F/T][C], val [N][F/T][C]."""

    def __init__(self, count, idx, val, tile, cap, overflow=0):
        self.count, self.idx, self.val = count, idx, val
        self.tile, self.cap, self.overflow = tile, cap, overflow

    @property
    def n_rows(self):
        return self.count.shape[0]

    @property
    def n_cols(self):
        return self.count.shape[1] * self.tile


def twell_pack(g, tile: int, cap: int, val_kind: int = VAL_F64) -> TwELL:
    g = _f64(g)
    n, f = g.shape
    assert f % tile == 0 and 0 < cap <= tile <= 255
    nt = f // tile
    count = np.zeros((n, nt), np.uint8)
    idx = np.zeros((n, nt, cap), np.uint8)
    val = np.zeros((n, nt, cap), np.float64)
    ov = _load().oracle_twell_pack(_p(g), n, f, tile, cap, val_kind, _p(count), _p(idx), _p(val))
    return TwELL(count, idx, val, tile, cap, int(ov))


def twell_unpack(tw: TwELL) -> np.ndarray:
    n, f = tw.n_rows, tw.n_cols
    h = np.empty((n, f), np.float64)
    _load().oracle_twell_unpack(_p(np.ascontiguousarray(tw.count)), _p(np.ascontiguousarray(tw.idx)),
                                _p(_f64(tw.val)), n, f, tw.tile, tw.cap, _p(h))
    return h


def fused_up_down(x, tw: TwELL, wu_t, wd) -> np.ndarray:
    x, wu_t, wd = _f64(x), _f64(wu_t), _f64(wd)
    n, d = x.shape
    f = wu_t.shape[0]
    assert tw.n_rows == n and tw.n_cols == f and wd.shape == (f, d)
    y = np.empty((n, d), np.float64)
    _load().oracle_fused_up_down(_p(x), _p(np.ascontiguousarray(tw.count)),
                                 _p(np.ascontiguousarray(tw.idx)), _p(_f64(tw.val)),
                                 _p(wu_t), _p(wd), n, d, f, tw.tile, tw.cap, _p(y))
    return y


def dense_ffn(x, wg_t, wu_t, wd) -> np.ndarray:
    x, wg_t, wu_t, wd = _f64(x), _f64(wg_t), _f64(wu_t), _f64(wd)
    n, d = x.shape
    f = wg_t.shape[0]
    y = np.empty((n, d), np.float64)
    _load().oracle_dense_ffn(_p(x), _p(wg_t), _p(wu_t), _p(wd), n, d, f, _p(y))
    return y


def sparse_ffn(x, wg_t, wu_t, wd, tile: int, cap: int, val_kind: int):
    """The whole inference forward: G, TwELL pack, fused up/down."""
    g = gate_preact(x, wg_t)
    tw = twell_pack(g, tile, cap, val_kind)
    return fused_up_down(x, tw, wu_t, wd), tw, g


class Hybrid:
    def __init__(self, **kw):
        self.__dict__.update(kw)


def hybrid_pack(tw: TwELL, k: int, s_max: int) -> Hybrid:
    n, f = tw.n_rows, tw.n_cols
    row_nnz = np.zeros(n, np.int32)
    spill_slot = np.zeros(n, np.int32)
    spill_rows = np.full(max(s_max, 1), -1, np.int32)
    ell_idx = np.zeros((n, max(k, 1)), np.int32)
    ell_a = np.zeros((n, max(k, 1)), np.float64)
    spill_a = np.zeros((max(s_max, 1), f), np.float64)
    r = _load().oracle_hybrid_pack(_p(np.ascontiguousarray(tw.count)), _p(np.ascontiguousarray(tw.idx)),
                                   _p(_f64(tw.val)), n, f, tw.tile, tw.cap, k, s_max,
                                   _p(row_nnz), _p(spill_slot), _p(spill_rows), _p(ell_idx),
                                   _p(ell_a), _p(spill_a))
    n_spill, dropped = int(r & 0xFFFFFFFF), int(r >> 32)
    return Hybrid(n_rows=n, n_cols=f, k=k, s_max=s_max, row_nnz=row_nnz, spill_slot=spill_slot,
                  spill_rows=spill_rows[:min(n_spill, s_max)], n_spill=n_spill, dropped=dropped,
                  ell_idx=ell_idx[:, :k], ell_a=ell_a[:, :k], spill_a=spill_a[:s_max])


def hybrid_fwd(x, hy: Hybrid, wu_t, wd):
    """Returns y; fills hy.ell_u and hy.spill_u."""
    x, wu_t, wd = _f64(x), _f64(wu_t), _f64(wd)
    n, d = x.shape
    f, k = hy.n_cols, hy.k
    kk = max(k, 1)
    ell_idx = np.zeros((n, kk), np.int32); ell_idx[:, :k] = hy.ell_idx
    ell_a = np.zeros((n, kk)); ell_a[:, :k] = hy.ell_a
    spill_a = np.zeros((max(hy.s_max, 1), f)); spill_a[:hy.s_max] = hy.spill_a
    ell_u = np.zeros((n, kk))
    spill_u = np.zeros((max(hy.s_max, 1), f))
    y = np.empty((n, d))
    _load().oracle_hybrid_fwd(_p(x), _p(hy.row_nnz), _p(hy.spill_slot), _p(ell_idx), _p(ell_a),
                              _p(spill_a), _p(wu_t), _p(wd), n, d, f, k, _p(ell_u), _p(spill_u), _p(y))
    hy.ell_u = ell_u[:, :k]
    hy.spill_u = spill_u[:hy.s_max]
    return y


def hybrid_bwd(x, dy, hy: Hybrid, wg_t, wu_t, wd):
    """Returns dx, dwg_t, dwu_t, dwd (all fp64; weight grads neuron-major)."""
    x, dy, wg_t, wu_t, wd = map(_f64, (x, dy, wg_t, wu_t, wd))
    n, d = x.shape
    f, k = hy.n_cols, hy.k
    kk = max(k, 1)
    ell_idx = pad(hy.ell_idx, (n, kk))
    ell_a = pad(_f64(hy.ell_a), (n, kk))
    ell_u = pad(_f64(hy.ell_u), (n, kk))
    spill_a = pad(_f64(hy.spill_a), (max(hy.s_max, 1), f))
    spill_u = pad(_f64(hy.spill_u), (max(hy.s_max, 1), f))
    dx = np.empty((n, d)); dwg = np.empty((f, d)); dwu = np.empty((f, d)); dwd = np.empty((f, d))
    du = np.empty((n, f)); dg = np.empty((n, f))
    _load().oracle_hybrid_bwd(_p(x), _p(dy), _p(hy.row_nnz), _p(hy.spill_slot), _p(ell_idx),
                              _p(ell_a), _p(ell_u), _p(spill_a), _p(spill_u), _p(wg_t), _p(wu_t),
                              _p(wd), n, d, f, k, _p(dx), _p(dwg), _p(dwu), _p(dwd), _p(du), _p(dg))
    return dx, dwg, dwu, dwd


def pad(a: np.ndarray, shape) -> np.ndarray:
    z = np.zeros(shape, a.dtype)
    z[tuple(slice(0, s) for s in a.shape)] = a
    return z


def max_abs_rel(a, b) -> float:
    """max_i |a_i - b_i| / max_i |b_i| (b the oracle; 0/0 counts as 0)."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = float(np.max(np.abs(b))) if b.size else 0.0
    num = float(np.max(np.abs(a - b))) if b.size else 0.0
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return num / den
