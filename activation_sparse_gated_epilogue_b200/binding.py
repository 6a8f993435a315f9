"""ctypes binding of libsge.so: argument marshalling only.

Each function has the name of the C entry point it calls and takes torch
tensors on a CUDA device; outputs not given are allocated with torch (device
memory is the only thing PyTorch provides here) and returned.  Launches go on
the current torch stream of the tensors' device unless ``stream`` is given.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

SGE_F32, SGE_BF16 = 0, 1
_DTYPES = {torch.float32: SGE_F32, torch.bfloat16: SGE_BF16}

_HERE = os.path.dirname(os.path.abspath(__file__))
# SGE_DEBUG=1 loads the debug build (index checks in every kernel, read with
# debug_flags); it is built by ``python -m activation_sparse_gated_epilogue_b200.build --debug``
_LIB_PATH = os.path.join(_HERE, "libsge_debug.so" if os.environ.get("SGE_DEBUG") == "1" else "libsge.so")
_lib = None


class _SgeHybrid(ctypes.Structure):
    """Mirror of `sge_hybrid` in include/sge.h."""
    _fields_ = [("n_tokens", ctypes.c_int64), ("d_ff", ctypes.c_int64),
                ("ell_cap", ctypes.c_int32), ("s_max", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("row_nnz", ctypes.c_void_p), ("spill_slot", ctypes.c_void_p),
                ("spill_rows", ctypes.c_void_p), ("n_spill", ctypes.c_void_p),
                ("ell_idx", ctypes.c_void_p), ("ell_a", ctypes.c_void_p),
                ("ell_u", ctypes.c_void_p), ("spill_a", ctypes.c_void_p),
                ("spill_u", ctypes.c_void_p)]


class LibraryError(RuntimeError):
    """A C entry point returned an error code (message from sge_last_error)."""

    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed (code {code}): {msg}")
        self.code = code


def library_path() -> str:
    return _LIB_PATH


def library() -> ctypes.CDLL:
    """Load libsge.so (built in-tree by ``python -m
    activation_sparse_gated_epilogue_b200.build``); raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                               "`python -m activation_sparse_gated_epilogue_b200.build`")
        lib = ctypes.CDLL(_LIB_PATH)
        P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        sigs = {
            "sge_version": (I, []),
            "sge_debug_flags": (I, [I]),
            "sge_last_error": (ctypes.c_char_p, []),
            "twell_gate_pack": (I, [P, P, I64, I64, I64, I, I, I, P, P, P, P, P]),
            "twell_fused_up_down_workspace_bytes": (ctypes.c_size_t, [I64, I64]),
            "twell_fused_up_down": (I, [P, P, P, P, P, P, I64, P, I64, I64, I64, I, I, I, P,
                                        ctypes.c_size_t, P, P]),
            "twell_fused_up_down_noalloc": (I, [P, P, P, P, P, P, I64, P, I64, I64, I64, I, I, I,
                                                P, P]),
            "sge_interleave_up_down": (I, [P, P, P, I64, I64, I, P]),
            "twell_hybrid_up_down_workspace_bytes": (ctypes.c_size_t, [I64, I64, I64, I]),
            "twell_hybrid_up_down": (I, [P, P, P, P, P, P, I64, P, P, I64, I64, I64, I, I, I, I, P,
                                         ctypes.c_size_t, P, P]),
            "twell_fused_up_down_noalloc_max_tokens": (I64, []),
            "dense_ffn_fwd": (I, [P, P, P, P, P, P, I64, I64, I64, P, P]),
            "hybrid_pack": (I, [P, P, P, I, I, ctypes.POINTER(_SgeHybrid), P, P]),
            "hybrid_ffn_fwd_workspace_bytes": (ctypes.c_size_t, [I64, I64, I]),
            "hybrid_ffn_fwd": (I, [P, ctypes.POINTER(_SgeHybrid), P, P, P, P, P, I64, P,
                                   ctypes.c_size_t, P]),
            "hybrid_ffn_bwd_workspace_bytes": (ctypes.c_size_t, [I64, I64, I64, I, I]),
            "hybrid_ffn_bwd": (I, [P, P, ctypes.POINTER(_SgeHybrid), P, P, P, P, P, P, P, P, I64, P,
                                   ctypes.c_size_t, P]),
            "sge_transpose_up_gate": (I, [P, P, P, I64, I64, P]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def debug_flags(clear: bool = True) -> int:
    """OR of the SGE_FLAG_* bits the debug build's index checks raised since
    the last clear (synchronises the device); -1 with the release build."""
    r = library().sge_debug_flags(1 if clear else 0)
    if r == -2:
        raise LibraryError("sge_debug_flags", 3, library().sge_last_error().decode())
    return r


def _call(name: str, *args) -> None:
    lib = library()
    rc = getattr(lib, name)(*args)
    if rc != 0:
        raise LibraryError(name, rc, lib.sge_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(t: torch.Tensor, name: str, dtype=None, shape=None) -> torch.Tensor:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _check_rows(t: torch.Tensor, name: str, dtype, shape) -> int:
    """A 2-D matrix of `shape` whose rows are contiguous (any row stride);
    returns the row stride in elements."""
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path)")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.stride(1) != 1 and t.shape[1] > 1:
        raise ValueError(f"{name} must have contiguous rows")
    return t.stride(0) if t.shape[0] > 1 else t.shape[1]


def _stream(dev: torch.device, stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream(dev) if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {t.dtype}")
    return _DTYPES[t.dtype]


def new_diag(device) -> torch.Tensor:
    """A zeroed int32[4] diagnostics word (see include/sge.h)."""
    return torch.zeros(4, dtype=torch.int32, device=device)


@dataclass
class TwELL:
    """Device TwELL buffers: count [N][F/T] u8, idx [N][F/T][C] u8,
    val [N][F/T][C] in the activation dtype."""
    count: torch.Tensor
    idx: torch.Tensor
    val: torch.Tensor
    tile: int
    cap: int

    @property
    def n_rows(self) -> int:
        return self.count.shape[0]

    @property
    def n_cols(self) -> int:
        return self.count.shape[1] * self.tile

    @staticmethod
    def empty(n: int, f: int, tile: int, cap: int, dtype, device) -> "TwELL":
        nt = f // tile
        return TwELL(torch.empty((n, nt), dtype=torch.uint8, device=device),
                     torch.empty((n, nt, cap), dtype=torch.uint8, device=device),
                     torch.empty((n, nt, cap), dtype=dtype, device=device), tile, cap)


def twell_gate_pack(x: torch.Tensor, wg_t: torch.Tensor, tile: int, cap: int,
                    out: Optional[TwELL] = None, diag: Optional[torch.Tensor] = None,
                    stream=None) -> TwELL:
    """TwELL of ReLU(x W_gate), produced in the gate GEMM's epilogue."""
    _check(x, "x")
    n, d = x.shape
    f = wg_t.shape[0]
    _check(wg_t, "wg_t", x.dtype, (f, d))
    if out is None:
        out = TwELL.empty(n, f, tile, cap, x.dtype, x.device)
    else:
        _check(out.count, "count", torch.uint8, (n, f // tile))
        _check(out.idx, "idx", torch.uint8, (n, f // tile, cap))
        _check(out.val, "val", x.dtype, (n, f // tile, cap))
    if diag is not None:
        _check(diag, "diag", torch.int32, (4,))
    _call("twell_gate_pack", _ptr(x), _ptr(wg_t), n, d, f, _dtype_code(x), tile, cap,
          _ptr(out.count), _ptr(out.idx), _ptr(out.val), _ptr(diag), _stream(x.device, stream))
    return out


def fused_workspace(n_tokens: int, d_model: int, device) -> torch.Tensor:
    """Scratch for twell_fused_up_down (entry counts, job lists, fp32 partial
    outputs of split heavy tokens, counters)."""
    nbytes = library().twell_fused_up_down_workspace_bytes(n_tokens, d_model)
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)


def interleave_up_down(wu_t: torch.Tensor, wd: torch.Tensor, stream=None):
    """The interleaved weight layout twell_fused_up_down streams fastest:
    returns (w_ud, wu_view, wd_view), w_ud [F][2d] with row j = wu_t[j] then
    wd[j], and the two [F][d] views of it (row stride 2d) to pass as wu_t and
    wd.  A weight-loading step, done once."""
    _check(wu_t, "wu_t")
    f, d = wu_t.shape
    _check(wd, "wd", wu_t.dtype, (f, d))
    w_ud = torch.empty((f, 2 * d), dtype=wu_t.dtype, device=wu_t.device)
    _call("sge_interleave_up_down", _ptr(wu_t), _ptr(wd), _ptr(w_ud), f, d, _dtype_code(wu_t),
          _stream(wu_t.device, stream))
    return w_ud, w_ud[:, :d], w_ud[:, d:]


def twell_fused_up_down(x: torch.Tensor, tw: TwELL, wu_t: torch.Tensor, wd: torch.Tensor,
                        y: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                        diag: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """y = sum over TwELL entries of a * (x . W_up[:, j]) * W_down[j] (h never stored).
    wu_t and wd may be row-strided views with one row stride, e.g. the two
    halves of interleave_up_down's matrix."""
    _check(x, "x")
    n, d = x.shape
    f = wu_t.shape[0]
    ldw = _check_rows(wu_t, "wu_t", x.dtype, (f, d))
    if _check_rows(wd, "wd", x.dtype, (f, d)) != ldw:
        raise ValueError("wu_t and wd must have the same row stride")
    _check(tw.count, "count", torch.uint8, (n, f // tw.tile))
    _check(tw.idx, "idx", torch.uint8, (n, f // tw.tile, tw.cap))
    _check(tw.val, "val", x.dtype, (n, f // tw.tile, tw.cap))
    if y is None:
        y = torch.empty_like(x)
    _check(y, "y", x.dtype, (n, d))
    if workspace is None:
        workspace = fused_workspace(n, d, x.device)
    _check(workspace, "workspace", torch.uint8)
    if diag is not None:
        _check(diag, "diag", torch.int32, (4,))
    _call("twell_fused_up_down", _ptr(x), _ptr(tw.count), _ptr(tw.idx), _ptr(tw.val),
          _ptr(wu_t), _ptr(wd), ldw, _ptr(y), n, d, f, _dtype_code(x), tw.tile, tw.cap,
          _ptr(workspace), workspace.numel(), _ptr(diag), _stream(x.device, stream))
    return y


def routed_workspace(n_tokens: int, d_model: int, d_ff: int, s_max: int, device) -> torch.Tensor:
    """Scratch for twell_hybrid_up_down (the caching allocator's blocks are
    512-byte aligned; 256 are needed)."""
    nbytes = library().twell_hybrid_up_down_workspace_bytes(n_tokens, d_model, d_ff, s_max)
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def twell_hybrid_up_down(x: torch.Tensor, tw: TwELL, wu_t: torch.Tensor, wd: torch.Tensor,
                         wd_t: Optional[torch.Tensor], ell_cap: int, s_max: int,
                         y: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                         diag: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """y from TwELL with tokens of more than ell_cap stored entries (the first
    s_max of them) on the tensor-core spill GEMMs and the others per entry on
    CUDA cores (batches of at most 64 tokens: every token per entry).  bf16.  ``wd_t`` is W_down transposed, [d][F]
    (None only when s_max == 0); wu_t and wd may be the row-strided halves of
    interleave_up_down's matrix."""
    _check(x, "x", torch.bfloat16)
    n, d = x.shape
    f = wu_t.shape[0]
    ldw = _check_rows(wu_t, "wu_t", x.dtype, (f, d))
    if _check_rows(wd, "wd", x.dtype, (f, d)) != ldw:
        raise ValueError("wu_t and wd must have the same row stride")
    if wd_t is None:
        if s_max > 0:
            raise ValueError("wd_t (W_down transposed, [d][F]) is required when s_max > 0")
    else:
        _check(wd_t, "wd_t", torch.bfloat16, (d, f))
    _check(tw.count, "count", torch.uint8, (n, f // tw.tile))
    _check(tw.idx, "idx", torch.uint8, (n, f // tw.tile, tw.cap))
    _check(tw.val, "val", x.dtype, (n, f // tw.tile, tw.cap))
    if y is None:
        y = torch.empty_like(x)
    _check(y, "y", x.dtype, (n, d))
    if workspace is None:
        workspace = routed_workspace(n, d, f, s_max, x.device)
    _check(workspace, "workspace", torch.uint8)
    if diag is not None:
        _check(diag, "diag", torch.int32, (4,))
    _call("twell_hybrid_up_down", _ptr(x), _ptr(tw.count), _ptr(tw.idx), _ptr(tw.val), _ptr(wu_t),
          _ptr(wd), ldw, _ptr(wd_t), _ptr(y), n, d, f, tw.tile, tw.cap, ell_cap, s_max,
          _ptr(workspace), workspace.numel(), _ptr(diag), _stream(x.device, stream))
    return y


def twell_ffn_forward(x, wg_t, wu_t, wd, tile: int, cap: int, tw: Optional[TwELL] = None,
                      y: Optional[torch.Tensor] = None, diag: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None, stream=None):
    """The sparse inference forward: gate GEMM + TwELL epilogue, then the
    fused up/down kernel.  Returns (y, twell)."""
    tw = twell_gate_pack(x, wg_t, tile, cap, out=tw, diag=diag, stream=stream)
    y = twell_fused_up_down(x, tw, wu_t, wd, y=y, workspace=workspace, diag=diag, stream=stream)
    return y, tw


def dense_ffn_fwd(x: torch.Tensor, wg_t: torch.Tensor, wu_t: torch.Tensor, wd_t: torch.Tensor,
                  h: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                  diag: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Dense bf16 gated FFN (baseline).  ``wd_t`` is W_down transposed, [d][F]."""
    _check(x, "x", torch.bfloat16)
    n, d = x.shape
    f = wg_t.shape[0]
    _check(wg_t, "wg_t", torch.bfloat16, (f, d))
    _check(wu_t, "wu_t", torch.bfloat16, (f, d))
    _check(wd_t, "wd_t", torch.bfloat16, (d, f))
    if h is None:
        h = torch.empty((n, f), dtype=torch.bfloat16, device=x.device)
    if y is None:
        y = torch.empty_like(x)
    _check(h, "h", torch.bfloat16, (n, f))
    _check(y, "y", torch.bfloat16, (n, d))
    _call("dense_ffn_fwd", _ptr(x), _ptr(wg_t), _ptr(wu_t), _ptr(wd_t), _ptr(h), _ptr(y),
          n, d, f, _ptr(diag), _stream(x.device, stream))
    return y


@dataclass
class Hybrid:
    """Device buffers of the hybrid format (see `sge_hybrid` in include/sge.h)."""
    n_tokens: int
    d_ff: int
    ell_cap: int
    s_max: int
    row_nnz: torch.Tensor
    spill_slot: torch.Tensor
    spill_rows: torch.Tensor
    n_spill: torch.Tensor
    ell_idx: torch.Tensor
    ell_a: torch.Tensor
    ell_u: torch.Tensor
    spill_a: torch.Tensor
    spill_u: torch.Tensor

    @staticmethod
    def empty(n: int, f: int, ell_cap: int, s_max: int, device) -> "Hybrid":
        kk, ss = max(ell_cap, 1), max(s_max, 1)
        z = lambda *shape, dt: torch.empty(shape, dtype=dt, device=device)
        return Hybrid(n, f, ell_cap, s_max, z(n, dt=torch.int32), z(n, dt=torch.int32),
                      z(ss, dt=torch.int32), z(1, dt=torch.int32), z(n, kk, dt=torch.uint16),
                      z(n, kk, dt=torch.bfloat16), z(n, kk, dt=torch.bfloat16),
                      z(ss, f, dt=torch.bfloat16), z(ss, f, dt=torch.bfloat16))

    def c_struct(self) -> _SgeHybrid:
        for name in ("row_nnz", "spill_slot", "spill_rows", "n_spill", "ell_idx", "ell_a", "ell_u",
                     "spill_a", "spill_u"):
            _check(getattr(self, name), name)
        return _SgeHybrid(self.n_tokens, self.d_ff, self.ell_cap, self.s_max, SGE_BF16, 0,
                          self.row_nnz.data_ptr(), self.spill_slot.data_ptr(),
                          self.spill_rows.data_ptr(), self.n_spill.data_ptr(),
                          self.ell_idx.data_ptr(), self.ell_a.data_ptr(), self.ell_u.data_ptr(),
                          self.spill_a.data_ptr(), self.spill_u.data_ptr())


def hybrid_pack(tw: TwELL, ell_cap: int, s_max: int, out: Optional[Hybrid] = None,
                diag: Optional[torch.Tensor] = None, stream=None) -> Hybrid:
    """Route each row of a bf16 TwELL to the ELL part (nnz <= K) or the dense spill."""
    _check(tw.count, "count", torch.uint8)
    _check(tw.val, "val", torch.bfloat16)
    n, f = tw.n_rows, tw.n_cols
    if out is None:
        out = Hybrid.empty(n, f, ell_cap, s_max, tw.count.device)
    cs = out.c_struct()
    _call("hybrid_pack", _ptr(tw.count), _ptr(tw.idx), _ptr(tw.val), tw.tile, tw.cap,
          ctypes.byref(cs), _ptr(diag), _stream(tw.count.device, stream))
    return out


def hybrid_fwd_workspace(d_model: int, d_ff: int, s_max: int, device) -> torch.Tensor:
    nbytes = library().hybrid_ffn_fwd_workspace_bytes(d_model, d_ff, s_max)
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)


def hybrid_ffn_fwd(x: torch.Tensor, hy: Hybrid, wu_t: torch.Tensor, wd: torch.Tensor,
                   wd_t: Optional[torch.Tensor], y: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None, stream=None,
                   wg_t: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y from the hybrid form; fills hy.ell_u and hy.spill_u.  ``wd_t`` is
    W_down transposed, [d][F] (a weight layout the caller builds once; None
    only when hy.s_max == 0).  With wg_t the spill rows' activations are
    recomputed from the gate (and written to hy.spill_a), so rows that
    reached the spill through an overflowing TwELL tile come out exact."""
    _check(x, "x", torch.bfloat16)
    n, d = x.shape
    f = hy.d_ff
    _check(wu_t, "wu_t", torch.bfloat16, (f, d))
    _check(wd, "wd", torch.bfloat16, (f, d))
    if wd_t is None:
        if hy.s_max > 0:
            raise ValueError("wd_t (W_down transposed, [d][F]) is required when s_max > 0")
    else:
        _check(wd_t, "wd_t", torch.bfloat16, (d, f))
    if wg_t is not None:
        _check(wg_t, "wg_t", torch.bfloat16, (f, d))
    if y is None:
        y = torch.empty_like(x)
    if workspace is None:
        workspace = hybrid_fwd_workspace(d, f, hy.s_max, x.device)
    cs = hy.c_struct()
    _call("hybrid_ffn_fwd", _ptr(x), ctypes.byref(cs), _ptr(wu_t), _ptr(wd), _ptr(wd_t),
          _ptr(wg_t) if wg_t is not None else None, _ptr(y), d,
          _ptr(workspace), workspace.numel(), _stream(x.device, stream))
    return y


def hybrid_bwd_workspace(n_tokens: int, d_model: int, d_ff: int, ell_cap: int, s_max: int,
                         device) -> torch.Tensor:
    nbytes = library().hybrid_ffn_bwd_workspace_bytes(n_tokens, d_model, d_ff, ell_cap, s_max)
    # 256-byte alignment: the caching allocator hands out 512-byte aligned blocks
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def transpose_up_gate(wu_t: torch.Tensor, wg_t: torch.Tensor, stream=None) -> torch.Tensor:
    """w_ug [d][2F] = [W_up | W_gate], hybrid_ffn_bwd's dX operand; a
    weight-loading step, done once per weight update."""
    _check(wu_t, "wu_t", torch.bfloat16)
    f, d = wu_t.shape
    _check(wg_t, "wg_t", torch.bfloat16, (f, d))
    w_ug = torch.empty((d, 2 * f), dtype=torch.bfloat16, device=wu_t.device)
    _call("sge_transpose_up_gate", _ptr(wu_t), _ptr(wg_t), _ptr(w_ug), f, d, _stream(wu_t.device, stream))
    return w_ug


def hybrid_ffn_bwd(x: torch.Tensor, dy: torch.Tensor, hy: Hybrid, wg_t: torch.Tensor,
                   wu_t: torch.Tensor, wd: torch.Tensor, workspace: Optional[torch.Tensor] = None,
                   stream=None, w_ug: Optional[torch.Tensor] = None, out=None):
    """Returns (dx bf16 [N][d], dwg_t, dwu_t, dwd fp32 [F][d]).  ``w_ug`` is
    transpose_up_gate's [W_up | W_gate] (None: built in the workspace per
    call); ``out`` optionally gives the four output tensors."""
    _check(x, "x", torch.bfloat16)
    n, d = x.shape
    f = hy.d_ff
    _check(dy, "dy", torch.bfloat16, (n, d))
    for name, w in (("wg_t", wg_t), ("wu_t", wu_t), ("wd", wd)):
        _check(w, name, torch.bfloat16, (f, d))
    if w_ug is not None:
        _check(w_ug, "w_ug", torch.bfloat16, (d, 2 * f))
    if out is None:
        out = (torch.empty_like(x),) + tuple(torch.empty((f, d), dtype=torch.float32, device=x.device)
                                              for _ in range(3))
    dx, dwg, dwu, dwd = out
    if workspace is None:
        workspace = hybrid_bwd_workspace(n, d, f, hy.ell_cap, hy.s_max, x.device)
    cs = hy.c_struct()
    _call("hybrid_ffn_bwd", _ptr(x), _ptr(dy), ctypes.byref(cs), _ptr(wg_t), _ptr(wu_t), _ptr(wd),
          _ptr(w_ug), _ptr(dx), _ptr(dwg), _ptr(dwu), _ptr(dwd), d, _ptr(workspace),
          workspace.numel(), _stream(x.device, stream))
    return dx, dwg, dwu, dwd
