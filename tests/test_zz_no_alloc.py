"""The allocation-free fused up/down entry point.

Callers that cannot allocate device memory (runtimes that forbid cudaMalloc
while serving, servers whose memory is all in their own pools, plugins that
only see their input and output tensors) use twell_fused_up_down_noalloc,
whose scratch is a device array built into the library.  This file is
collected last so that a run stopping at the first failure has already run
every other test; it passes alone and after the others.
"""
import ctypes

import numpy as np
import pytest
import torch

import activation_sparse_gated_epilogue_b200 as sge
import oracle
from activation_sparse_gated_epilogue_b200 import synth
from tests._util import BF16_TOL

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    lib = sge.library()
    fn = lib.twell_fused_up_down_noalloc
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    fn.restype = I
    fn.argtypes = [P, P, P, P, P, P, I64, P, I64, I64, I64, I, I, I, P, P]
    lib.twell_fused_up_down_noalloc_max_tokens.restype = I64
    return lib, fn


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _upload_twell(tw: "oracle.TwELL", dev):
    return sge.TwELL(torch.from_numpy(tw.count).to(dev), torch.from_numpy(tw.idx).to(dev),
                     torch.from_numpy(tw.val).to(torch.bfloat16).to(dev), tw.tile, tw.cap)


def test_noalloc_matches_oracle_and_workspace_entry_point(cuda_device):
    """Both sides get the oracle's TwELL of the same inputs (a few heavy
    tokens, so heavy-token units and light tokens both run): two calls in a
    row of the allocation-free entry point match the oracle's fused up/down
    and the workspace entry point within the bf16 bar."""
    lib, fn = _noalloc_fn()
    cfg = synth.CONFIGS["ffn_0p5b_bf16"]
    inp = synth.make_inputs(cfg, n_tokens=2048)
    inp.x[:6, :-1] *= 8.0          # exact in bf16 (a power of two)
    xf, wgf, wuf, wdf = (inp.as_f64(k) for k in ("x", "wg_t", "wu_t", "wd"))
    tw_ora = oracle.twell_pack(oracle.gate_preact(xf, wgf), cfg.tile, cfg.cap, oracle.VAL_BF16)
    assert tw_ora.count[:6].sum() > 4 * tw_ora.count[6:].sum(1).max()   # the heavy tokens
    want = oracle.fused_up_down(xf, tw_ora, wuf, wdf)
    x, wu, wd = (getattr(inp, k).to(cuda_device) for k in ("x", "wu_t", "wd"))
    tw = _upload_twell(tw_ora, cuda_device)
    y_ws = sge.twell_fused_up_down(x, tw, wu, wd)
    n, d = x.shape
    f = wu.shape[0]
    stream = ctypes.c_void_p(torch.cuda.current_stream(cuda_device).cuda_stream)
    torch.cuda.synchronize()
    got_ws = y_ws.double().cpu().numpy()
    assert oracle.max_abs_rel(got_ws, want) <= BF16_TOL
    for call in range(2):           # the second call reuses the array's old contents
        y = torch.full_like(x, float("nan"))
        rc = fn(_ptr(x), _ptr(tw.count), _ptr(tw.idx), _ptr(tw.val), _ptr(wu), _ptr(wd), d, _ptr(y),
                n, d, f, sge.SGE_BF16, tw.tile, tw.cap, None, stream)
        assert rc == 0, lib.sge_last_error()
        torch.cuda.synchronize()
        got = y.double().cpu().numpy()
        assert np.isfinite(got).all()
        assert oracle.max_abs_rel(got, want) <= BF16_TOL, call
        assert oracle.max_abs_rel(got, got_ws) <= BF16_TOL, call


def test_noalloc_zero_tokens_sets_up_only(cuda_device):
    """A call without tokens performs only the start-up lookup of the
    array's address; its pointers may be NULL."""
    lib, fn = _noalloc_fn()
    torch.cuda.synchronize()
    rc = fn(None, None, None, None, None, None, 64, None, 0, 64, 256, sge.SGE_BF16, 128, 128, None, None)
    assert rc == 0, lib.sge_last_error()


def test_noalloc_rejects_more_tokens_than_its_scratch_holds(cuda_device):
    lib, fn = _noalloc_fn()
    limit = lib.twell_fused_up_down_noalloc_max_tokens()
    assert limit >= 8192
    p = ctypes.c_void_p(16)
    rc = fn(p, p, p, p, p, p, 64, p, limit + 1, 64, 256, sge.SGE_BF16, 128, 128, None, None)
    assert rc == 2
    assert b"scratch limit" in lib.sge_last_error()


def test_noalloc_small_batch_full_density(cuda_device):
    """The built-in pool holds 512 fp32 partial rows at d_model = 2048; a
    64-token batch with every gate active needs units of 512 entries for its
    partials to fit, and still equals the dense FFN."""
    lib, fn = _noalloc_fn()
    n, d, f = 64, 2048, 4096
    inp = synth.make_inputs(synth.CONFIGS["ffn_0p5b_bf16"].with_(n_tokens=n, d_model=d, d_ff=f),
                            tau=-1e3)
    x, wg, wu, wd = (getattr(inp, k).to(cuda_device) for k in ("x", "wg_t", "wu_t", "wd"))
    tw = sge.twell_gate_pack(x, wg, 128, 128)
    stream = ctypes.c_void_p(torch.cuda.current_stream(cuda_device).cuda_stream)
    y = torch.full_like(x, float("nan"))
    rc = fn(_ptr(x), _ptr(tw.count), _ptr(tw.idx), _ptr(tw.val), _ptr(wu), _ptr(wd), d, _ptr(y),
            n, d, f, sge.SGE_BF16, tw.tile, tw.cap, None, stream)
    assert rc == 0, lib.sge_last_error()
    torch.cuda.synchronize()
    assert int(tw.count.sum()) == n * f
    want = oracle.dense_ffn(*[inp.as_f64(k) for k in ("x", "wg_t", "wu_t", "wd")])
    assert oracle.max_abs_rel(y.double().cpu().numpy(), want) <= BF16_TOL
