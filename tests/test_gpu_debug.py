"""The index-checking debug build (libsge_debug.so, compiled with SGE_DEBUG)
on the GPU: on valid inputs it gives the release build's bits and raises no
flag; given a TwELL whose stored columns lie outside their tiles it raises
SGE_FLAG_BOUNDS, keeps every access inside its buffers (a stored column is
clamped into its tile) and finishes with finite outputs."""
import contextlib
import os

import numpy as np
import pytest
import torch

import activation_sparse_gated_epilogue_b200 as sge
import oracle
from activation_sparse_gated_epilogue_b200 import binding, synth
from activation_sparse_gated_epilogue_b200 import build as sge_build

pytestmark = pytest.mark.gpu
SGE_FLAG_BOUNDS = 2


@contextlib.contextmanager
def library_at(path):
    """Route the binding's calls to the library at `path` for the block."""
    saved = (binding._lib, binding._LIB_PATH)
    binding._lib, binding._LIB_PATH = None, path
    try:
        yield binding.library()
    finally:
        binding._lib, binding._LIB_PATH = saved


def _case(dev, n=300, d=256, f=1024, seed=3):
    cfg = synth.CONFIGS["ffn_0p5b_bf16"].with_(n_tokens=n, d_model=d, d_ff=f, rho=0.02, seed=seed)
    inp = synth.make_inputs(cfg)
    inp.x[:7, :-1] *= 3.0  # heavy tokens for the spill path
    tw = oracle.twell_pack(oracle.gate_preact(inp.as_f64("x"), inp.as_f64("wg_t")), 128, 128,
                           oracle.VAL_BF16)
    x, wu, wd = (getattr(inp, k).to(dev) for k in ("x", "wu_t", "wd"))
    return tw, x, wu, wd


def _upload(tw, dev):
    return sge.TwELL(torch.from_numpy(tw.count).to(dev), torch.from_numpy(tw.idx).to(dev),
                     torch.from_numpy(tw.val).to(torch.bfloat16).to(dev), tw.tile, tw.cap)


def _forwards(tw_dev, x, wu, wd):
    """The routed call (spill GEMMs and light tokens), the per-entry call,
    the small-batch path and the hybrid pack + forward on the same TwELL."""
    wd_t = wd.t().contiguous()
    y_routed = sge.twell_hybrid_up_down(x, tw_dev, wu, wd, wd_t, 16, 64)
    y_fused = sge.twell_fused_up_down(x, tw_dev, wu, wd)
    small = sge.TwELL(tw_dev.count[:40], tw_dev.idx[:40], tw_dev.val[:40], tw_dev.tile, tw_dev.cap)
    y_small = sge.twell_fused_up_down(x[:40], small, wu, wd)
    hy = sge.hybrid_pack(tw_dev, 32, 64)
    y_hyb = sge.hybrid_ffn_fwd(x, hy, wu, wd, wd_t=wd_t)
    torch.cuda.synchronize()
    return [y_routed, y_fused, y_small, y_hyb]


def test_debug_build_matches_release_and_raises_nothing(cuda_device):
    tw, x, wu, wd = _case(cuda_device)
    tw_dev = _upload(tw, cuda_device)
    rel = _forwards(tw_dev, x, wu, wd)
    with library_at(sge_build.build_debug()):
        sge.debug_flags(clear=True)
        dbg = _forwards(tw_dev, x, wu, wd)
        assert sge.debug_flags(clear=True) == 0
    for a, b in zip(rel, dbg):
        assert torch.equal(a, b)


def test_debug_build_flags_columns_outside_their_tile(cuda_device):
    tw, x, wu, wd = _case(cuda_device, seed=4)
    bad_idx = tw.idx.copy()
    stored = np.arange(tw.cap)[None, None, :] < np.minimum(tw.count, tw.cap)[:, :, None]
    rows = np.nonzero(stored.any(axis=(1, 2)))[0]
    # the first stored entry of the first tile with one, in every 5th non-empty token
    for t in rows[::5]:
        b = int(np.nonzero(stored[t].any(axis=1))[0][0])
        bad_idx[t, b, 0] = 200  # outside the 128-column tile
    bad = oracle.TwELL(tw.count, bad_idx, tw.val, tw.tile, tw.cap, tw.overflow)
    tw_dev = _upload(bad, cuda_device)
    with library_at(sge_build.build_debug()):
        sge.debug_flags(clear=True)
        dbg = _forwards(tw_dev, x, wu, wd)
        flags = sge.debug_flags(clear=True)
    assert flags & SGE_FLAG_BOUNDS, flags
    for y in dbg:
        assert torch.isfinite(y.float()).all()
