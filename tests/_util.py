"""Test-side helpers: host copies of device outputs and comparisons.

Device results are only ever compared here; they are never fed to the oracle.
"""
import numpy as np
import torch

import oracle

BF16_TOL = 2e-2      # max-abs-rel bar for bf16 outputs
F32_TOL = 1e-5       # max-abs-rel bar for fp32 outputs
FLIP_EPS = 1e-3      # a gate may change sign between GPU and oracle only if |g| < this


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def unpack_np(count, idx, val, tile, cap) -> np.ndarray:
    """Dense [N][F] matrix of the stored TwELL entries (numpy, test side)."""
    count = np.asarray(count)
    idx = np.asarray(idx).astype(np.int64)
    val = np.asarray(val, np.float64)
    n, nt = count.shape
    h = np.zeros((n, nt * tile))
    keep = np.arange(cap)[None, None, :] < np.minimum(count, cap)[:, :, None]
    t_i, b_i, s_i = np.nonzero(keep)
    h[t_i, b_i * tile + idx[t_i, b_i, s_i]] = val[t_i, b_i, s_i]
    return h


def twell_host(tw):
    """(count, idx, val as float64) of a device TwELL."""
    return (tw.count.cpu().numpy(), tw.idx.cpu().numpy(), to_f64(tw.val))


def assert_twell_equal(tw_gpu, tw_ora: "oracle.TwELL"):
    """Bit-exact comparison of counts, and of the stored slots' indices and values."""
    c, i, v = twell_host(tw_gpu)
    np.testing.assert_array_equal(c, tw_ora.count)
    keep = np.arange(tw_ora.cap)[None, None, :] < np.minimum(tw_ora.count, tw_ora.cap)[:, :, None]
    np.testing.assert_array_equal(i[keep], tw_ora.idx[keep])
    np.testing.assert_array_equal(v[keep], tw_ora.val[keep])


def compare_twell_inexact(tw_gpu, tw_ora: "oracle.TwELL", g_ora: np.ndarray, val_kind: int,
                          abs_sum: np.ndarray, rows=None):
    """GPU TwELL (fp32 gate accumulation) vs the oracle's (fp64 gates).

    A tile may disagree (different count, or different stored indices, which
    a sign flip causes in a truncated tile by shifting its window) only if it
    holds oracle gates with |g| < FLIP_EPS, at least as many as the count
    difference.  Values of agreeing tiles match within one ulp of the value
    dtype plus the fp32 accumulation allowance 2^-16 * sum_i |x_i w_i|
    (``abs_sum``, [N][F]).  Returns (bad-row mask, number of disagreeing
    tiles)."""
    c, i, v = twell_host(tw_gpu)
    if rows is not None:
        c, i, v = c[rows], i[rows], v[rows]
    cap, tile = tw_ora.cap, tw_ora.tile
    n, nt = c.shape
    slots = np.arange(cap)[None, None, :]
    keep_g = slots < np.minimum(c, cap)[:, :, None]
    keep_o = slots < np.minimum(tw_ora.count, cap)[:, :, None]
    idx_g = np.where(keep_g, i.astype(np.int32), -1)
    idx_o = np.where(keep_o, tw_ora.idx.astype(np.int32), -1)
    tile_bad = (c != tw_ora.count) | np.any(idx_g != idx_o, axis=2)
    near = (np.abs(g_ora) < FLIP_EPS).reshape(n, nt, tile).sum(-1)
    dcount = np.abs(c.astype(np.int64) - tw_ora.count.astype(np.int64))
    assert np.all(near[tile_bad] >= np.maximum(1, dcount[tile_bad])), \
        "a tile disagrees without a near-zero gate to explain it"
    ok = (~tile_bad)[:, :, None] & keep_o
    vg, vo = v[ok], tw_ora.val[ok]
    t_i, b_i, s_i = np.nonzero(ok)
    s_abs = abs_sum[t_i, b_i * tile + tw_ora.idx[t_i, b_i, s_i].astype(np.int64)]
    ulp = 2.0 ** -7 if val_kind == oracle.VAL_BF16 else 2.0 ** -23
    excess = np.abs(vg - vo) - ulp * np.abs(vo) * 1.0001
    assert np.all(excess <= 2.0 ** -16 * s_abs), float(np.max(excess / s_abs))
    return tile_bad.any(1), int(tile_bad.sum())
