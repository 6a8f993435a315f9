"""Test-side helpers: host copies of device outputs and comparisons.

Device results are only ever compared here; they are never fed to the oracle.
"""
import numpy as np
import torch

import oracle
from activation_sparse_gated_epilogue_b200 import synth

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


def gamma_fp32(n_terms: int) -> float:
    """Worst-case relative bound of an fp32 inner product of n_terms terms,
    gamma_n = n u / (1 - n u) with u = 2^-24 (the standard backward-error
    bound of recursive or any other order of pairwise summation:
    |fl(sum p_i) - sum p_i| <= gamma_n sum |p_i|).  The gate GEMM's products
    of bf16 operands are exact in fp32, so the gate carries gamma_d; fp32
    operands add one rounding per product, gamma_(d+1) covers both."""
    nu = n_terms * 2.0 ** -24
    return nu / (1.0 - nu)


def compare_twell_inexact(tw_gpu, tw_ora: "oracle.TwELL", g_ora: np.ndarray, val_kind: int,
                          abs_sum: np.ndarray, rows=None, d_model: int = None):
    """GPU TwELL (fp32 gate accumulation) vs the oracle's (fp64 gates).

    A tile may disagree (different count, or different stored indices, which
    a sign flip causes in a truncated tile by shifting its window) only if it
    holds oracle gates with |g| < FLIP_EPS, at least as many as the count
    difference.  Stored values of agreeing tiles satisfy the bound of two
    roundings of nearby numbers: |v_gpu - v_ora| <= u_v (|v_gpu| + |v_ora|) +
    (1 + u_v) gamma_(d+1) sum_i |x_i w_i|, u_v the value dtype's unit
    roundoff (2^-8 bf16, 2^-24 fp32) and ``abs_sum`` [N][F] the sums of
    |x_i w_i|.  Returns (rows with a disagreeing tile, rows whose disagreeing
    tile is truncated (count > C on either side, so its stored window may
    shift), number of disagreeing tiles, largest observed fraction of the
    accumulation allowance)."""
    c, i, v = twell_host(tw_gpu)
    if rows is not None:
        c, i, v = c[rows], i[rows], v[rows]
    cap, tile = tw_ora.cap, tw_ora.tile
    n, nt = c.shape
    d = d_model if d_model is not None else 2 ** 14
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
    trunc_bad = tile_bad & ((c > cap) | (tw_ora.count > cap))
    ok = (~tile_bad)[:, :, None] & keep_o
    vg, vo = v[ok], tw_ora.val[ok]
    t_i, b_i, s_i = np.nonzero(ok)
    s_abs = abs_sum[t_i, b_i * tile + tw_ora.idx[t_i, b_i, s_i].astype(np.int64)]
    u_v = 2.0 ** -8 if val_kind == oracle.VAL_BF16 else 2.0 ** -24
    allow = (1.0 + u_v) * gamma_fp32(d + 1) * s_abs
    excess = np.abs(vg - vo) - u_v * (np.abs(vg) + np.abs(vo))
    assert np.all(excess <= allow), float(np.max(excess / allow))
    frac = float(np.max(np.maximum(excess, 0.0) / allow)) if allow.size else 0.0
    return tile_bad.any(1), trunc_bad.any(1), int(tile_bad.sum()), frac


_ORACLE_1B = {}


def oracle_1b():
    """Inputs and the oracle's whole forward of the 1B workload (all rows),
    computed once per test session: (inp, y, TwELL, G, sum |x w|)."""
    if not _ORACLE_1B:
        cfg = synth.CONFIGS["ffn_1b_bf16"]
        inp = synth.make_inputs(cfg)
        xf, wgf, wuf, wdf = (inp.as_f64(k) for k in ("x", "wg_t", "wu_t", "wd"))
        y_ora, tw_ora, g = oracle.sparse_ffn(xf, wgf, wuf, wdf, cfg.tile, cfg.cap, oracle.VAL_BF16)
        _ORACLE_1B.update(inp=inp, y=y_ora, tw=tw_ora, g=g, abs_sum=np.abs(xf) @ np.abs(wgf).T)
    o = _ORACLE_1B
    return o["inp"], o["y"], o["tw"], o["g"], o["abs_sum"]


def check_1b_all_rows(y_gpu: np.ndarray, tw_gpu=None):
    """y of the 1B workload against the oracle on all rows (and the GPU's
    TwELL against the oracle's, when given)."""
    inp, y_ora, tw_ora, g, abs_sum = oracle_1b()
    flips = 0
    if tw_gpu is not None:
        _, shifted, flips, _ = compare_twell_inexact(tw_gpu, tw_ora, g, oracle.VAL_BF16, abs_sum,
                                                     d_model=inp.x.shape[1])
        assert not shifted.any()
    err = oracle.max_abs_rel(y_gpu, y_ora)
    assert err <= BF16_TOL, err
    return err, flips


def heavy_and_strided_rows(inp, n_heavy=128, stride=4):
    """The n_heavy tokens with the largest per-token scale (the most active
    gates) and every stride-th token."""
    n = inp.x.shape[0]
    heavy = np.argsort(-inp.scale)[:n_heavy]
    return np.unique(np.concatenate([heavy, np.arange(0, n, stride), [n - 1]]))


_SWEEP_CACHE = {}


def sweep_gate0(inp, rows):
    """Oracle gate pre-activations of the checked rows with the bias column
    of W_gate set to zero, shared by the sweep's densities: the inputs differ
    only in that column (x's last feature is 1.0), and the oracle sums the
    bias term last, so G(tau) = fl(G0 - tau) bit for bit (pinned on the CPU
    by tests/test_oracle_pins.py)."""
    key = tuple(rows[:4]) + (len(rows),)
    if key not in _SWEEP_CACHE:
        _SWEEP_CACHE.clear()
        xf = inp.as_f64("x")[rows]
        wg0 = inp.as_f64("wg_t").copy()
        wg0[:, -1] = 0.0
        _SWEEP_CACHE[key] = (oracle.gate_preact(xf, wg0), np.abs(xf) @ np.abs(wg0).T)
    return _SWEEP_CACHE[key]
