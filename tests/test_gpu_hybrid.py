"""GPU parity of the hybrid training format (pack and forward) against the
fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import activation_sparse_gated_epilogue_b200 as sge
import oracle
from activation_sparse_gated_epilogue_b200 import synth
from tests._util import (BF16_TOL, check_1b_all_rows, compare_twell_inexact, oracle_1b,
                         to_f64)

pytestmark = pytest.mark.gpu


def _small_inputs(n=300, d=256, f=1024, seed=0):
    cfg = synth.CONFIGS["train_1b_hybrid"].with_(n_tokens=n, d_model=d, d_ff=f, spill_frac=None,
                                                 rho=0.02, seed=seed)
    return synth.make_inputs(cfg)


def _upload_twell(tw: oracle.TwELL, dev):
    return sge.TwELL(torch.from_numpy(tw.count).to(dev), torch.from_numpy(tw.idx).to(dev),
                     torch.from_numpy(tw.val).to(torch.bfloat16).to(dev), tw.tile, tw.cap)


def _check_pack(hy: sge.Hybrid, ora: oracle.Hybrid):
    np.testing.assert_array_equal(hy.row_nnz.cpu().numpy(), ora.row_nnz)
    np.testing.assert_array_equal(hy.spill_slot.cpu().numpy(), ora.spill_slot)
    assert int(hy.n_spill.item()) == ora.n_spill
    kept = min(ora.n_spill, ora.s_max)
    np.testing.assert_array_equal(hy.spill_rows.cpu().numpy()[:kept], ora.spill_rows[:kept])
    k = ora.k
    if k > 0:
        ell = ora.row_nnz <= k
        gidx = hy.ell_idx.cpu().numpy().astype(np.int64)[:, :k]
        gidx[gidx == 0xFFFF] = -1
        np.testing.assert_array_equal(gidx[ell], ora.ell_idx[ell])
        np.testing.assert_array_equal(to_f64(hy.ell_a)[:, :k][ell], ora.ell_a[ell])
    if kept:
        np.testing.assert_array_equal(to_f64(hy.spill_a)[:kept], ora.spill_a[:kept])


@pytest.mark.parametrize("k,s_max", [(16, 64), (16, 4), (0, 300), (512, 8), (40, 32)])
def test_hybrid_pack_and_fwd_match_oracle(cuda_device, k, s_max):
    inp = _small_inputs()
    x, wg, wu, wd = (inp.as_f64(n) for n in ("x", "wg_t", "wu_t", "wd"))
    x[:7, :-1] *= 3.0                                     # a few heavy rows
    xb = torch.from_numpy(x).to(torch.bfloat16)
    x = xb.double().numpy()
    tw = oracle.twell_pack(oracle.gate_preact(x, wg), 128, 128, oracle.VAL_BF16)
    ora = oracle.hybrid_pack(tw, k, s_max)
    y_ora = oracle.hybrid_fwd(x, ora, wu, wd)

    diag = sge.new_diag(cuda_device)
    hy = sge.hybrid_pack(_upload_twell(tw, cuda_device), k, s_max, diag=diag)
    torch.cuda.synchronize()
    _check_pack(hy, ora)
    assert int(diag[1]) == ora.n_spill
    assert int(diag[2]) == ora.dropped

    wd_d = inp.wd.to(cuda_device)
    y = sge.hybrid_ffn_fwd(xb.to(cuda_device), hy, inp.wu_t.to(cuda_device), wd_d, wd_d.t().contiguous())
    torch.cuda.synchronize()
    err = oracle.max_abs_rel(to_f64(y), y_ora)
    assert err <= BF16_TOL, err
    if k > 0:
        ell = ora.row_nnz <= k
        gu = to_f64(hy.ell_u)[:, :k][ell]
        mask = np.arange(k)[None, :] < ora.row_nnz[ell][:, None]
        assert oracle.max_abs_rel(gu[mask], ora.ell_u[ell][mask]) <= 1e-2
    kept = min(ora.n_spill, s_max)
    if kept:
        assert oracle.max_abs_rel(to_f64(hy.spill_u)[:kept], ora.spill_u[:kept]) <= 1e-2
    dropped = (ora.row_nnz > k) & (ora.spill_slot < 0)
    assert np.all(to_f64(y)[dropped] == 0.0)


@pytest.mark.parametrize("cap", [32, 16])
def test_hybrid_capacity_below_tile(cuda_device, cap):
    """TwELL with a capacity C below the tile width T: rows with a tile past
    C go to the spill (row_nnz = K + 1 when their stored count fits K), and
    the pack matches the oracle bit for bit.  Given W_gate, the forward
    recomputes the spill rows from the gate and equals the full-capacity
    (C = T) sparse FFN; without it the spill rows use the truncated
    activations, as the oracle's forward of the same pack does."""
    n, d, f, tile, k, s_max = 300, 256, 1024, 128, 64, 300
    inp = _small_inputs(n, d, f)
    x, wg, wu, wd = (inp.as_f64(nm) for nm in ("x", "wg_t", "wu_t", "wd"))
    x[:9, :-1] *= 5.0                                     # heavy rows: tiles past C, > K entries
    # rows 10..19 switch on 40 gates of tile 0 through feature 0: a tile past
    # C in a row whose stored entries still fit K
    x[:, 0] = 0.0
    x[10:20, 0] = 4.0
    wg = wg.copy()
    wg[:40, 0] = 2.0
    xb = torch.from_numpy(x).to(torch.bfloat16)
    x = xb.double().numpy()
    wgb = torch.from_numpy(wg).to(torch.bfloat16)
    wg = wgb.double().numpy()
    g = oracle.gate_preact(x, wg)
    tw_c = oracle.twell_pack(g, tile, cap, oracle.VAL_BF16)
    assert tw_c.overflow > 0
    ora = oracle.hybrid_pack(tw_c, k, s_max)
    assert np.any(ora.row_nnz == k + 1)                   # spilled only through the capacity
    dev = cuda_device
    wg_d = wgb.to(dev)
    wu_d, wd_d = (getattr(inp, nm).to(dev) for nm in ("wu_t", "wd"))

    hy = sge.hybrid_pack(_upload_twell(tw_c, dev), k, s_max)
    torch.cuda.synchronize()
    _check_pack(hy, ora)
    y = sge.hybrid_ffn_fwd(xb.to(dev), hy, wu_d, wd_d, wd_d.t().contiguous(), wg_t=wg_d)
    want = oracle.fused_up_down(x, oracle.twell_pack(g, tile, tile, oracle.VAL_BF16), wu, wd)
    torch.cuda.synchronize()
    err = oracle.max_abs_rel(to_f64(y), want)
    assert err <= BF16_TOL, err
    # the recomputed activations of the kept spill rows are the full ReLU(g)
    kept = min(ora.n_spill, s_max)
    full_a = oracle.round_array(np.maximum(g[ora.spill_rows[:kept]], 0.0), oracle.VAL_BF16)
    assert oracle.max_abs_rel(to_f64(hy.spill_a)[:kept], full_a) <= 1e-2

    hy2 = sge.hybrid_pack(_upload_twell(tw_c, dev), k, s_max)
    y2 = sge.hybrid_ffn_fwd(xb.to(dev), hy2, wu_d, wd_d, wd_d.t().contiguous())
    torch.cuda.synchronize()
    err2 = oracle.max_abs_rel(to_f64(y2), oracle.hybrid_fwd(x, ora, wu, wd))
    assert err2 <= BF16_TOL, err2


@pytest.mark.parametrize("k,s_max", [(16, 64), (16, 4), (0, 300), (512, 8), (40, 32)])
def test_hybrid_bwd_matches_oracle(cuda_device, k, s_max):
    inp = _small_inputs(seed=1)
    x, wg, wu, wd = (inp.as_f64(n) for n in ("x", "wg_t", "wu_t", "wd"))
    x[:7, :-1] *= 3.0
    xb = torch.from_numpy(x).to(torch.bfloat16)
    x = xb.double().numpy()
    dyb = torch.from_numpy(np.random.default_rng(5).standard_normal(x.shape)).to(torch.bfloat16)
    dy = dyb.double().numpy()
    tw = oracle.twell_pack(oracle.gate_preact(x, wg), 128, 128, oracle.VAL_BF16)
    ora = oracle.hybrid_pack(tw, k, s_max)
    oracle.hybrid_fwd(x, ora, wu, wd)
    want = oracle.hybrid_bwd(x, dy, ora, wg, wu, wd)

    dev = cuda_device
    hy = sge.hybrid_pack(_upload_twell(tw, dev), k, s_max)
    w_dev = [getattr(inp, n).to(dev) for n in ("wg_t", "wu_t", "wd")]
    sge.hybrid_ffn_fwd(xb.to(dev), hy, w_dev[1], w_dev[2], w_dev[2].t().contiguous())
    got = sge.hybrid_ffn_bwd(xb.to(dev), dyb.to(dev), hy, *w_dev)
    torch.cuda.synchronize()
    for name, a, b in zip(("dx", "dW_gate", "dW_up", "dW_down"), got, want):
        err = oracle.max_abs_rel(to_f64(a), b)
        assert err <= BF16_TOL, (name, err)
    dropped = (ora.row_nnz > k) & (ora.spill_slot < 0)
    assert np.all(to_f64(got[0])[dropped] == 0.0)


def test_hybrid_bwd_is_deterministic(cuda_device):
    inp = _small_inputs(seed=2)
    dev = cuda_device
    x, wg, wu, wd = (getattr(inp, n).to(dev) for n in ("x", "wg_t", "wu_t", "wd"))
    dy = torch.randn(x.shape, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16).to(dev)
    tw = sge.twell_gate_pack(x, wg, 128, 128)
    hy = sge.hybrid_pack(tw, 16, 64)
    sge.hybrid_ffn_fwd(x, hy, wu, wd, wd.t().contiguous())
    a = sge.hybrid_ffn_bwd(x, dy, hy, wg, wu, wd)
    b = sge.hybrid_ffn_bwd(x, dy, hy, wg, wu, wd)
    torch.cuda.synchronize()
    for u, v in zip(a, b):
        assert torch.equal(u, v)


@pytest.mark.parametrize("tau", [1e3, -1e3])
def test_hybrid_bwd_zero_and_full_density(cuda_device, tau):
    """No active gate (tau = 1e3): every row is an empty ELL row, and y, dx
    and all three weight gradients are exactly zero.  Every gate active
    (tau = -1e3): every row holds F entries, so with K = 16 and S_max = N all
    rows take the dense spill GEMMs and each hidden unit's gradient bucket
    holds all N tokens (more than one round of staged entries); the results
    match the oracle."""
    n, d, f, k = 300, 256, 1024, 16
    cfg = synth.CONFIGS["train_1b_hybrid"].with_(n_tokens=n, d_model=d, d_ff=f, spill_frac=None,
                                                 rho=0.02, seed=4)
    inp = synth.make_inputs(cfg, tau=tau)
    x, wg, wu, wd, dy = (inp.as_f64(nm) for nm in ("x", "wg_t", "wu_t", "wd", "dy"))
    tw = oracle.twell_pack(oracle.gate_preact(x, wg), 128, 128, oracle.VAL_BF16)
    assert int(tw.count.astype(np.int64).sum()) == (0 if tau > 0 else n * f)
    ora = oracle.hybrid_pack(tw, k, n)
    y_ora = oracle.hybrid_fwd(x, ora, wu, wd)
    want = oracle.hybrid_bwd(x, dy, ora, wg, wu, wd)

    dev = cuda_device
    xd, dyd = inp.x.to(dev), inp.dy.to(dev)
    w_dev = [getattr(inp, nm).to(dev) for nm in ("wg_t", "wu_t", "wd")]
    hy = sge.hybrid_pack(_upload_twell(tw, dev), k, n)
    y = sge.hybrid_ffn_fwd(xd, hy, w_dev[1], w_dev[2], w_dev[2].t().contiguous())
    got = sge.hybrid_ffn_bwd(xd, dyd, hy, *w_dev)
    torch.cuda.synchronize()
    assert int(hy.n_spill.item()) == (0 if tau > 0 else n)
    if tau > 0:
        for t in (y,) + tuple(got):
            assert not torch.any(t != 0)
        return
    assert oracle.max_abs_rel(to_f64(y), y_ora) <= BF16_TOL
    for name, a, b in zip(("dx", "dW_gate", "dW_up", "dW_down"), got, want):
        err = oracle.max_abs_rel(to_f64(a), b)
        assert err <= BF16_TOL, (name, err)


def test_hybrid_inference_1b_all_rows(cuda_device):
    """The hybrid path as the bench runs it for inference on the 1B workload
    (K = 64, S_max = N/4: about 1,400 heavy rows on the tensor-core spill),
    every row of y against the oracle's forward."""
    inp = oracle_1b()[0]
    cfg = inp.cfg
    dev = cuda_device
    x, wg, wu, wd = (getattr(inp, n).to(dev) for n in ("x", "wg_t", "wu_t", "wd"))
    tw = sge.twell_gate_pack(x, wg, cfg.tile, cfg.cap)
    diag = sge.new_diag(dev)
    s_max = cfg.n_tokens // 4
    hy = sge.hybrid_pack(tw, 64, s_max, diag=diag)
    y = sge.hybrid_ffn_fwd(x, hy, wu, wd, wd.t().contiguous())
    torch.cuda.synchronize()
    n_spill = int(hy.n_spill.item())
    assert 1000 < n_spill <= s_max and int(diag[2]) == 0
    err, flips = check_1b_all_rows(to_f64(y), tw)
    print(f"hybrid inference 1B: {n_spill} spill rows, max-abs-rel {err:.2e} on all rows, "
          f"{flips} flips")


_TRAIN_ORACLE = {}


def _train_oracle(inp):
    """The oracle's hybrid forward and backward of the whole training-shaped
    workload (N=8192, d=2048, F=8192, K=128, S_max=1024), computed once."""
    if not _TRAIN_ORACLE:
        cfg = inp.cfg
        xf, wgf, wuf, wdf, dyf = (inp.as_f64(n) for n in ("x", "wg_t", "wu_t", "wd", "dy"))
        g = oracle.gate_preact(xf, wgf)
        tw = oracle.twell_pack(g, cfg.tile, cfg.cap, oracle.VAL_BF16)
        hy = oracle.hybrid_pack(tw, cfg.ell_cap, cfg.s_max)
        y = oracle.hybrid_fwd(xf, hy, wuf, wdf)
        grads = oracle.hybrid_bwd(xf, dyf, hy, wgf, wuf, wdf)
        _TRAIN_ORACLE.update(g=g, tw=tw, hy=hy, y=y, grads=grads,
                             abs_sum=np.abs(xf) @ np.abs(wgf).T)
    return _TRAIN_ORACLE


def test_hybrid_train_workload_full_gradients(cuda_device):
    """The full training-shaped step on the GPU (gate GEMM + TwELL, hybrid
    pack, forward, backward) against the oracle: y and dx on every row, and
    dW_gate, dW_up and dW_down on every hidden unit.  A near-zero sign flip
    between the GPU's fp32 gate and the oracle's fp64 gate changes the
    gradients of its row and of its hidden unit by a full term (dg = dh u
    does not scale with a), so such rows and units are left out and
    counted; there may be at most two of each."""
    cfg = synth.CONFIGS["train_1b_hybrid"]
    inp = synth.make_inputs(cfg)
    dev = cuda_device
    x, wg, wu, wd, dy = (getattr(inp, n).to(dev) for n in ("x", "wg_t", "wu_t", "wd", "dy"))
    tw = sge.twell_gate_pack(x, wg, cfg.tile, cfg.cap)
    diag = sge.new_diag(dev)
    hy = sge.hybrid_pack(tw, cfg.ell_cap, cfg.s_max, diag=diag)
    y = sge.hybrid_ffn_fwd(x, hy, wu, wd, wd.t().contiguous())
    got = sge.hybrid_ffn_bwd(x, dy, hy, wg, wu, wd)
    # the dX operand built once (a weight-loading step) gives the same bits
    got2 = sge.hybrid_ffn_bwd(x, dy, hy, wg, wu, wd, w_ug=sge.transpose_up_gate(wu, wg))
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(got, got2))
    n_spill = int(hy.n_spill.item())
    assert 0 < n_spill <= cfg.s_max and int(diag[2]) == 0, n_spill
    o = _train_oracle(inp)
    _, shifted, flips, _ = compare_twell_inexact(tw, o["tw"], o["g"], oracle.VAL_BF16, o["abs_sum"],
                                                 d_model=cfg.d_model)
    assert not shifted.any()
    # rows and hidden units touched by a disagreeing TwELL entry
    gpu_dense = _dense_active(tw)
    ora_dense = o["g"] > 0
    diff = gpu_dense != ora_dense
    bad_t, bad_j = diff.any(1), diff.any(0)
    assert bad_t.sum() <= 2 and bad_j.sum() <= 2, (bad_t.sum(), bad_j.sum())
    assert oracle.max_abs_rel(to_f64(y)[~bad_t], o["y"][~bad_t]) <= BF16_TOL
    errs = {}
    for name, a, b, keep in zip(("dx", "dW_gate", "dW_up", "dW_down"), got, o["grads"],
                                (~bad_t, ~bad_j, ~bad_j, ~bad_j)):
        errs[name] = oracle.max_abs_rel(to_f64(a)[keep], b[keep])
        assert errs[name] <= BF16_TOL, (name, errs[name])
    print(f"train hybrid full: {n_spill} spill rows, {flips} flipped tiles, "
          + ", ".join(f"{k} {v:.2e}" for k, v in errs.items()))


def _dense_active(tw) -> np.ndarray:
    """[N][F] mask of the columns a device TwELL stores (C = T)."""
    count = tw.count.cpu().numpy()
    idx = tw.idx.cpu().numpy().astype(np.int64)
    n, nt = count.shape
    act = np.zeros((n, nt * tw.tile), bool)
    keep = np.arange(tw.cap)[None, None, :] < np.minimum(count, tw.cap)[:, :, None]
    t_i, b_i, s_i = np.nonzero(keep)
    act[t_i, b_i * tw.tile + idx[t_i, b_i, s_i]] = True
    return act
