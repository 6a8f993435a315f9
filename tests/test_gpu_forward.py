"""GPU parity of the inference path (gate GEMM + TwELL epilogue, fused
up/down, dense baseline) against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import activation_sparse_gated_epilogue_b200 as sge
import oracle
from activation_sparse_gated_epilogue_b200 import synth
from tests._util import (BF16_TOL, F32_TOL, FLIP_EPS, assert_twell_equal, check_1b_all_rows,
                         compare_twell_inexact, heavy_and_strided_rows, oracle_1b,
                         sweep_gate0, to_f64)

pytestmark = pytest.mark.gpu

KIND = {torch.bfloat16: oracle.VAL_BF16, torch.float32: oracle.VAL_F32}


def _dev(inp, dev):
    return [getattr(inp, k).to(dev) for k in ("x", "wg_t", "wu_t", "wd")]


def _f64(inp):
    return [inp.as_f64(k) for k in ("x", "wg_t", "wu_t", "wd")]


def _upload_twell(tw: oracle.TwELL, dtype, dev):
    return sge.TwELL(torch.from_numpy(tw.count).to(dev), torch.from_numpy(tw.idx).to(dev),
                     torch.from_numpy(tw.val).to(dtype).to(dev), tw.tile, tw.cap)


# ------------------------------------------------- gate GEMM + TwELL epilogue

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("n,d,f,tile,cap", [
    (300, 200, 640, 128, 128),    # ragged M, K tail, ragged N block
    (257, 136, 512, 64, 64),
    (128, 64, 256, 32, 5),        # overflow
    (520, 264, 768, 16, 16),
    (64, 512, 1024, 128, 12),
    (1, 136, 512, 128, 128),      # one token (batches of <= 256 rows: single-CTA tiles)
    (200, 264, 384, 64, 64),      # ragged rows inside one 128-row tile
    (128, 200, 640, 128, 128),    # one full row tile
    (100, 264, 384, 64, 64),
    (33, 136, 256, 16, 16),
    (9, 136, 512, 128, 128),      # A boxes of 16 and 32 rows for small batches
    (20, 264, 384, 64, 64),
])
def test_gate_pack_exact_on_grid_inputs(cuda_device, dtype, n, d, f, tile, cap):
    """Grid inputs make G exact in fp32, so counts, indices and values are
    bit-exact against the oracle, including overflow truncation."""
    inp = synth.make_grid_inputs(n, d, f, dtype, rho=0.05, seed=n + d)
    x, wg, _, _ = _dev(inp, cuda_device)
    diag = sge.new_diag(cuda_device)
    tw = sge.twell_gate_pack(x, wg, tile, cap, diag=diag)
    ora = oracle.twell_pack(oracle.gate_preact(inp.as_f64("x"), inp.as_f64("wg_t")), tile, cap,
                            KIND[dtype])
    torch.cuda.synchronize()
    assert_twell_equal(tw, ora)
    assert int(diag[0]) == ora.overflow


def test_gate_pack_identity_weights(cuda_device):
    """x := G (bf16), W_gate := I: the GEMM reproduces G exactly, so the
    epilogue's TwELL equals the oracle's pack of G bit for bit."""
    rng = np.random.default_rng(3)
    n, f = 384, 512
    g = torch.from_numpy(rng.standard_normal((n, f)) - 1.0).to(torch.bfloat16)
    eye = torch.eye(f, dtype=torch.bfloat16)
    tw = sge.twell_gate_pack(g.to(cuda_device), eye.to(cuda_device), 128, 128)
    ora = oracle.twell_pack(g.double().numpy(), 128, 128, oracle.VAL_BF16)
    torch.cuda.synchronize()
    assert_twell_equal(tw, ora)


@pytest.mark.parametrize("name,cap,n", [("ffn_0p5b_bf16", 128, 512), ("tiny_fp32", 64, 512),
                                        ("tiny_fp32", 16, 512), ("ffn_1b_bf16", 128, 100),
                                        ("ffn_1b_bf16", 128, 200)])
def test_gate_pack_gaussian_sign_flips(cuda_device, name, cap, n):
    """Realistic inputs: tiles disagree only where near-zero gates explain it
    (|g| < 1e-3); values agree within the fp32 accumulation bound.  100 and
    200 tokens take the single-CTA tiles of small batches."""
    cfg = synth.CONFIGS[name]
    inp = synth.make_inputs(cfg, n_tokens=n)
    x, wg, _, _ = _dev(inp, cuda_device)
    tw = sge.twell_gate_pack(x, wg, cfg.tile, cap)
    g = oracle.gate_preact(inp.as_f64("x"), inp.as_f64("wg_t"))
    kind = KIND[cfg.torch_dtype]
    ora = oracle.twell_pack(g, cfg.tile, cap, kind)
    torch.cuda.synchronize()
    abs_sum = np.abs(inp.as_f64("x")) @ np.abs(inp.as_f64("wg_t")).T
    _, _, bad_tiles, frac = compare_twell_inexact(tw, ora, g, kind, abs_sum, d_model=cfg.d_model)
    assert bad_tiles <= max(2, 0.002 * ora.count.size)
    print(f"{name} C={cap}: {bad_tiles} tiles differ by near-zero sign flips; values use "
          f"{frac:.2e} of the fp32 accumulation bound")


# ------------------------------------------------------------ fused up/down

@pytest.mark.parametrize("dtype,tol", [(torch.bfloat16, BF16_TOL), (torch.float32, F32_TOL)])
@pytest.mark.parametrize("n,d,f,tile,cap", [
    (300, 264, 640, 64, 64),      # d tail inside the last 16-byte chunk group
    (129, 1024, 512, 128, 128),
    (77, 520, 768, 32, 6),        # truncated tiles
    (64, 2560, 1024, 128, 128),   # the 2B d_model
    (200, 4096, 1024, 128, 128),  # the longest rows (8 KB in bf16): 16 pieces per lane
    (200, 2048, 1024, 128, 128),  # 8 KB rows in fp32
])
def test_fused_up_down_matches_oracle(cuda_device, dtype, tol, n, d, f, tile, cap):
    """Both sides get the same TwELL (the oracle's pack of its fp64 G)."""
    if dtype == torch.float32 and d > 2048:
        pytest.skip("fp32 rows are limited to d_model <= 2048 (test_fused_d_limit)")
    inp = synth.make_inputs(synth.CONFIGS["ffn_0p5b_bf16"].with_(
        n_tokens=n, d_model=d, d_ff=f, dtype="bf16" if dtype == torch.bfloat16 else "f32",
        rho=0.05))
    xf, wgf, wuf, wdf = _f64(inp)
    ora_tw = oracle.twell_pack(oracle.gate_preact(xf, wgf), tile, cap, KIND[dtype])
    x, _, wu, wd = _dev(inp, cuda_device)
    y = sge.twell_fused_up_down(x, _upload_twell(ora_tw, dtype, cuda_device), wu, wd)
    want = oracle.fused_up_down(xf, ora_tw, wuf, wdf)
    err = oracle.max_abs_rel(to_f64(y), want)
    assert err <= tol, err


@pytest.mark.parametrize("dtype,tol", [(torch.bfloat16, BF16_TOL), (torch.float32, F32_TOL)])
@pytest.mark.parametrize("n,d,f", [
    (300, 1024, 2048),            # rows of 512-byte multiples: one copy per entry when interleaved
    (300, 264, 640),              # ragged rows: two copies per entry in every layout
    (40, 512, 1024),              # the small-batch kernel
])
def test_fused_weight_layouts(cuda_device, dtype, tol, n, d, f):
    """W_up^T and W_down as separate matrices, interleaved row by row (one
    [F][2d] matrix), and with padded rows give the same bits, and match the
    oracle."""
    inp = synth.make_inputs(synth.CONFIGS["ffn_0p5b_bf16"].with_(
        n_tokens=n, d_model=d, d_ff=f, dtype="bf16" if dtype == torch.bfloat16 else "f32",
        rho=0.05))
    _, wgf, wuf, wdf = _f64(inp)
    x, _, wu, wd = _dev(inp, cuda_device)
    if n > 64:
        x[:3, :-1] *= 6.0          # heavy tokens: split units in the large-batch kernel
    xf = to_f64(x)
    ora_tw = oracle.twell_pack(oracle.gate_preact(xf, wgf), 128, 32, KIND[dtype])
    tw = _upload_twell(ora_tw, dtype, cuda_device)
    y_sep = sge.twell_fused_up_down(x, tw, wu, wd)
    w_ud, wu_i, wd_i = sge.interleave_up_down(wu, wd)
    assert torch.equal(w_ud[:, :d], wu) and torch.equal(w_ud[:, d:], wd)
    y_int = sge.twell_fused_up_down(x, tw, wu_i, wd_i)
    pad = torch.zeros((f, d + 40), dtype=dtype, device=cuda_device)
    pad2 = torch.zeros((f, d + 40), dtype=dtype, device=cuda_device)
    pad[:, :d] = wu
    pad2[:, :d] = wd
    y_pad = sge.twell_fused_up_down(x, tw, pad[:, :d], pad2[:, :d])
    torch.cuda.synchronize()
    assert torch.equal(y_sep, y_int)
    assert torch.equal(y_sep, y_pad)
    want = oracle.fused_up_down(xf, ora_tw, wuf, wdf)
    err = oracle.max_abs_rel(to_f64(y_int), want)
    assert err <= tol, err


def test_fused_rejects_mismatched_weight_strides(cuda_device):
    x = torch.zeros(4, 64, dtype=torch.bfloat16, device=cuda_device)
    w = torch.zeros(128, 64, dtype=torch.bfloat16, device=cuda_device)
    w2 = torch.zeros(128, 72, dtype=torch.bfloat16, device=cuda_device)
    tw = sge.TwELL.empty(4, 128, 128, 128, torch.bfloat16, cuda_device)
    tw.count.zero_()
    with pytest.raises(ValueError, match="row stride"):
        sge.twell_fused_up_down(x, tw, w, w2[:, :64])


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 4104), (torch.float32, 2056)])
def test_fused_d_limit(cuda_device, dtype, d):
    """A warp keeps at most 16 sixteen-byte pieces of a row per lane: rows of
    at most 8 KB (bf16 d <= 4096, fp32 d <= 2048); longer rows are rejected."""
    x = torch.zeros(4, d, dtype=dtype, device=cuda_device)
    w = torch.zeros(128, d, dtype=dtype, device=cuda_device)
    tw = sge.TwELL.empty(4, 128, 128, 128, dtype, cuda_device)
    tw.count.zero_()
    with pytest.raises(sge.LibraryError, match="too large"):
        sge.twell_fused_up_down(x, tw, w, w)


@pytest.mark.parametrize("dtype,tol", [(torch.bfloat16, BF16_TOL), (torch.float32, F32_TOL)])
def test_fused_heavy_and_light_tokens(cuda_device, dtype, tol):
    """Tokens far above the mean (split into units whose fp32 partial outputs
    are summed in unit order, several 32-entry chunks each) mixed with light
    ones; every row is checked."""
    n, d, f = 200, 264, 4096
    inp = synth.make_inputs(synth.CONFIGS["ffn_0p5b_bf16"].with_(
        n_tokens=n, d_model=d, d_ff=f, dtype="bf16" if dtype == torch.bfloat16 else "f32",
        rho=0.01))
    x = inp.x.clone()
    heavy = [0, 7, 8, 100, 199]
    x[heavy, :-1] *= 25.0        # these rows get hundreds to thousands of entries
    xf = x.double().numpy()
    wgf, wuf, wdf = inp.as_f64("wg_t"), inp.as_f64("wu_t"), inp.as_f64("wd")
    ora_tw = oracle.twell_pack(oracle.gate_preact(xf, wgf), 128, 128, KIND[dtype])
    nnz = np.minimum(ora_tw.count, 128).sum(1)
    assert nnz[heavy].min() > 600 and np.median(nnz) < 100
    y = sge.twell_fused_up_down(x.to(cuda_device), _upload_twell(ora_tw, dtype, cuda_device),
                                inp.wu_t.to(cuda_device), inp.wd.to(cuda_device))
    want = oracle.fused_up_down(xf, ora_tw, wuf, wdf)
    got = to_f64(y)
    for rows in (heavy, [r for r in range(n) if r not in heavy]):
        err = oracle.max_abs_rel(got[rows], want[rows])
        assert err <= tol, (rows[:3], err)


# Batches of at most 64 tokens take the small-batch path (units of E entries
# per CTA, one memory round trip per entry); these cases cover its row widths
# (2, 4 and 8 sixteen-byte pieces per lane), its tile-count widths (1 to 8
# registers of 32 tiles), truncated tiles and tokens split over many units.
@pytest.mark.parametrize("n,d,f,tile,cap,dt", [
    (1, 2048, 8192, 128, 128, "bf16"),   # one token, 8 pieces per lane
    (7, 264, 640, 64, 64, "f32"),        # ragged row: 66 pieces
    (33, 520, 768, 32, 6, "bf16"),       # truncated tiles
    (64, 1024, 8192, 32, 32, "bf16"),    # 256 tiles per row
    (40, 1024, 2048, 64, 64, "f32"),     # 4 KB fp32 rows
])
def test_fused_small_batch_matches_oracle(cuda_device, n, d, f, tile, cap, dt):
    dtype = torch.bfloat16 if dt == "bf16" else torch.float32
    tol = BF16_TOL if dt == "bf16" else F32_TOL
    inp = synth.make_inputs(synth.CONFIGS["ffn_0p5b_bf16"].with_(
        n_tokens=n, d_model=d, d_ff=f, dtype=dt, rho=0.05))
    xf, wgf, wuf, wdf = _f64(inp)
    ora_tw = oracle.twell_pack(oracle.gate_preact(xf, wgf), tile, cap, KIND[dtype])
    x, _, wu, wd = _dev(inp, cuda_device)
    y = sge.twell_fused_up_down(x, _upload_twell(ora_tw, dtype, cuda_device), wu, wd)
    want = oracle.fused_up_down(xf, ora_tw, wuf, wdf)
    err = oracle.max_abs_rel(to_f64(y), want)
    assert err <= tol, err


@pytest.mark.parametrize("dtype,tol", [(torch.bfloat16, BF16_TOL), (torch.float32, F32_TOL)])
def test_fused_small_batch_heavy_tokens(cuda_device, dtype, tol):
    """A 16-token batch whose heavy tokens hold thousands of entries: each is
    split into hundreds of units whose fp32 partials are summed in unit order
    by the CTA that completes the last one; every row is checked."""
    n, d, f = 16, 264, 4096
    inp = synth.make_inputs(synth.CONFIGS["ffn_0p5b_bf16"].with_(
        n_tokens=n, d_model=d, d_ff=f, dtype="bf16" if dtype == torch.bfloat16 else "f32",
        rho=0.01))
    x = inp.x.clone()
    heavy = [0, 5, 15]
    x[heavy, :-1] *= 25.0
    xf = x.double().numpy()
    wgf, wuf, wdf = inp.as_f64("wg_t"), inp.as_f64("wu_t"), inp.as_f64("wd")
    ora_tw = oracle.twell_pack(oracle.gate_preact(xf, wgf), 128, 128, KIND[dtype])
    nnz = np.minimum(ora_tw.count, 128).sum(1)
    assert nnz[heavy].min() > 600
    y = sge.twell_fused_up_down(x.to(cuda_device), _upload_twell(ora_tw, dtype, cuda_device),
                                inp.wu_t.to(cuda_device), inp.wd.to(cuda_device))
    want = oracle.fused_up_down(xf, ora_tw, wuf, wdf)
    got = to_f64(y)
    for rows in (heavy, [r for r in range(n) if r not in heavy]):
        err = oracle.max_abs_rel(got[rows], want[rows])
        assert err <= tol, (rows[:3], err)


def test_fused_small_batch_full_density(cuda_device):
    """64 tokens with every gate active: 4096 entries per token, more split
    units than the pool holds at the smallest unit length, so the planner
    doubles the unit length until the partials fit; the result is the dense
    FFN."""
    n, d, f = 64, 2048, 4096
    inp = synth.make_inputs(synth.CONFIGS["ffn_0p5b_bf16"].with_(n_tokens=n, d_model=d, d_ff=f),
                            tau=-1e3)
    x, wg, wu, wd = _dev(inp, cuda_device)
    y, tw = sge.twell_ffn_forward(x, wg, wu, wd, 128, 128)
    want = oracle.dense_ffn(*_f64(inp))
    torch.cuda.synchronize()
    assert int(tw.count.sum()) == n * f
    assert oracle.max_abs_rel(to_f64(y), want) <= BF16_TOL


def test_fused_small_batch_repeat_is_deterministic(cuda_device):
    cfg = synth.CONFIGS["decode_1b_bf16"]
    inp = synth.make_inputs(cfg)
    x, wg, wu, wd = _dev(inp, cuda_device)
    tw = sge.twell_gate_pack(x, wg, cfg.tile, cfg.cap)
    y1 = sge.twell_fused_up_down(x, tw, wu, wd)
    y2 = sge.twell_fused_up_down(x, tw, wu, wd)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_fused_up_down_repeat_is_deterministic(cuda_device):
    """Work is handed out dynamically; the result must not depend on it."""
    cfg = synth.CONFIGS["ffn_0p5b_bf16"]
    inp = synth.make_inputs(cfg, n_tokens=1024)
    x, wg, wu, wd = _dev(inp, cuda_device)
    tw = sge.twell_gate_pack(x, wg, cfg.tile, cfg.cap)
    y1 = sge.twell_fused_up_down(x, tw, wu, wd)
    y2 = sge.twell_fused_up_down(x, tw, wu, wd)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_fused_up_down_zero_density(cuda_device):
    n, d, f = 64, 256, 512
    inp = synth.make_inputs(synth.CONFIGS["ffn_0p5b_bf16"].with_(n_tokens=n, d_model=d, d_ff=f),
                            tau=1e4)
    x, wg, wu, wd = _dev(inp, cuda_device)
    y, tw = sge.twell_ffn_forward(x, wg, wu, wd, 128, 128)
    torch.cuda.synchronize()
    assert int(tw.count.sum()) == 0
    assert torch.all(y == 0)


def test_full_density_equals_dense(cuda_device):
    """tau -> -inf: every gate is active, TwELL with C = T is dense and the
    sparse forward equals the dense FFN (oracle)."""
    n, d, f = 96, 256, 512
    inp = synth.make_inputs(synth.CONFIGS["ffn_0p5b_bf16"].with_(n_tokens=n, d_model=d, d_ff=f),
                            tau=-1e3)
    x, wg, wu, wd = _dev(inp, cuda_device)
    y, tw = sge.twell_ffn_forward(x, wg, wu, wd, 128, 128)
    want = oracle.dense_ffn(*_f64(inp))
    torch.cuda.synchronize()
    assert int(tw.count.sum()) == n * f
    assert oracle.max_abs_rel(to_f64(y), want) <= BF16_TOL


# --------------------------------------------------------------- end to end

def _e2e_check(inp, dev, tile, cap, tol, rows=None, interleave=False, tau_shift=None):
    """Gate + TwELL and the fused up/down on the GPU; the oracle recomputes
    the rows ``rows`` (all when None) independently from the same inputs.
    TwELL tiles may differ only by near-zero sign flips (counted).  y is
    compared on every checked row: a flipped entry has |a| < 1e-3 and moves
    y far less than the bar; only a row whose flipped tile is truncated
    (count > C, so the stored window shifts) is left out, and there may be at
    most two such rows."""
    x, wg, wu, wd = _dev(inp, dev)
    if interleave:                 # the bench's weight layout
        _, wu, wd = sge.interleave_up_down(wu, wd)
    diag = sge.new_diag(dev)
    y, tw = sge.twell_ffn_forward(x, wg, wu, wd, tile, cap, diag=diag)
    torch.cuda.synchronize()
    return _e2e_compare(inp, tw, to_f64(y), tile, cap, tol, rows) + (int(diag[0]),)


def _e2e_compare(inp, tw, y_gpu, tile, cap, tol, rows=None):
    xf, wgf, wuf, wdf = _f64(inp)
    if rows is not None:
        xf = xf[rows]
        y_gpu = y_gpu[rows]
    kind = KIND[inp.x.dtype]
    y_ora, tw_ora, g = oracle.sparse_ffn(xf, wgf, wuf, wdf, tile, cap, kind)
    abs_sum = np.abs(xf) @ np.abs(wgf).T
    _, shifted, flips, frac = compare_twell_inexact(tw, tw_ora, g, kind, abs_sum, rows=rows,
                                                    d_model=xf.shape[1])
    assert shifted.sum() <= 2
    ok = ~shifted
    err = oracle.max_abs_rel(y_gpu[ok], y_ora[ok])
    assert err <= tol, err
    return err, flips, frac


def test_e2e_tiny_fp32(cuda_device):
    cfg = synth.CONFIGS["tiny_fp32"]
    inp = synth.make_inputs(cfg)
    err, flips, frac, over = _e2e_check(inp, cuda_device, cfg.tile, cfg.cap, F32_TOL)
    ora_over = oracle.twell_pack(oracle.gate_preact(inp.as_f64("x"), inp.as_f64("wg_t")),
                                 cfg.tile, cfg.cap, oracle.VAL_F32).overflow
    assert abs(over - ora_over) <= flips       # overflow count agrees up to flipped tiles
    print(f"tiny fp32: max-abs-rel {err:.2e}, {flips} flips, {over} overflowing tiles")


def test_e2e_0p5b_bf16_all_rows(cuda_device):
    cfg = synth.CONFIGS["ffn_0p5b_bf16"]
    err, flips, frac, _ = _e2e_check(synth.make_inputs(cfg), cuda_device, cfg.tile, cfg.cap,
                                     BF16_TOL)
    print(f"0.5B bf16: max-abs-rel {err:.2e} on all rows, {flips} flips")


@pytest.mark.parametrize("interleave", [True, False])
def test_e2e_1b_all_rows(cuda_device, interleave):
    """The headline 1B workload in the bench's launch configuration
    (interleaved weights; separate ones too), every row against the oracle."""
    inp = oracle_1b()[0]
    cfg = inp.cfg
    x, wg, wu, wd = _dev(inp, cuda_device)
    if interleave:
        _, wu, wd = sge.interleave_up_down(wu, wd)
    y, tw = sge.twell_ffn_forward(x, wg, wu, wd, cfg.tile, cfg.cap)
    torch.cuda.synchronize()
    err, flips = check_1b_all_rows(to_f64(y), tw)
    print(f"1B: max-abs-rel {err:.2e} on all {cfg.n_tokens} rows, {flips} flips")


@pytest.mark.parametrize("rho", [0.0025, 0.005, 0.01, 0.02, 0.05])
def test_e2e_2b_density_sweep(cuda_device, rho):
    """The 2B workload at each density of the sweep (the heavy tail grows
    with the density: at 5% tokens carry about 512 entries and the split-unit
    pool and the unit length run in their largest regime), interleaved
    weights as the bench runs it; the 128 heaviest tokens and every 4th
    token against the oracle."""
    cfg = synth.CONFIGS["ffn_2b_bf16"].with_(rho=rho)
    inp = synth.make_inputs(cfg)
    rows = heavy_and_strided_rows(inp)
    x, wg, wu, wd = _dev(inp, cuda_device)
    _, wu, wd = sge.interleave_up_down(wu, wd)
    y, tw = sge.twell_ffn_forward(x, wg, wu, wd, cfg.tile, cfg.cap)
    torch.cuda.synchronize()
    g0, abs0 = sweep_gate0(inp, rows)
    g = g0 - inp.tau
    tw_ora = oracle.twell_pack(g, cfg.tile, cfg.cap, oracle.VAL_BF16)
    y_ora = oracle.fused_up_down(inp.as_f64("x")[rows], tw_ora, inp.as_f64("wu_t"),
                                 inp.as_f64("wd"))
    _, shifted, flips, frac = compare_twell_inexact(tw, tw_ora, g, oracle.VAL_BF16,
                                                    abs0 + abs(inp.tau), rows=rows,
                                                    d_model=cfg.d_model)
    assert not shifted.any()          # C = T: no truncated tile
    err = oracle.max_abs_rel(to_f64(y)[rows], y_ora)
    assert err <= BF16_TOL, err
    heavy_n = int(tw_ora.count.astype(np.int64).sum(1).max())
    print(f"2B rho={rho}: max-abs-rel {err:.2e} on {len(rows)} rows (heaviest {heavy_n} "
          f"entries), {flips} flips")


# ------------------------------------------------------------ dense baseline

@pytest.mark.parametrize("n,d,f", [(300, 264, 640), (256, 1024, 2048)])
def test_dense_ffn_matches_oracle(cuda_device, n, d, f):
    inp = synth.make_inputs(synth.CONFIGS["ffn_0p5b_bf16"].with_(n_tokens=n, d_model=d, d_ff=f,
                                                                 rho=0.3))
    x, wg, wu, wd = _dev(inp, cuda_device)
    y = sge.dense_ffn_fwd(x, wg, wu, wd.t().contiguous())
    want = oracle.dense_ffn(*_f64(inp))
    err = oracle.max_abs_rel(to_f64(y), want)
    assert err <= BF16_TOL, err


def test_dense_ffn_full_size_sampled(cuda_device):
    cfg = synth.CONFIGS["ffn_1b_bf16"]
    inp = synth.make_inputs(cfg)
    x, wg, wu, wd = _dev(inp, cuda_device)
    y = sge.dense_ffn_fwd(x, wg, wu, wd.t().contiguous())
    rows = np.arange(3, cfg.n_tokens, cfg.n_tokens // 16)
    xf, wgf, wuf, wdf = _f64(inp)
    want = oracle.dense_ffn(xf[rows], wgf, wuf, wdf)
    err = oracle.max_abs_rel(to_f64(y)[rows], want)
    assert err <= BF16_TOL, err


def test_diag_counts_overflow_tiles(cuda_device):
    cfg = synth.CONFIGS["tiny_fp32"]
    inp = synth.make_grid_inputs(256, 256, 1024, torch.float32, rho=0.05)
    x, wg, _, _ = _dev(inp, cuda_device)
    diag = sge.new_diag(cuda_device)
    sge.twell_gate_pack(x, wg, 64, 4, diag=diag)
    sge.twell_gate_pack(x, wg, 64, 4, diag=diag)       # accumulates
    ora = oracle.twell_pack(oracle.gate_preact(inp.as_f64("x"), inp.as_f64("wg_t")), 64, 4,
                            oracle.VAL_F32)
    torch.cuda.synchronize()
    assert int(diag[0]) == 2 * ora.overflow
    assert int(diag[3]) == 0


def test_library_errors_raise(cuda_device):
    x = torch.zeros(8, 64, dtype=torch.bfloat16, device=cuda_device)
    w = torch.zeros(200, 64, dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(sge.LibraryError):
        sge.twell_gate_pack(x, w, 64, 64)          # 64 does not divide 200
