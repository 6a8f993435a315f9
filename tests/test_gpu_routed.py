"""GPU parity of the routed forward (twell_hybrid_up_down: light tokens per
entry from TwELL, heavy tokens on the tensor-core spill GEMMs) against the
fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import activation_sparse_gated_epilogue_b200 as sge
import oracle
from activation_sparse_gated_epilogue_b200 import synth
from tests._util import (BF16_TOL, check_1b_all_rows, compare_twell_inexact,
                         heavy_and_strided_rows, oracle_1b, sweep_gate0, to_f64)

pytestmark = pytest.mark.gpu


def _inputs(n, d, f, seed=0, rho=0.02, heavy=7, scale=3.0):
    """bf16 inputs of the 0.5B recipe at the given sizes, with the first
    `heavy` tokens' features scaled so that they carry many active gates."""
    cfg = synth.CONFIGS["ffn_0p5b_bf16"].with_(n_tokens=n, d_model=d, d_ff=f, rho=rho, seed=seed)
    inp = synth.make_inputs(cfg)
    inp.x[:heavy, :-1] *= scale          # exact in bf16 for powers of two
    return inp


def _upload(tw: oracle.TwELL, dev):
    return sge.TwELL(torch.from_numpy(tw.count).to(dev), torch.from_numpy(tw.idx).to(dev),
                     torch.from_numpy(tw.val).to(torch.bfloat16).to(dev), tw.tile, tw.cap)


def _stored(tw: oracle.TwELL) -> np.ndarray:
    return np.minimum(tw.count, tw.cap).astype(np.int64).sum(1)


@pytest.mark.parametrize("n,d,f,tile,cap,k,s_max", [
    (300, 256, 1024, 128, 128, 16, 64),     # heavy tokens in the spill, light per entry
    (300, 256, 1024, 128, 128, 16, 4),      # heavy tokens past S_max run per entry
    (300, 256, 1024, 128, 128, 0, 300),     # every non-empty token spills
    (520, 264, 768, 64, 64, 8, 520),        # ragged d and a ragged last spill tile
    (700, 1024, 2048, 128, 128, 32, 512),   # several 256-row spill tiles
    (257, 512, 1024, 128, 16, 24, 64),      # truncated tiles: stored entries only
    (129, 2560, 1024, 128, 128, 8, 128),    # the 2B d_model (rows of 5 KB)
])
def test_routed_matches_oracle(cuda_device, n, d, f, tile, cap, k, s_max):
    """Both sides get the oracle's TwELL: y equals the oracle's fused up/down
    over the stored entries, and diag counts the heavy tokens."""
    inp = _inputs(n, d, f, seed=n + k)
    xf, wgf, wuf, wdf = (inp.as_f64(nm) for nm in ("x", "wg_t", "wu_t", "wd"))
    tw_ora = oracle.twell_pack(oracle.gate_preact(xf, wgf), tile, cap, oracle.VAL_BF16)
    want = oracle.fused_up_down(xf, tw_ora, wuf, wdf)
    heavy = int((_stored(tw_ora) > k).sum())
    assert heavy > 0
    dev = cuda_device
    x, wu, wd = (getattr(inp, nm).to(dev) for nm in ("x", "wu_t", "wd"))
    diag = sge.new_diag(dev)
    y = sge.twell_hybrid_up_down(x, _upload(tw_ora, dev), wu, wd, wd.t().contiguous(), k, s_max,
                                 diag=diag)
    torch.cuda.synchronize()
    err = oracle.max_abs_rel(to_f64(y), want)
    assert err <= BF16_TOL, err
    assert int(diag[1]) == heavy and int(diag[3]) == 0


@pytest.mark.parametrize("k,s_max", [(16, 64), (16, 4)])
def test_routed_weight_layouts_and_repeats_give_the_same_bits(cuda_device, k, s_max):
    """Separate and interleaved weights, and repeated calls, give identical
    bits (no atomics on data, fixed summation orders)."""
    inp = _inputs(300, 256, 1024, seed=5)
    tw_ora = oracle.twell_pack(oracle.gate_preact(inp.as_f64("x"), inp.as_f64("wg_t")), 128, 128,
                               oracle.VAL_BF16)
    dev = cuda_device
    x, wu, wd = (getattr(inp, nm).to(dev) for nm in ("x", "wu_t", "wd"))
    tw = _upload(tw_ora, dev)
    wd_t = wd.t().contiguous()
    a = sge.twell_hybrid_up_down(x, tw, wu, wd, wd_t, k, s_max)
    _, wu_i, wd_i = sge.interleave_up_down(wu, wd)
    b = sge.twell_hybrid_up_down(x, tw, wu_i, wd_i, wd_t, k, s_max)
    c = sge.twell_hybrid_up_down(x, tw, wu_i, wd_i, wd_t, k, s_max)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(b, c)


def test_routed_small_batch_runs_per_entry(cuda_device):
    """At most 64 tokens: every token takes the per-entry path, bit for bit
    the result of twell_fused_up_down."""
    inp = _inputs(48, 1024, 2048, seed=9, heavy=5)
    tw_ora = oracle.twell_pack(oracle.gate_preact(inp.as_f64("x"), inp.as_f64("wg_t")), 128, 128,
                               oracle.VAL_BF16)
    dev = cuda_device
    x, wu, wd = (getattr(inp, nm).to(dev) for nm in ("x", "wu_t", "wd"))
    tw = _upload(tw_ora, dev)
    y = sge.twell_hybrid_up_down(x, tw, wu, wd, wd.t().contiguous(), 8, 16)
    y_f = sge.twell_fused_up_down(x, tw, wu, wd)
    torch.cuda.synchronize()
    assert torch.equal(y, y_f)
    want = oracle.fused_up_down(inp.as_f64("x"), tw_ora, inp.as_f64("wu_t"), inp.as_f64("wd"))
    assert oracle.max_abs_rel(to_f64(y), want) <= BF16_TOL


def test_routed_zero_and_full_density(cuda_device):
    """No active gate: y = 0 exactly.  Every gate active (C = T): every token
    spills and y equals the dense FFN."""
    n, d, f = 300, 256, 512
    dev = cuda_device
    for tau, check in ((1e3, "zero"), (-1e3, "dense")):
        cfg = synth.CONFIGS["ffn_0p5b_bf16"].with_(n_tokens=n, d_model=d, d_ff=f)
        inp = synth.make_inputs(cfg, tau=tau)
        x, wg, wu, wd = (getattr(inp, nm).to(dev) for nm in ("x", "wg_t", "wu_t", "wd"))
        tw = sge.twell_gate_pack(x, wg, 128, 128)
        y = sge.twell_hybrid_up_down(x, tw, wu, wd, wd.t().contiguous(), 32, n)
        torch.cuda.synchronize()
        if check == "zero":
            assert int(tw.count.sum()) == 0 and not y.any()
        else:
            assert int(tw.count.sum()) == n * f
            want = oracle.dense_ffn(*(inp.as_f64(nm) for nm in ("x", "wg_t", "wu_t", "wd")))
            assert oracle.max_abs_rel(to_f64(y), want) <= BF16_TOL


@pytest.mark.parametrize("k,s_div", [(16, 1), (32, 4), (64, 4), (128, 4)])
def test_routed_1b_all_rows(cuda_device, k, s_div):
    """The 1B workload (gate GEMM + TwELL on the GPU, interleaved weights),
    every row against the oracle.  K = F/512 = 16 with S_max = N is the
    launch configuration bench.py times; the others move the light/heavy
    boundary and cap the spill at N/4."""
    inp = oracle_1b()[0]
    cfg = inp.cfg
    dev = cuda_device
    x, wg, wu, wd = (getattr(inp, nm).to(dev) for nm in ("x", "wg_t", "wu_t", "wd"))
    _, wu_i, wd_i = sge.interleave_up_down(wu, wd)
    tw = sge.twell_gate_pack(x, wg, cfg.tile, cfg.cap)
    diag = sge.new_diag(dev)
    y = sge.twell_hybrid_up_down(x, tw, wu_i, wd_i, wd.t().contiguous(), k, cfg.n_tokens // s_div,
                                 diag=diag)
    torch.cuda.synchronize()
    assert int(diag[3]) == 0
    err, flips = check_1b_all_rows(to_f64(y), tw)
    print(f"routed 1B K={k}: {int(diag[1])} spill rows, max-abs-rel {err:.2e}, {flips} flips")


@pytest.mark.parametrize("rho,k,s_div", [
    (0.0025, 20, 1), (0.005, 20, 1), (0.01, 20, 1), (0.02, 20, 1), (0.05, 20, 1),
    (0.0025, 64, 4), (0.05, 64, 4),
])
def test_routed_2b_sweep(cuda_device, rho, k, s_div):
    """The 2B workload at every density of the sweep in bench.py's launch
    configuration (K = F/512 = 20, S_max = N), and at the lightest and
    densest points with K = 64, S_max = N/4 (at 5% most tokens are heavy and
    those past S_max run per entry): the 128 heaviest tokens and every 4th
    token against the oracle."""
    cfg = synth.CONFIGS["ffn_2b_bf16"].with_(rho=rho)
    inp = synth.make_inputs(cfg)
    rows = heavy_and_strided_rows(inp)
    dev = cuda_device
    x, wg, wu, wd = (getattr(inp, nm).to(dev) for nm in ("x", "wg_t", "wu_t", "wd"))
    _, wu_i, wd_i = sge.interleave_up_down(wu, wd)
    tw = sge.twell_gate_pack(x, wg, cfg.tile, cfg.cap)
    diag = sge.new_diag(dev)
    y = sge.twell_hybrid_up_down(x, tw, wu_i, wd_i, wd.t().contiguous(), k, cfg.n_tokens // s_div,
                                 diag=diag)
    torch.cuda.synchronize()
    assert int(diag[3]) == 0
    g0, abs0 = sweep_gate0(inp, rows)
    g = g0 - inp.tau
    tw_ora = oracle.twell_pack(g, cfg.tile, cfg.cap, oracle.VAL_BF16)
    y_ora = oracle.fused_up_down(inp.as_f64("x")[rows], tw_ora, inp.as_f64("wu_t"), inp.as_f64("wd"))
    _, shifted, flips, _ = compare_twell_inexact(tw, tw_ora, g, oracle.VAL_BF16, abs0 + abs(inp.tau),
                                                 rows=rows, d_model=cfg.d_model)
    assert not shifted.any()
    err = oracle.max_abs_rel(to_f64(y)[rows], y_ora)
    assert err <= BF16_TOL, err
    print(f"routed 2B rho={rho} K={k}: {int(diag[1])} heavy tokens, max-abs-rel {err:.2e}, {flips} flips")


@pytest.mark.parametrize("n", [64, 32, 8, 1])
def test_routed_decode_1b_all_rows(cuda_device, n):
    """The decode-shaped workload (a small batch against the 1B weights) as
    bench.py runs it: the gate GEMM on single-CTA tiles, then the routed call
    with K = F/512 = 16, S_max = N, which takes the small-batch path; every
    row against the oracle's whole forward."""
    cfg = synth.CONFIGS["decode_1b_bf16"].with_(n_tokens=n)
    inp = synth.make_inputs(cfg)
    dev = cuda_device
    x, wg, wu, wd = (getattr(inp, nm).to(dev) for nm in ("x", "wg_t", "wu_t", "wd"))
    _, wu_i, wd_i = sge.interleave_up_down(wu, wd)
    tw = sge.twell_gate_pack(x, wg, cfg.tile, cfg.cap)
    diag = sge.new_diag(dev)
    y = sge.twell_hybrid_up_down(x, tw, wu_i, wd_i, wd.t().contiguous(), cfg.d_ff // 512, n,
                                 diag=diag)
    torch.cuda.synchronize()
    assert int(diag[3]) == 0
    xf, wgf, wuf, wdf = (inp.as_f64(nm) for nm in ("x", "wg_t", "wu_t", "wd"))
    y_ora, tw_ora, g = oracle.sparse_ffn(xf, wgf, wuf, wdf, cfg.tile, cfg.cap, oracle.VAL_BF16)
    abs_sum = np.abs(xf) @ np.abs(wgf).T
    _, shifted, flips, _ = compare_twell_inexact(tw, tw_ora, g, oracle.VAL_BF16, abs_sum,
                                                 d_model=cfg.d_model)
    assert not shifted.any()          # C = T: no truncated tile
    err = oracle.max_abs_rel(to_f64(y), y_ora)
    assert err <= BF16_TOL, err
    print(f"routed decode N={n}: max-abs-rel {err:.2e}, {flips} flips")


def test_routed_heavy_tokens_past_s_max(cuda_device):
    """Every gate active with F = 1536 and S_max = 8: the first 8 tokens take
    the spill GEMMs, the other 292 (1536 entries each) take the CUDA-core
    kernel in rounds of 512 entries; y equals the dense FFN."""
    n, d, f = 300, 256, 1536
    cfg = synth.CONFIGS["ffn_0p5b_bf16"].with_(n_tokens=n, d_model=d, d_ff=f)
    inp = synth.make_inputs(cfg, tau=-1e3)
    dev = cuda_device
    x, wg, wu, wd = (getattr(inp, nm).to(dev) for nm in ("x", "wg_t", "wu_t", "wd"))
    tw = sge.twell_gate_pack(x, wg, 128, 128)
    diag = sge.new_diag(dev)
    y = sge.twell_hybrid_up_down(x, tw, wu, wd, wd.t().contiguous(), 64, 8, diag=diag)
    torch.cuda.synchronize()
    assert int(tw.count.sum()) == n * f and int(diag[1]) == n
    want = oracle.dense_ffn(*(inp.as_f64(nm) for nm in ("x", "wg_t", "wu_t", "wd")))
    assert oracle.max_abs_rel(to_f64(y), want) <= BF16_TOL
