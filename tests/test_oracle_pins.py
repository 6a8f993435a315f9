"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test ties one oracle function to a library routine, a closed form, a
format invariant or brute force on tiny inputs, chosen so that a dropped term,
a wrong sign or index, or a transposed operand in the oracle fails at least
one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from activation_sparse_gated_epilogue_b200 import synth


def _rand(rng, *shape):
    return rng.standard_normal(shape)


# ------------------------------------------------------------------ rounding

def _round_cases(dt, seed):
    rng = np.random.default_rng(seed)
    fi = torch.finfo(dt)
    v = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-8, 8, 20000),
        rng.standard_normal(2000) * float(fi.tiny),          # subnormal range
        rng.standard_normal(2000) * float(fi.max),            # around overflow
        [0.0, -0.0, np.inf, -np.inf, float(fi.max), -float(fi.max)],
    ])
    # exact ties: midpoints between neighbouring representable values
    base = torch.from_numpy(rng.standard_normal(4000)).to(dt)
    nxt = torch.nextafter(base, torch.full_like(base, float("inf")))
    ties = (base.double() + nxt.double()) / 2
    return np.concatenate([v, ties.numpy()])


@pytest.mark.parametrize("kind,dt", [(oracle.VAL_BF16, torch.bfloat16),
                                     (oracle.VAL_F16, torch.float16)])
def test_round_matches_torch_cast_from_f32(kind, dt):
    """Round-to-nearest-even to bf16 / fp16 equals torch's cast of the same
    float32 values (one rounding on both sides) on normals, subnormals, exact
    ties, overflow and specials."""
    with np.errstate(over="ignore"):
        v32 = _round_cases(dt, 1).astype(np.float32)
    want = torch.from_numpy(v32).to(dt).double().numpy()
    got = oracle.round_array(v32.astype(np.float64), kind)
    np.testing.assert_array_equal(got, want)
    assert math.isnan(oracle.round_value(float("nan"), kind))


def test_round_f16_matches_numpy_from_f64():
    """float64 -> float16 in one rounding equals numpy's direct cast."""
    v = _round_cases(torch.float16, 2)
    with np.errstate(over="ignore"):
        want = v.astype(np.float16).astype(np.float64)
    np.testing.assert_array_equal(oracle.round_array(v, oracle.VAL_F16), want)


def test_round_f32_matches_numpy_from_f64():
    v = _round_cases(torch.float32, 3)
    with np.errstate(over="ignore"):
        want = v.astype(np.float32).astype(np.float64)
    np.testing.assert_array_equal(oracle.round_array(v, oracle.VAL_F32), want)


def test_round_f64_is_identity():
    v = np.random.default_rng(2).standard_normal(1000)
    np.testing.assert_array_equal(oracle.round_array(v, oracle.VAL_F64), v)


# --------------------------------------------------------------- gate GEMM

def test_gate_preact_matches_numpy_matmul():
    rng = np.random.default_rng(3)
    x, wg = _rand(rng, 37, 53), _rand(rng, 71, 53)
    g = oracle.gate_preact(x, wg)
    np.testing.assert_allclose(g, x @ wg.T, rtol=1e-12, atol=1e-12)


def test_gate_preact_not_transposed():
    """A non-square case where x W and x W^T differ in shape and value."""
    rng = np.random.default_rng(4)
    x, wg = _rand(rng, 3, 5), _rand(rng, 7, 5)
    g = oracle.gate_preact(x, wg)
    assert g.shape == (3, 7)
    assert g[1, 4] == pytest.approx(sum(x[1, i] * wg[4, i] for i in range(5)), rel=1e-14)


# ------------------------------------------------------------- TwELL pack

def _brute_twell(g, tile, cap, kind):
    """Brute force: per tile, numpy's list of positive positions."""
    n, f = g.shape
    out = {}
    for t in range(n):
        for b in range(f // tile):
            seg = g[t, b * tile:(b + 1) * tile]
            pos = np.flatnonzero(seg > 0)
            out[(t, b)] = (len(pos), list(pos[:cap]),
                           [oracle.round_value(seg[p], kind) for p in pos[:cap]])
    return out


@pytest.mark.parametrize("tile,cap", [(4, 4), (8, 3), (8, 8), (16, 5)])
@pytest.mark.parametrize("kind", [oracle.VAL_F64, oracle.VAL_BF16])
def test_twell_pack_brute_force(tile, cap, kind):
    rng = np.random.default_rng(5 + tile + cap)
    g = _rand(rng, 8, 32)
    g[0, :5] = 0.0          # zeros are inactive
    g[1, 3] = -0.0
    g[2, 7] = np.nan        # NaN is inactive
    tw = oracle.twell_pack(g, tile, cap, kind)
    ref = _brute_twell(g, tile, cap, kind)
    over = 0
    for (t, b), (c, pos, vals) in ref.items():
        assert tw.count[t, b] == c
        k = min(c, cap)
        assert list(tw.idx[t, b, :k]) == pos
        np.testing.assert_array_equal(tw.val[t, b, :k], vals)
        over += c > cap
    assert tw.overflow == over


def test_twell_invariants_and_unpack():
    """count == nnz, local indices ascending and inside the tile, and
    unpack(pack(G)) == ReLU(G) exactly when no tile overflows (C = T)."""
    rng = np.random.default_rng(6)
    g = _rand(rng, 64, 256) - 1.5
    tw = oracle.twell_pack(g, 64, 64, oracle.VAL_F64)
    assert tw.overflow == 0
    np.testing.assert_array_equal(tw.count, (g > 0).reshape(64, 4, 64).sum(-1))
    for t in range(64):
        for b in range(4):
            c = tw.count[t, b]
            ii = tw.idx[t, b, :c].astype(int)
            assert np.all(np.diff(ii) > 0) and np.all(ii < 64)
    np.testing.assert_array_equal(oracle.twell_unpack(tw), np.maximum(g, 0.0))


def test_twell_unpack_with_overflow_keeps_first_c():
    rng = np.random.default_rng(7)
    g = np.abs(_rand(rng, 4, 32)) + 0.1       # every gate active
    tw = oracle.twell_pack(g, 16, 5, oracle.VAL_F64)
    assert tw.overflow == 8 and np.all(tw.count == 16)
    h = oracle.twell_unpack(tw)
    want = np.zeros_like(g)
    for b in range(2):
        want[:, b * 16:b * 16 + 5] = g[:, b * 16:b * 16 + 5]
    np.testing.assert_array_equal(h, want)


# --------------------------------------------------------- FFN definitions

def _numpy_ffn(x, wg, wu, wd):
    return (np.maximum(x @ wg.T, 0.0) * (x @ wu.T)) @ wd


def test_dense_ffn_matches_numpy():
    rng = np.random.default_rng(8)
    x, wg, wu, wd = _rand(rng, 19, 24), _rand(rng, 40, 24), _rand(rng, 40, 24), _rand(rng, 40, 24)
    y = oracle.dense_ffn(x, wg, wu, wd)
    np.testing.assert_allclose(y, _numpy_ffn(x, wg, wu, wd), rtol=1e-11, atol=1e-11)


def test_sparse_equals_dense_exactly_when_lossless():
    """With fp64 values and C = T the sparse path adds exactly the dense
    path's nonzero terms in the same order: equal bit for bit."""
    rng = np.random.default_rng(9)
    x, wg, wu, wd = _rand(rng, 16, 32), _rand(rng, 64, 32), _rand(rng, 64, 32), _rand(rng, 64, 32)
    y, tw, _ = oracle.sparse_ffn(x, wg, wu, wd, 16, 16, oracle.VAL_F64)
    np.testing.assert_array_equal(y, oracle.dense_ffn(x, wg, wu, wd))


def test_sparse_with_overflow_matches_truncated_numpy():
    """With C < T the path uses exactly the stored entries: it equals
    (unpack(TwELL) (.) x W_up) W_down computed by numpy."""
    cfg = synth.CONFIGS["tiny_fp32"]
    inp = synth.make_inputs(cfg, n_tokens=64)
    x, wg, wu, wd = (inp.as_f64(k) for k in ("x", "wg_t", "wu_t", "wd"))
    y, tw, g = oracle.sparse_ffn(x, wg, wu, wd, cfg.tile, cfg.cap, oracle.VAL_F32)
    h = oracle.twell_unpack(tw)
    want = (h * (x @ wu.T)) @ wd
    np.testing.assert_allclose(y, want, rtol=1e-10, atol=1e-12)


def test_zero_density_gives_zero_output():
    rng = np.random.default_rng(10)
    x, wu, wd = _rand(rng, 8, 16), _rand(rng, 32, 16), _rand(rng, 32, 16)
    x[:, -1] = 1.0
    wg = _rand(rng, 32, 16) * 0.01
    wg[:, -1] = -1e6
    y, tw, _ = oracle.sparse_ffn(x, wg, wu, wd, 8, 8, oracle.VAL_BF16)
    assert np.all(tw.count == 0)
    assert np.all(y == 0.0)


def test_full_density_gives_dense_output():
    rng = np.random.default_rng(11)
    x, wu, wd = _rand(rng, 8, 16), _rand(rng, 32, 16), _rand(rng, 32, 16)
    x[:, -1] = 1.0
    wg = _rand(rng, 32, 16) * 0.01
    wg[:, -1] = 1e3
    y, tw, _ = oracle.sparse_ffn(x, wg, wu, wd, 8, 8, oracle.VAL_F64)
    assert np.all(tw.count == 8)
    np.testing.assert_allclose(y, _numpy_ffn(x, wg, wu, wd), rtol=1e-11, atol=1e-9)


# ------------------------------------------------------------------ hybrid

def _tw(seed, n=32, f=64, tile=16, shift=1.0, cap=None):
    rng = np.random.default_rng(seed)
    g = _rand(rng, n, f) - shift
    g[:3] += 3.0       # a few heavy rows
    return oracle.twell_pack(g, tile, cap or tile, oracle.VAL_F64), g


@pytest.mark.parametrize("k,s_max", [(8, 32), (4, 32), (8, 2), (0, 32), (64, 32)])
def test_hybrid_pack_invariants(k, s_max):
    tw, g = _tw(12)
    hy = oracle.hybrid_pack(tw, k, s_max)
    nnz = (g > 0).sum(1)
    np.testing.assert_array_equal(hy.row_nnz, nnz)
    spill = nnz > k
    assert hy.n_spill == spill.sum()
    ell_rows = (~spill).sum()
    assert ell_rows + hy.n_spill == tw.n_rows                 # every row is routed once
    assert hy.dropped == max(0, hy.n_spill - s_max)
    np.testing.assert_array_equal(hy.spill_rows, np.flatnonzero(spill)[:s_max])  # ascending t
    for t in range(tw.n_rows):
        if not spill[t]:
            assert hy.spill_slot[t] == -1
            c = nnz[t]
            np.testing.assert_array_equal(hy.ell_idx[t, :c], np.flatnonzero(g[t] > 0))
            np.testing.assert_array_equal(hy.ell_a[t, :c], g[t][g[t] > 0])
            assert np.all(hy.ell_idx[t, c:] == -1)
        elif hy.spill_slot[t] >= 0:
            np.testing.assert_array_equal(hy.spill_a[hy.spill_slot[t]], np.maximum(g[t], 0))
    if k >= tw.n_cols:
        assert hy.n_spill == 0
    if k == 0:
        assert hy.n_spill == (nnz > 0).sum()


def test_hybrid_pack_routes_overflowing_rows_to_spill():
    """Capacity C below the tile width: a row with a tile holding more than C
    active gates has lost entries and goes to the spill even when its stored
    count fits K (its row_nnz is then K + 1); rows without overflow route by
    their count as before; the spill row holds the stored (first C per tile)
    entries."""
    tile, cap, k = 8, 2, 6
    f = 32
    g = np.full((4, f), -1.0)
    g[0, [1, 5]] = [0.5, 0.25]            # 2 entries in tile 0: fits C, ELL
    g[1, [0, 1, 2]] = [1.0, 2.0, 3.0]     # 3 entries in tile 0 > C: spill, K + 1
    g[2, [0, 9, 17, 25]] = 1.5            # 4 entries, one per tile: ELL
    g[3, :] = 0.75                        # every gate: 4 tiles x 8 > C: spill
    tw = oracle.twell_pack(g, tile, cap, oracle.VAL_F64)
    assert tw.overflow == 2 * 0 + 1 + 4
    hy = oracle.hybrid_pack(tw, k, 8)
    np.testing.assert_array_equal(hy.row_nnz, [2, k + 1, 4, 8])
    np.testing.assert_array_equal(hy.spill_slot, [-1, 0, -1, 1])
    np.testing.assert_array_equal(hy.spill_rows, [1, 3])
    assert hy.n_spill == 2 and hy.dropped == 0
    want1 = np.zeros(f); want1[[0, 1]] = [1.0, 2.0]     # the first C of tile 0
    np.testing.assert_array_equal(hy.spill_a[0], want1)
    want3 = np.zeros(f)
    for b in range(f // tile):
        want3[b * tile:b * tile + cap] = 0.75
    np.testing.assert_array_equal(hy.spill_a[1], want3)
    np.testing.assert_array_equal(hy.ell_idx[0, :2], [1, 5])
    np.testing.assert_array_equal(hy.ell_idx[2, :4], [0, 9, 17, 25])


def _hy_inputs(seed, n=24, d=16, f=64, shift=1.2):
    rng = np.random.default_rng(seed)
    x, wg, wu, wd = _rand(rng, n, d), _rand(rng, f, d), _rand(rng, f, d), _rand(rng, f, d)
    x[:, -1] = 1.0
    wg[:, -1] = -shift
    x[:2, :-1] *= 4.0          # heavy rows
    return x, wg, wu, wd


@pytest.mark.parametrize("k,s_max", [(6, 24), (0, 24), (64, 24), (6, 1)])
def test_hybrid_fwd_matches_numpy(k, s_max):
    x, wg, wu, wd = _hy_inputs(13)
    g = x @ wg.T
    tw = oracle.twell_pack(oracle.gate_preact(x, wg), 16, 16, oracle.VAL_F64)
    hy = oracle.hybrid_pack(tw, k, s_max)
    y = oracle.hybrid_fwd(x, hy, wu, wd)
    keep = np.ones(x.shape[0], bool)
    keep[(hy.row_nnz > k) & (hy.spill_slot < 0)] = False        # dropped rows
    want = (np.maximum(g, 0) * (x @ wu.T)) @ wd
    want[~keep] = 0.0
    np.testing.assert_allclose(y, want, rtol=1e-10, atol=1e-10)
    u = x @ wu.T
    for t in range(x.shape[0]):
        if hy.row_nnz[t] <= k:
            c = hy.row_nnz[t]
            np.testing.assert_allclose(hy.ell_u[t, :c], u[t, hy.ell_idx[t, :c]], rtol=1e-12, atol=1e-12)
        elif hy.spill_slot[t] >= 0:
            np.testing.assert_allclose(hy.spill_u[hy.spill_slot[t]], u[t], rtol=1e-12, atol=1e-12)


def _torch_grads(x, wg, wu, wd, dy, keep):
    tx, twg, twu, twd = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (x, wg, wu, wd))
    y = (torch.relu(tx @ twg.T) * (tx @ twu.T)) @ twd
    y = y * torch.tensor(keep, dtype=torch.float64)[:, None]
    (y * torch.tensor(dy)).sum().backward()
    return [a.grad.numpy() for a in (tx, twg, twu, twd)]


@pytest.mark.parametrize("k,s_max", [(6, 24), (0, 24), (64, 24), (6, 1)])
def test_hybrid_bwd_matches_torch_autograd(k, s_max):
    x, wg, wu, wd = _hy_inputs(14)
    dy = _rand(np.random.default_rng(15), *x.shape)
    tw = oracle.twell_pack(oracle.gate_preact(x, wg), 16, 16, oracle.VAL_F64)
    hy = oracle.hybrid_pack(tw, k, s_max)
    oracle.hybrid_fwd(x, hy, wu, wd)
    got = oracle.hybrid_bwd(x, dy, hy, wg, wu, wd)
    keep = ~((hy.row_nnz > k) & (hy.spill_slot < 0))
    want = _torch_grads(x, wg, wu, wd, dy, keep)
    for a, b in zip(got, want):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-10)


def test_hybrid_bwd_central_differences():
    """Directional derivatives of L = <dy, y(x, W)> by central differences of
    the oracle's own forward (away from the ReLU kink)."""
    x, wg, wu, wd = _hy_inputs(16, n=6, d=8, f=32, shift=0.8)
    dy = _rand(np.random.default_rng(17), *x.shape)

    def loss(x_, wg_, wu_, wd_):
        tw = oracle.twell_pack(oracle.gate_preact(x_, wg_), 16, 16, oracle.VAL_F64)
        hy = oracle.hybrid_pack(tw, 4, 6)
        return float((oracle.hybrid_fwd(x_, hy, wu_, wd_) * dy).sum()), hy

    _, hy = loss(x, wg, wu, wd)
    g = x @ wg.T
    assert np.min(np.abs(g)) > 1e-6
    grads = oracle.hybrid_bwd(x, dy, hy, wg, wu, wd)
    rng = np.random.default_rng(18)
    eps = 1e-6
    for which in range(4):
        args = [x, wg, wu, wd]
        v = _rand(rng, *args[which].shape)
        if which == 0:
            v[:, -1] = 0.0             # the bias feature is a constant 1
        plus = list(args); plus[which] = args[which] + eps * v
        minus = list(args); minus[which] = args[which] - eps * v
        fd = (loss(*plus)[0] - loss(*minus)[0]) / (2 * eps)
        an = float((grads[which] * v).sum())
        assert fd == pytest.approx(an, rel=1e-6, abs=1e-8), which


def test_hybrid_zero_density_gives_zero_grads():
    x, wg, wu, wd = _hy_inputs(19)
    wg[:, -1] = -1e6
    dy = _rand(np.random.default_rng(20), *x.shape)
    tw = oracle.twell_pack(oracle.gate_preact(x, wg), 16, 16, oracle.VAL_F64)
    hy = oracle.hybrid_pack(tw, 4, 24)
    y = oracle.hybrid_fwd(x, hy, wu, wd)
    assert np.all(y == 0)
    for a in oracle.hybrid_bwd(x, dy, hy, wg, wu, wd):
        assert np.all(a == 0)


# ---------------------------------------------------------------- recipe

def test_generator_realised_density_near_target():
    """The solved tau gives the intended mean density on a sample of rows
    (numpy float32 gate pre-activations; sampling error ~ a few %)."""
    cfg = synth.CONFIGS["ffn_0p5b_bf16"]
    inp = synth.make_inputs(cfg, n_tokens=512)
    g = inp.x.float().numpy() @ inp.wg_t.float().numpy().T
    rho = float((g > 0).mean())
    assert abs(rho - cfg.rho) / cfg.rho < 0.25


def test_grid_inputs_are_exact_in_fp32():
    """The grid recipe's gate pre-activations are exact in fp32 for any
    summation order: float32 and float64 matmuls agree bit for bit."""
    inp = synth.make_grid_inputs(32, 512, 256, torch.bfloat16, rho=0.05)
    x, w = inp.as_f64("x"), inp.as_f64("wg_t")
    g64 = x @ w.T
    g32 = (inp.x.float() @ inp.wg_t.float().T).double().numpy()
    np.testing.assert_array_equal(g32, g64)
    np.testing.assert_array_equal(oracle.gate_preact(x, w), g64)


def test_gate_bias_is_exactly_additive():
    """The density sweep's harness reuses G0 = G(tau = 0): with x's last
    feature 1.0 and the bias (-tau) in W_gate's last input row, which the
    oracle adds last, G(tau) = fl(G0 - tau) holds bit for bit."""
    cfg = synth.CONFIGS["ffn_2b_bf16"].with_(n_tokens=48, d_model=96, d_ff=256)
    for rho in (0.0025, 0.05):
        inp = synth.make_inputs(cfg.with_(rho=rho))
        x, wg = inp.as_f64("x"), inp.as_f64("wg_t")
        assert np.all(x[:, -1] == 1.0) and np.all(wg[:, -1] == -inp.tau)
        wg0 = wg.copy()
        wg0[:, -1] = 0.0
        np.testing.assert_array_equal(oracle.gate_preact(x, wg),
                                      oracle.gate_preact(x, wg0) - inp.tau)
