"""Seeded synthetic inputs for the activation-sparse gated FFN.

This module only draws random numbers and calibrates the gate bias; it holds
none of the FFN's arithmetic, so both the CUDA path and the fp64 oracle can be
fed from it.

Recipe (the pages print no workload, so this stands in for the FFN blocks of
the 0.5B-2B models of "Sparser, Faster, Lighter Transformer Language Models",
section "04 ... tokens" of the pwwt.cn summary):

* ``numpy.random.default_rng(seed)``, draws in the fixed order
  x -> s -> W_gate -> W_up -> W_down -> dy, all float32 normals.
* x ~ N(0, 1), shape N x d.  Each row's first d-1 features are multiplied by
  s ~ LogNormal(0, sigma); the last feature is set to 1.0, so that the last
  input row of W_gate acts as the gate bias and the per-token scale makes the
  per-token nonzero count uneven (the pages' per-token activity plots).
* W_gate and W_up ~ N(0, 1/d), W_down ~ N(0, 1/F).  Weights are stored
  neuron-major: ``wg_t`` and ``wu_t`` are F x d (row j = column j of W_gate /
  W_up), ``wd`` is F x d (row j = row j of W_down).
* The bias column of ``wg_t`` is -tau, with tau solved so that the mean gate
  density E_s[P(g > 0)] is rho (Gauss-Hermite quadrature over log s), then
  rounded to the weight dtype.
* dy ~ N(0, 1), N x d (training configs only).
* Everything is cast once to the config dtype (round to nearest even); the
  oracle reads the cast values upcast exactly to float64.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

__all__ = [
    "Config", "CONFIGS", "Inputs", "solve_tau_density", "solve_tau_spill",
    "make_inputs", "make_grid_inputs", "realised_density",
]


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    n_tokens: int
    d_model: int
    d_ff: int
    dtype: str            # "f32" or "bf16"
    tile: int             # TwELL tile width T
    cap: int              # TwELL per-tile capacity C
    sigma: float          # per-token LogNormal(0, sigma) scale
    rho: Optional[float] = None        # target mean density (solved tau)
    tau: Optional[float] = None        # given tau (overrides rho)
    ell_cap: Optional[int] = None      # hybrid ELL capacity K
    spill_frac: Optional[float] = None  # target fraction of rows with nnz > K
    s_max: Optional[int] = None        # hybrid spill capacity (rows)
    seed: int = 0

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


# The five workloads: tiny fp32 inference, 0.5B / 1B / 2B-shaped bf16
# inference, and a 1B-shaped bf16 training step on the hybrid format.
CONFIGS = {
    "tiny_fp32": Config("tiny_fp32", 256, 256, 1024, "f32", 64, 16, 0.5, tau=2.326),
    "ffn_0p5b_bf16": Config("ffn_0p5b_bf16", 4096, 1024, 4096, "bf16", 128, 128, 0.5, rho=0.02),
    "ffn_1b_bf16": Config("ffn_1b_bf16", 8192, 2048, 8192, "bf16", 128, 128, 0.7, rho=0.01),
    "ffn_2b_bf16": Config("ffn_2b_bf16", 16384, 2560, 10240, "bf16", 128, 128, 0.5, rho=0.01),
    # decode-shaped: a small batch of tokens against the 1B FFN's weights
    "decode_1b_bf16": Config("decode_1b_bf16", 64, 2048, 8192, "bf16", 128, 128, 0.7, rho=0.01),
    "train_1b_hybrid": Config("train_1b_hybrid", 8192, 2048, 8192, "bf16", 128, 128, 1.0,
                              ell_cap=128, spill_frac=0.02, s_max=1024),
}
SWEEP_2B_RHO = (0.0025, 0.005, 0.01, 0.02, 0.05)


def _phi_upper(z: float) -> float:
    """P(Z > z) for a standard normal Z."""
    return 0.5 * math.erfc(z / math.sqrt(2.0))


def _hermite(n: int = 64):
    x, w = np.polynomial.hermite.hermgauss(n)
    return x, w / math.sqrt(math.pi)


def _expect_over_scale(fn, sigma: float) -> float:
    x, w = _hermite()
    return float(sum(wi * fn(math.exp(math.sqrt(2.0) * sigma * xi)) for xi, wi in zip(x, w)))


def _density_given_tau(tau: float, sigma: float, d: int) -> float:
    c = math.sqrt((d - 1) / d)
    return _expect_over_scale(lambda s: _phi_upper(tau / (s * c)), sigma)


def _bisect(f, lo: float, hi: float, target: float, decreasing: bool = True) -> float:
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        v = f(mid)
        if (v > target) == decreasing:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def solve_tau_density(rho: float, sigma: float, d: int) -> float:
    """tau such that the expected fraction of positive gates is rho."""
    return _bisect(lambda t: _density_given_tau(t, sigma, d), 0.0, 100.0, rho)


def solve_tau_spill(frac: float, sigma: float, d: int, d_ff: int, k: int) -> float:
    """tau such that the expected fraction of tokens with more than k active
    gates (out of d_ff) is ``frac``; per token the count is taken as
    Binomial(d_ff, P(g > 0 | s))."""
    from scipy.stats import binom
    c = math.sqrt((d - 1) / d)

    def spill(tau):
        return _expect_over_scale(lambda s: float(binom.sf(k, d_ff, _phi_upper(tau / (s * c)))), sigma)
    return _bisect(spill, 0.0, 200.0, frac)


def round_to(value: float, dtype: torch.dtype) -> float:
    return float(torch.tensor(value, dtype=torch.float64).to(dtype).to(torch.float64))


@dataclasses.dataclass
class Inputs:
    """Host tensors in the config dtype (contiguous, row-major)."""
    cfg: Config
    x: torch.Tensor        # N x d
    wg_t: torch.Tensor     # F x d
    wu_t: torch.Tensor     # F x d
    wd: torch.Tensor       # F x d
    dy: Optional[torch.Tensor]  # N x d or None
    tau: float             # the bias actually stored (rounded to the dtype)
    scale: np.ndarray      # per-token s, float64

    def as_f64(self, name: str) -> np.ndarray:
        """Exact float64 upcast of one tensor, for the oracle."""
        return getattr(self, name).to(torch.float64).numpy()


def config_tau(cfg: Config) -> float:
    if cfg.tau is not None:
        return cfg.tau
    if cfg.rho is not None:
        return solve_tau_density(cfg.rho, cfg.sigma, cfg.d_model)
    if cfg.spill_frac is not None:
        return solve_tau_spill(cfg.spill_frac, cfg.sigma, cfg.d_model, cfg.d_ff, cfg.ell_cap)
    raise ValueError("config names neither tau, rho nor spill_frac")


def make_inputs(cfg: Config, n_tokens: Optional[int] = None, with_dy: Optional[bool] = None,
                tau: Optional[float] = None) -> Inputs:
    """Draw the seeded inputs of ``cfg``.  ``n_tokens`` overrides N (the first
    rows of a larger draw are NOT the same as a smaller draw; each N is its own
    seeded workload)."""
    n = cfg.n_tokens if n_tokens is None else n_tokens
    d, f = cfg.d_model, cfg.d_ff
    if with_dy is None:
        with_dy = cfg.ell_cap is not None
    dt = cfg.torch_dtype
    t = config_tau(cfg) if tau is None else tau
    t = round_to(t, dt)
    rng = np.random.default_rng(cfg.seed)
    x = rng.standard_normal((n, d), dtype=np.float32)
    s = rng.lognormal(0.0, cfg.sigma, size=n)
    x[:, : d - 1] *= s[:, None].astype(np.float32)
    x[:, d - 1] = 1.0
    wg = rng.standard_normal((f, d), dtype=np.float32) * np.float32(1.0 / math.sqrt(d))
    wu = rng.standard_normal((f, d), dtype=np.float32) * np.float32(1.0 / math.sqrt(d))
    wd = rng.standard_normal((f, d), dtype=np.float32) * np.float32(1.0 / math.sqrt(f))
    wg[:, d - 1] = -t
    dy = rng.standard_normal((n, d), dtype=np.float32) if with_dy else None
    cast = lambda a: torch.from_numpy(a).to(dt).contiguous()
    return Inputs(cfg, cast(x), cast(wg), cast(wu), cast(wd),
                  cast(dy) if dy is not None else None, t, s)


def make_grid_inputs(n: int, d: int, f: int, dtype: torch.dtype = torch.bfloat16,
                     rho: float = 0.02, seed: int = 0, with_dy: bool = False) -> Inputs:
    """Inputs on a small dyadic grid: x = k/8 * s with k in [-8, 8] and
    s in {1/2, 1, 2}; W_gate = m/64 with m in [-16, 16]; the bias is a multiple
    of 1/64 that the dtype holds exactly.  Every product is an integer
    multiple of 2^-10 bounded by 2^-1, so for d <= 2^14 every fp32 partial
    sum is exact whatever the summation order: the gate
    pre-activations of the GPU and of the oracle are identical bit for bit.
    W_up and W_down are ordinary N(0, 1/fan_in) draws."""
    assert d <= 1 << 14
    rng = np.random.default_rng(seed)
    k = rng.integers(-8, 9, size=(n, d)).astype(np.float32) / 8.0
    s = 2.0 ** rng.integers(-1, 2, size=n)
    k[:, : d - 1] *= s[:, None].astype(np.float32)
    k[:, d - 1] = 1.0
    m = rng.integers(-16, 17, size=(f, d)).astype(np.float32) / 64.0
    wu = rng.standard_normal((f, d), dtype=np.float32) * np.float32(1.0 / math.sqrt(d))
    wd = rng.standard_normal((f, d), dtype=np.float32) * np.float32(1.0 / math.sqrt(f))
    # std of the unbiased gate, E over s of s^2 is (1/4 + 1 + 4)/3
    var = (d - 1) * (24.0 / 64.0) * (2.0 * 1496.0 / 33.0 / 4096.0) * (5.25 / 3.0)
    z = _bisect(lambda q: _phi_upper(q), 0.0, 10.0, rho)
    tau = round_to(round(z * math.sqrt(var) * 64.0) / 64.0, dtype)
    m[:, d - 1] = -tau
    dy = rng.standard_normal((n, d), dtype=np.float32) if with_dy else None
    cast = lambda a: torch.from_numpy(a).to(dtype).contiguous()
    cfg = Config(f"grid_{n}x{d}x{f}", n, d, f, "f32" if dtype == torch.float32 else "bf16",
                 0, 0, 0.0, tau=tau, seed=seed)
    return Inputs(cfg, cast(k), cast(m), cast(wu), cast(wd),
                  cast(dy) if dy is not None else None, tau, s)


def realised_density(count: np.ndarray, d_ff: int) -> float:
    """Mean fraction of active gates, from TwELL per-tile counts."""
    return float(count.astype(np.int64).sum()) / (count.shape[0] * d_ff)
