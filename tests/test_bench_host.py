"""Host-side pieces of bench.py that need no GPU: the reference arm (the
oracle timed on the host cores) keeps the bench's JSON contract, and the
token-count override reaches the workload configuration."""
import argparse
import json

import bench


def _args(**kw):
    base = dict(gpus=1, steps=1, warmup=0, workload="decode_1b_bf16", impl="reference", tokens=2,
                no_cpu=False, sweep=False, cap_sweep=False, profile=False, profile_hybrid=False)
    base.update(kw)
    return argparse.Namespace(**base)


def test_tokens_override():
    assert bench.workload_config(_args(tokens=7)).n_tokens == 7
    assert bench.workload_config(_args(tokens=0)).n_tokens == 64
    assert bench.workload_config(_args(workload="ffn_1b_bf16", tokens=0)).n_tokens == 8192


def test_reference_arm_json_contract():
    out = bench.run_reference(_args())
    json.dumps(out)
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "dtype", "config", "cpu_baseline", "e2e"):
        assert key in out, key
    assert out["impl"] == "reference" and out["metric"] == bench.METRIC
    assert out["value"] > 0 and out["unit"] == "tokens/s" and out["steps"] == 1
    assert out["config"]["workload"].startswith("decode_1b_bf16: N=2 ")
    assert out["cpu_baseline"]["kind"] == "oracle" and out["cpu_baseline"]["cores"] >= 1
    assert out["e2e"]["h2d_bytes_per_step"] == 0 and out["e2e"]["d2h_bytes_per_step"] == 0
    assert out["e2e"]["value"] == out["value"]


def test_reference_arm_fp32_workload():
    out = bench.run_reference(_args(workload="tiny_fp32", tokens=4))
    assert out["value"] > 0 and out["config"]["workload"].startswith("tiny_fp32: N=4 ")


def test_own_arm_refuses_fp32_workloads_before_touching_a_gpu():
    import pytest
    with pytest.raises(SystemExit, match="parity case"):
        bench.run_own(_args(workload="tiny_fp32", impl="own", tokens=0), 0, 1, 0)


def test_twell_bytes_counts_sectors_per_tile():
    """Counts 0, 1, 32, 33 and 200 (> C = 128, so 128 stored) in bf16:
    0 + 2 + 3 + 5 + 12 sectors of 32 B over the index and value runs."""
    import torch
    count = torch.tensor([[0, 1, 32, 33, 200]], dtype=torch.uint8)
    got = bench.twell_bytes(count, 128, 2)
    assert got["allocated"] == 5 * (1 + 3 * 128)
    assert got["algorithmic"] == 5 + 3 * (0 + 1 + 32 + 33 + 128)
    assert got["sector_granular"] == 5 + 32 * (0 + 2 + 3 + 5 + 12)
    assert bench.twell_bytes(count, 48, 2)["sector_granular"] is None


def test_routed_k_rule():
    assert bench.routed_k(8192) == 16 and bench.routed_k(10240) == 20 and bench.routed_k(1024) == 8


def test_routed_split_counts_heavy_tokens_in_order():
    """Stored entries per token 3, 40, 0, 17, 200 (capped at C = 128 per
    tile) with K = 16, S_max = 2: tokens 1 and 3 take the spill, token 4
    (heavy, past S_max) stays with the per-entry path."""
    import torch
    count = torch.tensor([[3, 0], [20, 20], [0, 0], [17, 0], [100, 100]], dtype=torch.uint8)
    n_spill, nnz_light, nnz = bench.routed_split(count, 128, 16, 2)
    assert (n_spill, nnz_light, nnz) == (2, 3 + 200, 3 + 40 + 17 + 200)
    # C = 10 stores 3, 20, 0, 10, 20 entries: tokens 1 and 4 are heavy
    assert bench.routed_split(count, 10, 16, 8) == (2, 3 + 10, 3 + 20 + 10 + 20)
