"""Failure handling of the tcgen05 GEMM engines, on the GPU, without a fault:
the self-test library runs the engines with a 20 ms wait deadline on a tile
pipeline whose stage barriers can never complete (the copies are in bounds,
the barriers only wait for bytes that never come).  The wait runs out, the
kernel reports SGE_FLAG_TIMEOUT, drains, frees its tensor memory and
returns; the context stays usable."""
import ctypes
import time

import numpy as np
import pytest
import torch

import activation_sparse_gated_epilogue_b200 as sge
import oracle
from activation_sparse_gated_epilogue_b200 import build as sge_build
from activation_sparse_gated_epilogue_b200 import synth
from tests._util import assert_twell_equal

pytestmark = pytest.mark.gpu


def _selftest():
    st = ctypes.CDLL(sge_build.SELFTEST_LIB)
    P = ctypes.c_void_p
    st.sge_selftest_wait_timeout.argtypes = [ctypes.c_int, P, P, ctypes.c_int64, ctypes.c_int64,
                                             ctypes.c_int64, P, P, P]
    st.sge_selftest_wait_timeout.restype = ctypes.c_int
    return st


@pytest.mark.parametrize("pair", [0, 1])
def test_bounded_wait_runs_out_and_the_context_survives(cuda_device, pair):
    st = _selftest()
    m, n, k = 512, 512, 256
    a = torch.zeros(m, k, dtype=torch.bfloat16, device=cuda_device)
    b = torch.zeros(n, k, dtype=torch.bfloat16, device=cuda_device)
    diag = sge.new_diag(cuda_device)
    tiles = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    stream = ctypes.c_void_p(torch.cuda.current_stream(cuda_device).cuda_stream)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    rc = st.sge_selftest_wait_timeout(pair, ctypes.c_void_p(a.data_ptr()), ctypes.c_void_p(b.data_ptr()),
                                      m, n, k, ctypes.c_void_p(diag.data_ptr()),
                                      ctypes.c_void_p(tiles.data_ptr()), stream)
    assert rc == 0
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(diag[3]) & 1, "SGE_FLAG_TIMEOUT not set"
    assert int(tiles.item()) == 0          # no accumulator reached the epilogue
    assert elapsed < 5.0, elapsed          # bounded: a few 20 ms waits
    # the context is intact: the library's gate GEMM still gives exact results
    inp = synth.make_grid_inputs(300, 200, 640, torch.bfloat16, rho=0.05, seed=7)
    x, wg = inp.x.to(cuda_device), inp.wg_t.to(cuda_device)
    tw = sge.twell_gate_pack(x, wg, 128, 128)
    ora = oracle.twell_pack(oracle.gate_preact(inp.as_f64("x"), inp.as_f64("wg_t")), 128, 128,
                            oracle.VAL_BF16)
    torch.cuda.synchronize()
    assert_twell_equal(tw, ora)
