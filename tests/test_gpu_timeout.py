"""Failure detection on the device: a pipeline wait that runs out.

Every wait inside the GEMM kernels is bounded.  With the main-loop limit set
to 0 (dg_set_wait_limit_ns) an ordinary call gives up at its first wait that
is not already satisfied: it must still return, leave DG_DEVERR_TIMEOUT in
the device error word, free its resources, and leave the context usable, so
that the next call with the default limit is correct.  Nothing here faults
or traps the GPU: the kernels report and return.

Only 1-CTA tiles are exercised on the GPU (one pipeline, and split-K over two
pipelines): their exit drain waits on barriers of their own CTA.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_grouped_gemm_05_b200 import binding as dg
from moe_grouped_gemm_05_b200 import synth

from helpers import bits, check_close, packed, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dg.set_config(0)
    dg.get_device_error()
    yield
    dg.set_config(0)


@pytest.mark.parametrize("cfg", [(128, 1, 1), (64, 1, 2)])
def test_wait_that_runs_out_reports_timeout_and_next_call_is_correct(cfg):
    # 256 K blocks: the epilogue's first wait (a whole tile's K loop, tens of
    # microseconds) outlasts any suspended probe and the clock's granularity
    M, N, K = 128, 512, 32768
    p = synth.dense_problem(M, N, K, seed=4242)
    sa, sb = packed(p)
    t = to_device(p, sa, sb)
    ref = oracle.fp8_gemm_nt(p.a, sa, p.b, sb, M, N, K)
    dg.set_config(*cfg)
    prev = dg.set_wait_limit_ns(0)
    try:
        dg.fp8_gemm_nt(t["a"], t["sfa"], t["b"], t["sfb"])
        torch.cuda.synchronize()  # the call returns
    finally:
        assert dg.set_wait_limit_ns(prev) == 0
    assert dg.get_device_error() & dg.DG_DEVERR_TIMEOUT
    # the context is usable and the next calls (default limit) are correct
    for _ in range(2):
        d = dg.fp8_gemm_nt(t["a"], t["sfa"], t["b"], t["sfb"])
        torch.cuda.synchronize()
        check_close(bits(d), ref, f"after a timeout, cfg={cfg}")
        assert dg.get_device_error() == 0
