"""The device-side timeout path, end to end, without faulting or hanging the GPU.

The kernels' waits are bounded: after the limit a kernel records 0x10000 | site in the
workspace status word and returns, and moe_get_device_status reports
MOE_ERR_DEVICE_TIMEOUT. moe_selftest_bounded_wait runs that same bounded wait on an
mbarrier; with nothing arriving it must give up after a short limit (1 ms here), report
the timeout with its site, leave the context usable, and a forward afterwards must still
be correct."""
import ctypes
import time

import numpy as np
import pytest
import torch

import mixture_experts_expert_topk_b200 as moe
from mixture_experts_expert_topk_b200._capi import MOE_ERR_DEVICE_TIMEOUT, MOE_ERR_INVALID_ARG, MOE_OK

from _cases import CONFIGS, GpuForward, bf16_to_f64, err_beyond_rounding, oracle_out

pytestmark = pytest.mark.gpu


def _wait(ws, limit_us, arrive):
    L = moe.lib()
    return L.moe_selftest_bounded_wait(ctypes.c_void_p(ws.data_ptr()), limit_us, arrive,
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_bounded_wait_completes_when_the_barrier_arrives():
    ws = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    assert _wait(ws, 1000, 1) == MOE_OK
    st, word = moe.device_status(ws)
    assert st == MOE_OK and word == 0


def test_bounded_wait_times_out_and_reports_site():
    ws = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    assert _wait(ws, 1000, 0) == MOE_OK          # 1 ms limit, nothing arrives
    st, word = moe.device_status(ws)             # synchronises the stream
    dt = time.perf_counter() - t0
    assert st == MOE_ERR_DEVICE_TIMEOUT, st
    assert word == 0x10000 | 0x7F, hex(word)
    assert dt < 1.0, dt                           # gave up at its limit, not at the 2 s default
    assert moe.device_status(ws) == (MOE_OK, 0)   # the query cleared the word
    # the context is still usable: a forward on the same device matches the oracle
    cfg = CONFIGS["tiny"]
    run = GpuForward(cfg)
    out = run.forward()
    ref = oracle_out(cfg, run.inp)
    assert err_beyond_rounding(bf16_to_f64(out), ref) <= 2e-2
    assert moe.device_status(run.ws)[0] == MOE_OK


def test_bounded_wait_rejects_bad_arguments():
    ws = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    assert _wait(ws, 0, 0) == MOE_ERR_INVALID_ARG
    assert _wait(ws, 2_000_000, 0) == MOE_ERR_INVALID_ARG
    assert _wait(ws[1:], 1000, 1) == MOE_ERR_INVALID_ARG
