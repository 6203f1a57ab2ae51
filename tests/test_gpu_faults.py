"""Failure detection without a GPU fault: a signal that never comes.

With the fault-injection hook on, CTA 0 of the gate/up GEMM (and of the down
GEMM) skips the signal that hands its first accumulator to the epilogue.  The
epilogue's bounded wait must run out (about 2 s), record MOK_STATUS_TIMEOUT in
the device status word and let the kernel return; the context stays usable and
the next forward is correct.  The tiny workload gives every CTA a single tile, so nothing of CTA 0
is still in flight when its wait runs out.
"""
import time

import numpy as np
import pytest
import torch

from mixture_experts_layer_persistent_b200 import MoELayer, abi, cfg_for, synth
from tests._support import assert_close, make_case, to_np

pytestmark = pytest.mark.gpu


def test_missing_signal_times_out_and_context_survives():
    wl = synth.WORKLOADS["tiny"]
    case = make_case(wl, device="cuda", gen_device="cpu")
    layer = MoELayer(cfg_for(wl), case["params"], training=False, device=torch.device("cuda"))
    layer.forward(case["x"])
    torch.cuda.synchronize()
    assert layer.status() == 0
    abi.moe_test_drop_signal(True)
    try:
        t0 = time.perf_counter()
        layer.forward(case["x"])
        torch.cuda.synchronize()
        dt = time.perf_counter() - t0
    finally:
        abi.moe_test_drop_signal(False)
    assert layer.status() == abi.MOK_STATUS_TIMEOUT
    assert 1.0 < dt < 60.0, dt
    assert layer.status() == 0                   # reading clears the word
    y = layer.forward(case["x"])
    torch.cuda.synchronize()
    assert layer.status() == 0
    assert_close(to_np(y), case["L"].fwd(case["idx"], case["w"]), "y after the timeout")
