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


@pytest.mark.parametrize("schedule", ["persistent", "split"])
def test_missing_signal_in_backward_times_out_and_context_survives(schedule):
    """The same for the backward: CTA 0 of the down dgrad never gets its first
    accumulator.  Under the persistent schedule the gate/up dgrad's and the gate/up
    weight gradient's waits for that tile's rows run out as well, and every CTA
    still reaches the pass's grid barriers; the launch ends with MOK_STATUS_TIMEOUT
    and the next backward on the same context is correct."""
    wl = synth.WORKLOADS["tiny"]
    case = make_case(wl, device="cuda", gen_device="cpu")
    layer = MoELayer(cfg_for(wl), case["params"], training=True, device=torch.device("cuda"))
    sched = abi.MOK_SCHEDULE_PERSISTENT if schedule == "persistent" else abi.MOK_SCHEDULE_SPLIT
    abi.moe_set_schedule(sched)
    try:
        layer.forward(case["x"])
        layer.backward(case["x"], case["dy"])
        torch.cuda.synchronize()
        assert layer.status() == 0
        abi.moe_test_drop_signal(True)
        try:
            t0 = time.perf_counter()
            layer.backward(case["x"], case["dy"])
            torch.cuda.synchronize()
            dt = time.perf_counter() - t0
        finally:
            abi.moe_test_drop_signal(False)
        assert layer.status() == abi.MOK_STATUS_TIMEOUT
        assert 1.0 < dt < 60.0, dt
        assert layer.status() == 0
        grads = layer.backward(case["x"], case["dy"])
        torch.cuda.synchronize()
        assert layer.status() == 0
    finally:
        abi.moe_set_schedule(abi.MOK_SCHEDULE_PERSISTENT)
    dx, _, _ = case["L"].bwd(case["idx"], case["w"])
    assert_close(to_np(grads["dx"]), dx, "dx after the timeout")
