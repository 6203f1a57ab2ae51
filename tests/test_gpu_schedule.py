"""The persistent (one-launch) forward against the split (one launch per step) forward.

The split schedule also runs with programmatic dependent launch (PDL); the
backward after a persistent forward uses PDL, after a split forward it does not.

Both schedules run the same device code with the same fixed reduction orders,
so every output and every saved tensor must agree byte for byte: y, the routing
record, the saved h / g,u / w*h (or the MXFP8 h codes and scales), and the
gradients of a backward that reads either forward's state.  The persistent
forward is one kernel launch with nothing else enqueued before it; reruns are
bit-identical (the grid barriers' launch epoch must not let a stale tag
through), and the device phase stamps come out in order.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_persistent_b200 import (MoELayer, abi, cfg_for, quantize_mxfp8_weights,
                                                   quantize_mxfp8_weights_t, synth)
from tests._support import assert_close, make_case, to_np

pytestmark = pytest.mark.gpu

CASES = [
    synth.WORKLOADS["tiny"],
    synth.Workload("sched_sigmoid", T=700, H=512, E=16, k=4, I=256, S=1, Is=256, score_fn=1, n_group=4,
                   topk_group=2, seed=41),
    synth.Workload("sched_softmax_i384", T=333, H=768, E=12, k=3, I=384, S=2, Is=384, seed=42),
    synth.Workload("sched_zipf", T=900, H=512, E=16, k=4, I=256, S=1, Is=256, score_fn=1, n_group=4, topk_group=2,
                   zipf=3.5, seed=43),
    # ten dispatch chunks of 256 tokens (the last one ragged), one token per expert or none
    synth.Workload("sched_chunks", T=2500, H=256, E=64, k=2, I=128, score_fn=0, seed=44),
]
MX_CASES = [
    synth.Workload("sched_mx", T=700, H=512, E=16, k=4, I=256, S=1, Is=256, score_fn=1, n_group=4, topk_group=2,
                   mxfp8=True, backward=False, seed=45),
    synth.Workload("sched_mx_i384", T=411, H=768, E=12, k=3, I=384, S=2, Is=384, score_fn=1, n_group=4,
                   topk_group=2, mxfp8=True, backward=False, seed=46),
    # the MXFP8 training step: the persistent backward is one launch here too
    synth.Workload("sched_mx_train", T=700, H=512, E=16, k=4, I=256, S=1, Is=256, score_fn=0, mxfp8=True,
                   seed=47),
]


def _params(wl, dev):
    params = synth.draw_params(wl, "cpu")
    params = {k: (v.to(dev) if v is not None else None) for k, v in params.items()}
    if not wl.mxfp8:
        return params
    out = {k: params[k] for k in ("router_w", "e_bias", "logit_bias")}
    for name, sname in (("w_gate_up", "s_gate_up"), ("w_down", "s_down"), ("ws_gate_up", "ss_gate_up"),
                        ("ws_down", "ss_down")):
        out[name], out[sname] = quantize_mxfp8_weights(params[name]) if params.get(name) is not None else (None, None)
        if wl.backward:
            t = "wt" + name[1:] if name.startswith("w_") else "wst" + name[2:]
            ts = "st" + name[1:] if name.startswith("w_") else "sst" + name[2:]
            out[t], out[ts] = quantize_mxfp8_weights_t(params[name]) if params.get(name) is not None else (None, None)
    return out


def _same(a, b):
    return torch.equal(a.contiguous().view(torch.uint8), b.contiguous().view(torch.uint8))


def _forward(layer, x, schedule):
    abi.moe_set_schedule(schedule)
    try:
        routing = layer.new_routing()
        y = layer.forward(x, routing=routing)
        n = abi.moe_launch_count()
        torch.cuda.synchronize()
    finally:
        abi.moe_set_schedule(abi.MOK_SCHEDULE_PERSISTENT)
    assert layer.status() == 0
    return y, routing, n


def _saved(layer, mx):
    names = ([abi.MOK_SAVED_HQ, abi.MOK_SAVED_HS] if mx else [abi.MOK_SAVED_H]) + [abi.MOK_SAVED_ROW_TOKEN,
                                                                                    abi.MOK_SAVED_ROW_W]
    if layer.training:
        names += [abi.MOK_SAVED_GU, abi.MOK_SAVED_HW] + ([abi.MOK_SAVED_H] if mx else [])
    return {n: layer.saved(n).clone() for n in names}


@pytest.mark.parametrize("wl", CASES + MX_CASES, ids=lambda w: w.name)
def test_persistent_forward_equals_split_forward(wl):
    dev = torch.device("cuda")
    params = _params(wl, dev)
    x = synth.draw_x(wl, "cpu").to(dev)
    training = wl.backward
    layer = MoELayer(cfg_for(wl), params, training=training, device=dev)
    y_s, r_s, n_s = _forward(layer, x, abi.MOK_SCHEDULE_SPLIT)
    saved_s = _saved(layer, wl.mxfp8)
    g_s = None
    if training:
        dy = synth.draw_dy(wl, "cpu").to(dev)
        abi.moe_set_schedule(abi.MOK_SCHEDULE_SPLIT)          # plain launches, no PDL
        try:
            g_s = {k: v.clone() for k, v in layer.backward(x, dy).items() if v is not None}
            torch.cuda.synchronize()
        finally:
            abi.moe_set_schedule(abi.MOK_SCHEDULE_PERSISTENT)
    # the split launches with programmatic dependent launch: the same bytes
    y_d, r_d, n_d = _forward(layer, x, abi.MOK_SCHEDULE_SPLIT_PDL)
    assert n_d == n_s
    assert _same(y_d, y_s), "y differs between the split and the PDL-split schedules"
    for k in r_s:
        assert _same(r_d[k], r_s[k]), k
    y_p, r_p, n_p = _forward(layer, x, abi.MOK_SCHEDULE_PERSISTENT)
    assert n_p == 1, n_p
    assert n_s >= 9, n_s
    assert _same(y_p, y_s), "y differs between the schedules"
    for k in r_s:
        assert _same(r_p[k], r_s[k]), k
    for k, v in _saved(layer, wl.mxfp8).items():
        assert _same(v, saved_s[k]), f"saved tensor {k} differs"
    if training:
        g_p = layer.backward(x, dy)        # persistent schedule: one launch
        assert abi.moe_launch_count() == 1
        torch.cuda.synchronize()
        assert layer.status() == 0
        for k, v in g_s.items():
            assert _same(g_p[k], v), f"gradient {k} differs (persistent backward)"
        abi.moe_set_schedule(abi.MOK_SCHEDULE_SPLIT_PDL)
        try:
            g_d = layer.backward(x, dy)    # split launches with PDL
            torch.cuda.synchronize()
        finally:
            abi.moe_set_schedule(abi.MOK_SCHEDULE_PERSISTENT)
        for k, v in g_s.items():
            assert _same(g_d[k], v), f"gradient {k} differs (PDL split backward)"
    # reruns of the persistent forward: byte-identical (a fresh launch epoch each time)
    for _ in range(3):
        y2, _, _ = _forward(layer, x, abi.MOK_SCHEDULE_PERSISTENT)
        assert _same(y2, y_s)


def test_persistent_forward_matches_oracle_on_many_chunks():
    """The chunked dispatch (every CTA scans the chunk histograms itself) against
    the oracle's routing and forward, with 3 dispatch chunks."""
    wl = CASES[-1]
    case = make_case(wl, device="cuda", gen_device="cpu")
    layer = MoELayer(cfg_for(wl), case["params"], training=False, device=torch.device("cuda"))
    y, routing, n = _forward(layer, case["x"], abi.MOK_SCHEDULE_PERSISTENT)
    assert n == 1
    L, idx = case["L"], case["idx"]
    assert np.array_equal(routing["topk_idx"].cpu().numpy(), idx)
    counts, offsets, perm, inv = L.dispatch(idx)
    assert np.array_equal(routing["counts"].cpu().numpy(), counts)
    assert np.array_equal(routing["offsets"].cpu().numpy(), offsets)
    assert np.array_equal(routing["perm"].cpu().numpy(), perm)
    assert np.array_equal(routing["inv_perm"].cpu().numpy(), inv)
    assert_close(to_np(y), L.fwd(idx, case["w"]), "y")


def test_device_phase_stamps():
    wl = CASES[1]
    dev = torch.device("cuda")
    layer = MoELayer(cfg_for(wl), _params(wl, dev), training=True, device=dev)
    x = synth.draw_x(wl, "cpu").to(dev)
    dy = synth.draw_dy(wl, "cpu").to(dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    buf = torch.zeros(abi.MOK_TRACE_POINTS * sms, dtype=torch.int64, device=dev)
    bbuf = torch.zeros_like(buf)
    abi.moe_trace_device(buf.data_ptr(), buf.numel() * 8, bbuf.data_ptr(), bbuf.numel() * 8)
    try:
        layer.forward(x)
        layer.backward(x, dy)
        torch.cuda.synchronize()
    finally:
        abi.moe_trace_device(None, 0)
    for b in (buf, bbuf):
        t = b.view(abi.MOK_TRACE_POINTS, sms).cpu().numpy()
        assert (t > 0).all()
        assert (np.diff(t, axis=0) >= 0).all()           # every CTA passes the points in order
        # the phases behind the first grid barrier end after every CTA finished the first phase
        assert (t[2:].min(axis=1) >= t[1].max()).all()
    assert buf.view(abi.MOK_TRACE_POINTS, sms).max() <= bbuf.view(abi.MOK_TRACE_POINTS, sms).min()


@pytest.mark.parametrize("wl", [CASES[1], MX_CASES[2]], ids=lambda w: w.name)
def test_persistent_passes_on_buffers_of_ones(wl):
    """The persistent forward and backward on ctx and scratch buffers filled with 0xFF
    bytes before their first use (leftover memory of an int array of -1s): the grid
    barriers must not read those words as arrivals, so every output equals the one
    on zeroed buffers byte for byte, with no status bit set."""
    dev = torch.device("cuda")
    params = _params(wl, dev)
    x = synth.draw_x(wl, dev)
    dy = synth.draw_dy(wl, dev) if wl.backward else None
    res = []
    for fill in (0x00, 0xFF):
        layer = MoELayer(cfg_for(wl), params, training=wl.backward, device=dev)
        for t in (layer.ctx, layer.scratch, layer.bwd_scratch):
            t.fill_(fill)
        y = layer.forward(x).clone()
        g = layer.backward(x, dy) if wl.backward else {}
        torch.cuda.synchronize()
        assert layer.status() == 0, f"fill {fill:#x}"
        res.append((y, g))
    assert _same(res[0][0], res[1][0]), "y"
    for k, v in res[0][1].items():
        if v is not None:
            assert _same(v, res[1][1][k]), k
