"""The host-buffer entry points (moe_fwd_host, moe_bwd_host) against the device API.

They run the same kernels on copies of the same inputs, so y, dx and the weight
gradients must match the device-pointer calls byte for byte, both when
moe_bwd_host uploads x itself and when it reuses the x that moe_fwd_host left in
the scratch buffer (x_host = NULL).
"""
import pytest
import torch

from mixture_experts_layer_persistent_b200 import MoELayer, abi, cfg_for, synth
from tests._support import make_case

pytestmark = pytest.mark.gpu

WL = synth.Workload("host_medium", T=333, H=768, E=12, k=3, I=384, S=2, Is=384, seed=41)


@pytest.mark.parametrize("reuse_x", [False, True], ids=["upload_x", "reuse_x"])
def test_host_entry_points_match_device_api(reuse_x):
    case = make_case(WL, device="cuda", gen_device="cpu")
    dev = torch.device("cuda")
    layer = MoELayer(cfg_for(WL), case["params"], training=True, device=dev)
    y_ref = layer.forward(case["x"]).clone()
    g_ref = {k: (v.clone() if v is not None else None) for k, v in layer.backward(case["x"], case["dy"]).items()}
    torch.cuda.synchronize()

    c = layer.cfg
    hx = case["x"].cpu().pin_memory()
    hdy = case["dy"].cpu().pin_memory()
    hy = torch.empty_like(hx).pin_memory()
    hdx = torch.empty_like(hx).pin_memory()
    n = max(abi.moe_host_scratch_size(c, False), abi.moe_host_scratch_size(c, True))
    scratch = torch.empty(n, dtype=torch.uint8, device=dev)
    grads = layer.new_grads()
    g = abi.moe_grads(None, grads["dw_gate_up"].data_ptr(), grads["dw_down"].data_ptr(),
                      grads["drouter_w"].data_ptr(),
                      grads["dws_gate_up"].data_ptr() if grads["dws_gate_up"] is not None else None,
                      grads["dws_down"].data_ptr() if grads["dws_down"] is not None else None)
    st = layer.stream()
    abi.moe_fwd_host(c, hx.data_ptr(), layer.cparams, hy.data_ptr(), layer.ctx.data_ptr(), layer.ctx_bytes, 1,
                     scratch.data_ptr(), n, st)
    abi.moe_bwd_host(c, None if reuse_x else hx.data_ptr(), hdy.data_ptr(), layer.cparams, layer.ctx.data_ptr(),
                     layer.ctx_bytes, hdx.data_ptr(), g, scratch.data_ptr(), n, st)
    torch.cuda.synchronize()
    assert layer.status() == 0
    assert torch.equal(hy.view(torch.int16), y_ref.cpu().view(torch.int16))
    assert torch.equal(hdx.view(torch.int16), g_ref["dx"].cpu().view(torch.int16))
    for k in ("dw_gate_up", "dw_down", "dws_gate_up", "dws_down"):
        assert torch.equal(grads[k].view(torch.int16), g_ref[k].view(torch.int16)), k
    assert torch.equal(grads["drouter_w"].view(torch.int32), g_ref["drouter_w"].view(torch.int32))


def test_step_host_matches_device_api():
    """moe_step_host (forward + backward through host buffers, transfers overlapping
    the passes on a second stream) against the device calls, byte for byte, twice in
    a row (the second step reuses the scratch buffer the first one left)."""
    case = make_case(WL, device="cuda", gen_device="cpu")
    dev = torch.device("cuda")
    layer = MoELayer(cfg_for(WL), case["params"], training=True, device=dev)
    y_ref = layer.forward(case["x"]).clone()
    g_ref = {k: (v.clone() if v is not None else None) for k, v in layer.backward(case["x"], case["dy"]).items()}
    torch.cuda.synchronize()
    c = layer.cfg
    hx = case["x"].cpu().pin_memory()
    hdy = case["dy"].cpu().pin_memory()
    n = abi.moe_host_scratch_size(c, 2)
    scratch = torch.empty(n, dtype=torch.uint8, device=dev)
    for _ in range(2):
        hy = torch.empty_like(hx).pin_memory()
        hdx = torch.empty_like(hx).pin_memory()
        grads = layer.new_grads()
        g = abi.moe_grads(None, grads["dw_gate_up"].data_ptr(), grads["dw_down"].data_ptr(),
                          grads["drouter_w"].data_ptr(),
                          grads["dws_gate_up"].data_ptr() if grads["dws_gate_up"] is not None else None,
                          grads["dws_down"].data_ptr() if grads["dws_down"] is not None else None)
        abi.moe_step_host(c, hx.data_ptr(), hdy.data_ptr(), layer.cparams, hy.data_ptr(), hdx.data_ptr(),
                          layer.ctx.data_ptr(), layer.ctx_bytes, g, scratch.data_ptr(), n, layer.stream())
        assert layer.status() == 0
        assert torch.equal(hy.view(torch.int16), y_ref.cpu().view(torch.int16))
        assert torch.equal(hdx.view(torch.int16), g_ref["dx"].cpu().view(torch.int16))
        for k in ("dw_gate_up", "dw_down", "dws_gate_up", "dws_down"):
            assert torch.equal(grads[k].view(torch.int16), g_ref[k].view(torch.int16)), k
        assert torch.equal(grads["drouter_w"].view(torch.int32), g_ref["drouter_w"].view(torch.int32))


def test_step_host_async_pipeline_matches_device_api():
    """moe_step_host_async over three steps with different inputs (each call prefetching
    the next step's x; y and dx of a step leaving while the next one runs): every
    step's y and dx, and the last step's weight and router gradients, equal those of
    the device calls byte for byte.  A second sequence on the same scratch, without
    prefetch, gives the same bytes again."""
    case = make_case(WL, device="cuda", gen_device="cpu")
    dev = torch.device("cuda")
    layer = MoELayer(cfg_for(WL), case["params"], training=True, device=dev)
    xs = [torch.roll(case["x"], 7 * i, 0).contiguous() for i in range(3)]
    dys = [torch.roll(case["dy"], 5 * i, 0).contiguous() for i in range(3)]
    refs = []
    for x, dy in zip(xs, dys):
        y = layer.forward(x).clone()
        g = {k: (v.clone() if v is not None else None) for k, v in layer.backward(x, dy).items()}
        refs.append((y, g))
    torch.cuda.synchronize()
    c = layer.cfg
    hxs = [x.cpu().pin_memory() for x in xs]
    hdys = [dy.cpu().pin_memory() for dy in dys]
    n = abi.moe_host_scratch_size(c, 3)
    scratch = torch.empty(n, dtype=torch.uint8, device=dev)
    grads = layer.new_grads()
    g = abi.moe_grads(None, grads["dw_gate_up"].data_ptr(), grads["dw_down"].data_ptr(),
                      grads["drouter_w"].data_ptr(),
                      grads["dws_gate_up"].data_ptr() if grads["dws_gate_up"] is not None else None,
                      grads["dws_down"].data_ptr() if grads["dws_down"] is not None else None)
    for prefetch in (True, False):
        hys = [torch.empty_like(hxs[0]).pin_memory() for _ in range(3)]
        hdxs = [torch.empty_like(hxs[0]).pin_memory() for _ in range(3)]
        for i in range(3):
            nxt = hxs[i + 1].data_ptr() if prefetch and i + 1 < 3 else None
            abi.moe_step_host_async(c, hxs[i].data_ptr(), nxt, hdys[i].data_ptr(), layer.cparams, hys[i].data_ptr(),
                                    hdxs[i].data_ptr(), layer.ctx.data_ptr(), layer.ctx_bytes, g, scratch.data_ptr(),
                                    n, layer.stream())
        abi.moe_step_host_sync(layer.stream())
        assert layer.status() == 0
        for i, (y_ref, g_ref) in enumerate(refs):
            assert torch.equal(hys[i].view(torch.int16), y_ref.cpu().view(torch.int16)), (prefetch, i)
            assert torch.equal(hdxs[i].view(torch.int16), g_ref["dx"].cpu().view(torch.int16)), (prefetch, i)
        g_last = refs[-1][1]
        for k in ("dw_gate_up", "dw_down", "dws_gate_up", "dws_down"):
            assert torch.equal(grads[k].view(torch.int16), g_last[k].view(torch.int16)), (prefetch, k)
        assert torch.equal(grads["drouter_w"].view(torch.int32), g_last["drouter_w"].view(torch.int32))


def test_step_host_async_mxfp8_matches_device_api():
    """The pipelined host steps drive the MXFP8 training step too (MXFP8 forward and data
    gradients, BF16 weight gradients): two steps with different inputs, each step's y and
    dx and the last step's gradients byte for byte against the device calls."""
    from tests.test_gpu_layer import MX_BWD_CASES, _mx_train_params
    wl = MX_BWD_CASES[0]
    case = make_case(wl, device="cuda", gen_device="cpu", mx=True)
    dev = torch.device("cuda")
    layer = MoELayer(cfg_for(wl), _mx_train_params(case["params"]), training=True, device=dev)
    xs = [case["x"], torch.roll(case["x"], 11, 0).contiguous()]
    dys = [case["dy"], torch.roll(case["dy"], 3, 0).contiguous()]
    refs = []
    for x, dy in zip(xs, dys):
        y = layer.forward(x).clone()
        g = {k: (v.clone() if v is not None else None) for k, v in layer.backward(x, dy).items()}
        refs.append((y, g))
    torch.cuda.synchronize()
    c = layer.cfg
    hxs = [x.cpu().pin_memory() for x in xs]
    hdys = [dy.cpu().pin_memory() for dy in dys]
    hys = [torch.empty_like(hxs[0]).pin_memory() for _ in range(2)]
    hdxs = [torch.empty_like(hxs[0]).pin_memory() for _ in range(2)]
    n = abi.moe_host_scratch_size(c, 3)
    scratch = torch.empty(n, dtype=torch.uint8, device=dev)
    grads = layer.new_grads()
    g = abi.moe_grads(None, grads["dw_gate_up"].data_ptr(), grads["dw_down"].data_ptr(),
                      grads["drouter_w"].data_ptr(),
                      grads["dws_gate_up"].data_ptr() if grads["dws_gate_up"] is not None else None,
                      grads["dws_down"].data_ptr() if grads["dws_down"] is not None else None)
    for i in range(2):
        nxt = hxs[1].data_ptr() if i == 0 else None
        abi.moe_step_host_async(c, hxs[i].data_ptr(), nxt, hdys[i].data_ptr(), layer.cparams, hys[i].data_ptr(),
                                hdxs[i].data_ptr(), layer.ctx.data_ptr(), layer.ctx_bytes, g, scratch.data_ptr(), n,
                                layer.stream())
    abi.moe_step_host_sync(layer.stream())
    assert layer.status() == 0
    for i, (y_ref, g_ref) in enumerate(refs):
        assert torch.equal(hys[i].view(torch.int16), y_ref.cpu().view(torch.int16)), i
        assert torch.equal(hdxs[i].view(torch.int16), g_ref["dx"].cpu().view(torch.int16)), i
    for k in ("dw_gate_up", "dw_down", "dws_gate_up", "dws_down"):
        if refs[-1][1][k] is not None:
            assert torch.equal(grads[k].view(torch.int16), refs[-1][1][k].view(torch.int16)), k
    assert torch.equal(grads["drouter_w"].view(torch.int32), refs[-1][1]["drouter_w"].view(torch.int32))
