"""The layer runs under CUDA-graph capture: a forward + backward captured once and
replayed gives the eager results byte for byte, also after new inputs are copied
into the captured buffers.  (Capture needs one eager call first, which sets up the
library's per-device state; no call inside the layer allocates or synchronises.)
"""
import pytest
import torch

from mixture_experts_layer_persistent_b200 import MoELayer, abi, cfg_for, synth
from tests._support import make_case

pytestmark = pytest.mark.gpu

WL = synth.Workload("graph_medium", T=333, H=768, E=12, k=3, I=384, S=2, Is=384, score_fn=1, n_group=4,
                    topk_group=2, seed=61)


def _eager(layer, x, dy):
    y = layer.forward(x).clone()
    g = {k: (v.clone() if v is not None else None) for k, v in layer.backward(x, dy).items()}
    torch.cuda.synchronize()
    return y, g


def _same(a, b):
    if a.dtype == torch.float32:
        return torch.equal(a.view(torch.int32), b.view(torch.int32))
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_captured_step_replays_eager_results():
    case = make_case(WL, device="cuda", gen_device="cpu")
    layer = MoELayer(cfg_for(WL), case["params"], training=True, device=torch.device("cuda"))
    x = case["x"].clone()
    dy = case["dy"].clone()
    y_ref, g_ref = _eager(layer, x, dy)

    y = torch.empty_like(x)
    grads = layer.new_grads()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):           # one eager step on the capture stream first
        layer.forward(x, y)
        layer.backward(x, dy, grads)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph):
        layer.forward(x, y)
        layer.backward(x, dy, grads)
    for _ in range(3):
        y.zero_()
        graph.replay()
    torch.cuda.synchronize()
    assert abi.moe_status(torch.cuda.current_stream().cuda_stream) == 0
    assert _same(y, y_ref)
    for k, v in g_ref.items():
        if v is not None:
            assert _same(grads[k], v), k

    # new inputs in the captured buffers: the replay reads them
    x2 = synth.draw_x(WL, "cpu", attempt=7).to(x.device)
    dy2 = synth.draw_dy(WL, "cpu").to(x.device).mul_(0.5)
    x.copy_(x2)
    dy.copy_(dy2)
    graph.replay()
    torch.cuda.synchronize()
    y2_ref, g2_ref = _eager(layer, x2, dy2)
    assert _same(y, y2_ref)
    for k, v in g2_ref.items():
        if v is not None:
            assert _same(grads[k], v), k
