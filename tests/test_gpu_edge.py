"""Degenerate and boundary configurations on the GPU against the fp64 oracle.

One token; every expert selected (top_k = E); a single routed expert (a dense
SwiGLU MLP plus a shared expert); the largest top_k (16); sigmoid scoring without
a group limit and with a routing scale other than 1; the minimum H and I; groups
of exactly 128, 129, 256 and 257 rows (one routed and one shared expert, every
token in both: the edges of the 128-row tiles and of the 256-row pair tiles,
whose second half is then full, absent, or a single row).  Each
runs the forward and the backward; routing is bit-exact, floats within
|gpu - oracle| <= 1e-2 + 1e-2 |oracle|.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_persistent_b200 import MoELayer, cfg_for, synth
from tests._support import assert_close, make_case, to_np

pytestmark = pytest.mark.gpu

EDGE = [
    synth.Workload("one_token", T=1, H=256, E=8, k=2, I=128, seed=51),
    synth.Workload("all_experts", T=37, H=256, E=4, k=4, I=256, seed=52),
    synth.Workload("one_expert", T=50, H=512, E=1, k=1, I=128, S=1, Is=128, seed=53),
    synth.Workload("top16", T=64, H=256, E=32, k=16, I=128, score_fn=1, seed=54),
    synth.Workload("sigmoid_scaled", T=96, H=512, E=16, k=4, I=256, score_fn=1, routed_scale=2.5, seed=55),
    synth.Workload("groups_scaled", T=80, H=256, E=16, k=3, I=128, S=1, Is=128, score_fn=1, n_group=4,
                   topk_group=2, routed_scale=0.5, seed=56),
] + [synth.Workload(f"rows_{t}", T=t, H=256, E=1, k=1, I=256, S=1, Is=256, seed=57 + i)
     for i, t in enumerate((128, 129, 256, 257))]


@pytest.mark.parametrize("wl", EDGE, ids=lambda w: w.name)
def test_edge_configuration(wl):
    case = make_case(wl, device="cuda", gen_device="cpu")
    layer = MoELayer(cfg_for(wl), case["params"], training=True, device=torch.device("cuda"))
    routing = layer.new_routing()
    y = layer.forward(case["x"], routing=routing)
    grads = layer.backward(case["x"], case["dy"])
    torch.cuda.synchronize()
    assert layer.status() == 0
    L, idx, w = case["L"], case["idx"], case["w"]
    assert np.array_equal(routing["topk_idx"].cpu().numpy(), idx)
    assert_close(to_np(routing["topk_w"]), w, "topk_w", rtol=1e-5, atol=1e-6)
    assert_close(to_np(y), L.fwd(idx, w), "y")
    dx, _, _ = L.bwd(idx, w)
    assert_close(to_np(grads["dx"]), dx, "dx")
    assert_close(to_np(grads["drouter_w"]), L.drouter(idx, w, np.arange(wl.E)), "drouter_w")
    for e in range(wl.E):
        dgu, ddn = L.dw_full(idx, w, e, False)
        assert_close(to_np(grads["dw_gate_up"][e]), dgu, f"dw_gate_up[{e}]")
        assert_close(to_np(grads["dw_down"][e]), ddn, f"dw_down[{e}]")
    for s in range(wl.S):
        dgu, ddn = L.dw_full(idx, w, s, True)
        assert_close(to_np(grads["dws_gate_up"][s]), dgu, f"dws_gate_up[{s}]")
        assert_close(to_np(grads["dws_down"][s]), ddn, f"dws_down[{s}]")
