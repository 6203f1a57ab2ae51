"""moe_fwd_static: the forward pass for callers that cannot allocate device memory.

Some callers cannot hand the layer a workspace: runtimes that plan all device
memory up front and forbid allocation while running, or plug-in hosts that give
a layer nothing but its inputs and outputs.  moe_fwd_static serves them by
keeping its intermediate buffers in a fixed-size array the library owns.  This
test calls it through the C ABI twice in a row and checks each result against
moe_fwd with a caller-provided workspace.  Both run the same kernels on the
same inputs over identically laid-out buffers, so the outputs must agree byte
for byte (a stale or aliased byte of the shared array would show); the layer's
tolerance is checked too.  It covers the BF16 and the MXFP8 forward, and that a
shape too large for the static array is refused with a clear message.  The
file is named to be collected last.
"""
import pytest
import torch

from mixture_experts_layer_persistent_b200 import MoELayer, abi, cfg_for, quantize_mxfp8_weights, synth
from tests._support import assert_close, to_np

pytestmark = pytest.mark.gpu

SHAPES = [synth.WORKLOADS["tiny"],
          synth.Workload("static_medium", T=333, H=768, E=12, k=3, I=384, S=2, Is=384, score_fn=1,
                         n_group=4, topk_group=2, seed=31),
          synth.Workload("static_medium_mx", T=300, H=512, E=16, k=4, I=256, S=1, Is=256, score_fn=1,
                         n_group=4, topk_group=2, mxfp8=True, backward=False, seed=32)]


def _params(wl, dev):
    params = synth.draw_params(wl, "cpu")
    params = {k: (v.to(dev) if v is not None else None) for k, v in params.items()}
    if not wl.mxfp8:
        return params
    out = {k: params[k] for k in ("router_w", "e_bias", "logit_bias")}
    for name, sname in (("w_gate_up", "s_gate_up"), ("w_down", "s_down"), ("ws_gate_up", "ss_gate_up"),
                        ("ws_down", "ss_down")):
        out[name], out[sname] = quantize_mxfp8_weights(params[name]) if params.get(name) is not None else (None, None)
    return out


@pytest.mark.parametrize("wl", SHAPES, ids=lambda w: w.name)
def test_static_forward_matches_workspace_forward(wl):
    dev = torch.device("cuda")
    params = _params(wl, dev)
    x = synth.draw_x(wl, "cpu").to(dev)
    layer = MoELayer(cfg_for(wl), params, training=False, device=dev)
    _, fwd_bytes, _ = abi.moe_workspace_size(layer.cfg)
    assert fwd_bytes <= abi.MOK_STATIC_SCRATCH_BYTES
    y_ref = layer.forward(x)
    stream = layer.stream()
    for _ in range(2):                      # two calls in a row share the static array
        y = torch.full_like(x, float("nan"))
        abi.moe_fwd_static(layer.cfg, x.data_ptr(), layer.cparams, y.data_ptr(), stream)
        torch.cuda.synchronize()
        assert abi.moe_status(stream) == 0
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), f"{wl.name}: static forward differs"
        assert_close(to_np(y), to_np(y_ref), f"{wl.name} static forward")


def test_static_forward_refuses_oversized_shapes():
    wl = synth.WORKLOADS["dsv3"]
    dev = torch.device("cuda")
    cfg = cfg_for(wl)
    _, fwd_bytes, _ = abi.moe_workspace_size(cfg)
    assert fwd_bytes > abi.MOK_STATIC_SCRATCH_BYTES
    w = torch.zeros(16, dtype=torch.bfloat16, device=dev)        # never read: the size check comes first
    p = abi.moe_params(w.data_ptr(), None, None, w.data_ptr(), w.data_ptr(), None, None,
                       w.data_ptr(), w.data_ptr(), None, None)
    with pytest.raises(abi.MokError) as ei:
        abi.moe_fwd_static(cfg, w.data_ptr(), p, w.data_ptr(), None)
    assert ei.value.code == abi.MOK_ERR_WORKSPACE
    assert "static scratch" in str(ei.value)
