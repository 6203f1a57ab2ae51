"""GPU parity of the layer (through the C ABI) against the fp64 oracle.

Routing indices, counts, offsets and permutations must match bit-exactly;
floating-point outputs and gradients must satisfy
|gpu - oracle| <= 1e-2 + 1e-2 |oracle| elementwise; reruns must be
bit-identical.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_persistent_b200 import MoELayer, cfg_for, synth
from tests._support import assert_close, check_mx_h, make_case, rel_rms_per_token, to_np

pytestmark = pytest.mark.gpu

# reduced shapes that still span several tiles, ragged tails and every routing mode
MEDIUM_SIGMOID = synth.Workload("medium_sigmoid", T=700, H=512, E=16, k=4, I=256, S=1, Is=256,
                                score_fn=1, n_group=4, topk_group=2, seed=11)
MEDIUM_SOFTMAX = synth.Workload("medium_softmax", T=333, H=768, E=12, k=3, I=384, S=2, Is=384,
                                seed=12)
# skewed routing: groups on both sides of the 192-row split between the resident and the
# streaming weight-gradient kernels (one of exactly 192 rows), and an empty group
RESIDENT_ROWS = 192
MEDIUM_ZIPF = synth.Workload("medium_zipf", T=900, H=512, E=16, k=4, I=256, S=1, Is=256, score_fn=1,
                             n_group=4, topk_group=2, zipf=1.5, seed=142)
MEDIUM_ZIPF_SPARSE = synth.scaled(MEDIUM_ZIPF, name="medium_zipf_sparse", zipf=3.5)
CASES = [synth.WORKLOADS["tiny"], MEDIUM_SIGMOID, MEDIUM_SOFTMAX, MEDIUM_ZIPF, MEDIUM_ZIPF_SPARSE]


def _run(wl, case):
    dev = torch.device("cuda")
    layer = MoELayer(cfg_for(wl), case["params"], training=True, device=dev)
    routing = layer.new_routing()
    y = layer.forward(case["x"], routing=routing)
    grads = layer.backward(case["x"], case["dy"])
    torch.cuda.synchronize()
    assert layer.status() == 0
    return layer, y, routing, grads


@pytest.fixture(scope="module", params=CASES, ids=lambda w: w.name)
def ran(request):
    wl = request.param
    case = make_case(wl, device="cuda", gen_device="cpu")
    layer, y, routing, grads = _run(wl, case)
    return wl, case, layer, y, routing, grads


def test_routing_bit_exact(ran):
    wl, case, layer, y, routing, grads = ran
    L = case["L"]
    idx = case["idx"]
    assert np.array_equal(routing["topk_idx"].cpu().numpy(), idx)
    counts, offsets, perm, inv = L.dispatch(idx)
    assert np.array_equal(routing["counts"].cpu().numpy(), counts)
    assert np.array_equal(routing["offsets"].cpu().numpy(), offsets)
    assert np.array_equal(routing["perm"].cpu().numpy(), perm)
    assert np.array_equal(routing["inv_perm"].cpu().numpy(), inv)
    assert_close(to_np(routing["topk_w"]), case["w"], "topk_w", rtol=1e-5, atol=1e-6)


def test_forward_matches_oracle(ran):
    wl, case, layer, y, routing, grads = ran
    yo = case["L"].fwd(case["idx"], case["w"])
    assert_close(to_np(y), yo, "y")


def test_backward_matches_oracle(ran):
    wl, case, layer, y, routing, grads = ran
    L, idx, w = case["L"], case["idx"], case["w"]
    dx, dl, G = L.bwd(idx, w)
    assert_close(to_np(grads["dx"]), dx, "dx")
    dwr = L.drouter(idx, w, np.arange(wl.E))
    assert_close(to_np(grads["drouter_w"]), dwr, "drouter_w")
    counts = np.bincount(idx.ravel(), minlength=wl.E)
    experts = {0, wl.E - 1, int(np.argmax(counts)), int(np.argmin(counts))}
    small, large = np.flatnonzero(counts <= RESIDENT_ROWS), np.flatnonzero(counts > RESIDENT_ROWS)
    if small.size:
        experts.add(int(small[np.argmax(counts[small])]))     # largest group of the resident kernel
    if large.size:
        experts.add(int(large[np.argmin(counts[large])]))     # smallest group of the streaming kernel
    experts = sorted(experts)
    for e in experts:
        dgu, ddn = L.dw_full(idx, w, e, False)
        assert_close(to_np(grads["dw_gate_up"][e]), dgu, f"dw_gate_up[{e}]")
        assert_close(to_np(grads["dw_down"][e]), ddn, f"dw_down[{e}]")
    for s in range(wl.S):
        dgu, ddn = L.dw_full(idx, w, s, True)
        assert_close(to_np(grads["dws_gate_up"][s]), dgu, f"dws_gate_up[{s}]")
        assert_close(to_np(grads["dws_down"][s]), ddn, f"dws_down[{s}]")


def test_reruns_bit_identical(ran):
    wl, case, layer, y, routing, grads = ran
    y0 = y.clone()
    g0 = {k: v.clone() for k, v in grads.items() if v is not None}
    for _ in range(9):
        y1 = layer.forward(case["x"])
        g1 = layer.backward(case["x"], case["dy"])
        torch.cuda.synchronize()
        assert torch.equal(y1.view(torch.int16), y0.view(torch.int16))
        for k, v in g0.items():
            a = g1[k].view(torch.int32) if v.dtype == torch.float32 else g1[k].view(torch.int16)
            b = v.view(torch.int32) if v.dtype == torch.float32 else v.view(torch.int16)
            assert torch.equal(a, b), k


# ---------------------------------------------------------------- MXFP8 forward
MEDIUM_MX = synth.Workload("medium_mx", T=700, H=512, E=16, k=4, I=256, S=1, Is=256, score_fn=1,
                           n_group=4, topk_group=2, mxfp8=True, backward=False, seed=21)


def _mx_params(params):
    from mixture_experts_layer_persistent_b200 import quantize_mxfp8_weights
    out = {k: params[k] for k in ("router_w", "e_bias", "logit_bias")}
    for name, sname in (("w_gate_up", "s_gate_up"), ("w_down", "s_down"), ("ws_gate_up", "ss_gate_up"),
                        ("ws_down", "ss_down")):
        if params.get(name) is None:
            out[name] = out[sname] = None
            continue
        out[name], out[sname] = quantize_mxfp8_weights(params[name])
    return out


MX_CASES = [MEDIUM_MX,
            synth.scaled(MEDIUM_MX, name="medium_mx_softmax", score_fn=0, n_group=1, topk_group=1, S=0, Is=0,
                         T=333, seed=22),
            # I = 384: not a multiple of 256 (three 128-column h tiles, a K of three blocks in the
            # down GEMM), two shared experts, groups ending in partial 32-row blocks
            synth.scaled(MEDIUM_MX, name="medium_mx_i384", T=411, H=768, E=12, k=3, I=384, S=2, Is=384,
                         n_group=4, topk_group=2, seed=23)]


@pytest.mark.parametrize("wl", MX_CASES, ids=lambda w: w.name)
def test_mxfp8_forward_matches_oracle(wl):
    """MXFP8 forward: routing bit-exact; the h codes and scales the gate/up epilogue
    stored agree with the oracle's quantisation of h (see check_mx_h); y within
    2e-2 relative RMS (the acceptance of record), pooled and for every token."""
    import oracle
    case = make_case(wl, device="cuda", gen_device="cpu", mx=True)
    params = _mx_params(case["params"])
    layer = MoELayer(cfg_for(wl), params, training=False, device=torch.device("cuda"))
    routing = layer.new_routing()
    y = layer.forward(case["x"], routing=routing)
    torch.cuda.synchronize()
    assert layer.status() == 0
    assert np.array_equal(routing["topk_idx"].cpu().numpy(), case["idx"])
    L = case["L"]
    for name in ("Wgu", "Wdn", "Wgu_s", "Wdn_s"):
        if L.arrays.get(name) is not None:
            a = L.arrays[name].copy()
            oracle.mx_fakequant_bf16(a)
            L.set(**{name: a})
    hstat = check_mx_h(layer, L, case["idx"], np.arange(wl.T), routing["inv_perm"].cpu().numpy())
    yo = L.fwd(case["idx"], case["w"])
    err, worst = rel_rms_per_token(to_np(y), yo)
    print(f"{wl.name}: relative RMS of y {err:.3g} pooled, {worst:.3g} worst token; h {hstat}")
    assert err <= 2e-2, err
    assert worst <= 2e-2, worst
    # reruns are bit-identical
    y2 = layer.forward(case["x"])
    torch.cuda.synchronize()
    assert torch.equal(y2.view(torch.int16), y.view(torch.int16))


# ---------------------------------------------------------------- MXFP8 backward
def _mx_train_params(params):
    from mixture_experts_layer_persistent_b200 import quantize_mxfp8_weights_t
    out = _mx_params(params)
    for name, tname, sname in (("w_gate_up", "wt_gate_up", "st_gate_up"), ("w_down", "wt_down", "st_down"),
                               ("ws_gate_up", "wst_gate_up", "sst_gate_up"), ("ws_down", "wst_down", "sst_down")):
        if params.get(name) is None:
            out[tname] = out[sname] = None
            continue
        out[tname], out[sname] = quantize_mxfp8_weights_t(params[name])
    return out


def _rel_rms(got, want):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    return float(np.sqrt(np.sum((got - want) ** 2) / max(np.sum(want ** 2), 1e-300)))


MX_BWD_CASES = [
    synth.scaled(MEDIUM_MX, name="medium_mx_bwd", backward=True, seed=24),
    synth.scaled(MEDIUM_MX, name="medium_mx_bwd_softmax", T=333, score_fn=0, n_group=1, topk_group=1, S=2,
                 Is=256, backward=True, seed=25),
]


@pytest.mark.parametrize("wl", MX_BWD_CASES, ids=lambda w: w.name)
def test_mxfp8_backward_matches_oracle(wl):
    """MXFP8 training step: the forward as above, then dx (pooled and per token), the
    router weight gradient of the hottest, a median and the lightest routed expert,
    and the weight gradients of the hottest and a median routed expert and of every
    shared expert, each within 2e-2 relative RMS of the oracle's MXFP8 backward (the
    data gradients on MXFP8 operands, the weight gradients BF16); reruns
    bit-identical."""
    import oracle
    case = make_case(wl, device="cuda", gen_device="cpu", mx=True)
    params = _mx_train_params(case["params"])
    layer = MoELayer(cfg_for(wl), params, training=True, device=torch.device("cuda"))
    routing = layer.new_routing()
    y = layer.forward(case["x"], routing=routing)
    grads = layer.backward(case["x"], case["dy"])
    torch.cuda.synchronize()
    assert layer.status() == 0
    assert np.array_equal(routing["topk_idx"].cpu().numpy(), case["idx"])
    L = case["L"]
    for name in ("Wgu", "Wdn", "Wgu_s", "Wdn_s"):
        if L.arrays.get(name) is not None:
            a, b = L.arrays[name].copy(), L.arrays[name].copy()
            oracle.mx_fakequant_bf16(a)
            oracle.mx_fakequant_cols_bf16(b)
            L.set(**{name: a, name.replace("_s", "") + ("_sb" if name.endswith("_s") else "_b"): b})
    idx, w = case["idx"], case["w"]
    yo = L.fwd(idx, w)
    ey, _ = rel_rms_per_token(to_np(y), yo)
    dxo, _, _ = L.bwd(idx, w)
    edx, wdx = rel_rms_per_token(to_np(grads["dx"]), dxo)
    counts = np.bincount(idx.ravel(), minlength=wl.E)
    order = np.argsort(-counts, kind="stable")
    experts = [int(order[0]), int(order[len(order) // 2]), int(order[np.nonzero(counts[order])[0][-1]])]
    edr = _rel_rms(grads["drouter_w"].cpu().numpy()[experts], L.drouter(idx, w, experts))
    edw = []
    for grp, shared in [(experts[0], False), (experts[1], False)] + [(s_, True) for s_ in range(wl.S)]:
        dgu, ddn = L.dw_full(idx, w, grp, shared)
        gdgu = to_np(grads["dws_gate_up" if shared else "dw_gate_up"][grp])
        gddn = to_np(grads["dws_down" if shared else "dw_down"][grp])
        edw += [_rel_rms(gdgu, dgu), _rel_rms(gddn, ddn)]
    print(f"{wl.name}: relative RMS y {ey:.3g}, dx {edx:.3g} (worst token {wdx:.3g}), dWr {edr:.3g}, "
          f"dW {max(edw):.3g} (worst of {len(edw)})")
    for e in (ey, edx, wdx, edr, max(edw)):
        assert e <= 2e-2, (ey, edx, wdx, edr, edw)
    # reruns of the training step are bit-identical
    y2 = layer.forward(case["x"])
    g2 = layer.backward(case["x"], case["dy"])
    torch.cuda.synchronize()
    assert torch.equal(y2.view(torch.int16), y.view(torch.int16))
    for k, v in grads.items():
        if v is None:
            continue
        a = g2[k].view(torch.int32) if v.dtype == torch.float32 else g2[k].view(torch.int16)
        b = v.view(torch.int32) if v.dtype == torch.float32 else v.view(torch.int16)
        assert torch.equal(a, b), k
