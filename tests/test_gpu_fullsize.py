"""Full-size parity of the layer against the fp64 oracle (the workloads and the
launch configuration the benchmark times).

Routing (indices for every token, counts, offsets, permutations) must match
bit-exactly; outputs and gradients are compared on samples the oracle computes
one by one: sampled tokens of y and dx, sampled entries of the weight
gradients of the hottest, a median, the emptiest and the shared experts, and
full router-gradient rows of lightly loaded experts.  BF16 bound:
|gpu - oracle| <= 1e-2 + 1e-2 |oracle|; MXFP8 forward: relative RMS <= 2e-2.
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_persistent_b200 import MoELayer, cfg_for, quantize_mxfp8_weights, synth
from tests._support import (assert_close, bits_to_bf16, check_mx_h, oracle_layer, packed_scale_offsets,
                            rel_rms_per_token, to_np)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _case(wl, mx=False):
    dev = torch.device("cuda")
    params = synth.draw_params(wl, dev)
    x_bits = synth.bf16_bits(synth.draw_x(wl, dev))
    dy_bits = synth.bf16_bits(synth.draw_dy(wl, dev)) if wl.backward else None
    L = oracle_layer(wl, params, x_bits, dy_bits, mx=mx)
    x_bits, idx, w, _ = oracle.margin_reject(L, lambda a: synth.bf16_bits(synth.draw_x(wl, dev, attempt=a)))
    return params, L, bits_to_bf16(x_bits, dev), (bits_to_bf16(dy_bits, dev) if dy_bits is not None else None), idx, w


def _check_routing(L, routing, idx):
    assert np.array_equal(routing["topk_idx"].cpu().numpy(), idx)
    counts, offsets, perm, inv = L.dispatch(idx)
    assert np.array_equal(routing["counts"].cpu().numpy(), counts)
    assert np.array_equal(routing["offsets"].cpu().numpy(), offsets)
    assert np.array_equal(routing["perm"].cpu().numpy(), perm)
    assert np.array_equal(routing["inv_perm"].cpu().numpy(), inv)
    return counts


def _sample_tokens(T, n, seed):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, T - 1], rng.choice(T, n, replace=False)])).astype(np.int32)


@pytest.mark.parametrize("name", ["small", "dsv3", "dsv3_zipf"])
def test_bf16_full_size(name):
    wl = synth.WORKLOADS[name]
    params, L, x, dy, idx, w = _case(wl)
    layer = MoELayer(cfg_for(wl), params, training=wl.backward, device=torch.device("cuda"))
    routing = layer.new_routing()
    y = layer.forward(x, routing=routing)
    grads = layer.backward(x, dy) if wl.backward else None
    torch.cuda.synchronize()
    assert layer.status() == 0
    counts = _check_routing(L, routing, idx)

    toks = _sample_tokens(wl.T, 30, 1)
    assert_close(to_np(y[torch.from_numpy(toks).long().cuda()]), L.fwd(idx, w, tokens=toks), f"{name} y")

    # reruns are bit-identical
    y2 = layer.forward(x)
    torch.cuda.synchronize()
    assert torch.equal(y2.view(torch.int16), y.view(torch.int16))
    if not wl.backward:
        return
    g2 = layer.backward(x, dy, layer.new_grads())
    torch.cuda.synchronize()
    for k, v in grads.items():
        if v is not None:
            assert torch.equal(g2[k].view(torch.int16 if v.dtype == torch.bfloat16 else torch.int32),
                               v.view(torch.int16 if v.dtype == torch.bfloat16 else torch.int32)), k

    toks = _sample_tokens(wl.T, 12, 2)
    dx, _, _ = L.bwd(idx, w, tokens=toks)
    assert_close(to_np(grads["dx"][torch.from_numpy(toks).long().cuda()]), dx, f"{name} dx")

    rng = np.random.default_rng(3)
    order = np.argsort(counts, kind="stable")
    groups = [(int(order[-1]), False), (int(order[len(order) // 2]), False), (int(order[0]), False)]
    groups += [(s, True) for s in range(wl.S)]
    for g, shared in groups:
        gu = grads["dws_gate_up" if shared else "dw_gate_up"][g]
        dn = grads["dws_down" if shared else "dw_down"][g]
        n = 24 if shared else 32
        rr, cc = rng.integers(0, 2 * wl.I, n), rng.integers(0, wl.H, n)
        want = L.dw_entries(idx, w, g, shared, 0, rr, cc)
        got = to_np(gu[torch.from_numpy(rr).long().cuda(), torch.from_numpy(cc).long().cuda()])
        assert_close(got, want, f"{name} dW_gate_up[{g}{' shared' if shared else ''}]")
        rr, cc = rng.integers(0, wl.H, n), rng.integers(0, wl.I, n)
        want = L.dw_entries(idx, w, g, shared, 1, rr, cc)
        got = to_np(dn[torch.from_numpy(rr).long().cuda(), torch.from_numpy(cc).long().cuda()])
        assert_close(got, want, f"{name} dW_down[{g}{' shared' if shared else ''}]")

    light = [int(e) for e in order if 0 < counts[e] <= 40][:2]
    empty = [int(e) for e in order if counts[e] == 0][:1]
    experts = light + empty
    if experts:
        assert_close(to_np(grads["drouter_w"][torch.tensor(experts).cuda()]), L.drouter(idx, w, experts),
                     f"{name} drouter_w")


def test_mxfp8_full_size():
    wl = synth.WORKLOADS["dsv3_mxfp8"]
    params, L, x, _, idx, w = _case(wl, mx=True)
    qp = {k: params[k] for k in ("router_w", "e_bias", "logit_bias")}
    for name, sname in (("w_gate_up", "s_gate_up"), ("w_down", "s_down"), ("ws_gate_up", "ss_gate_up"),
                        ("ws_down", "ss_down")):
        qp[name], qp[sname] = quantize_mxfp8_weights(params[name])
    torch.cuda.synchronize()
    # weight quantisation is bit-exact against the oracle's (sampled rows)
    rows = np.array([0, 1, 777, 2 * wl.I * wl.E - 1])
    wq, ws = oracle.mx_quantize(L.arrays["Wgu"].reshape(-1, wl.H)[rows])
    assert np.array_equal(qp["w_gate_up"].view(-1, wl.H)[torch.from_numpy(rows).cuda()].cpu().numpy(), wq)
    at = packed_scale_offsets(rows, wl.H // 32, 2 * wl.I * wl.E)
    assert np.array_equal(qp["s_gate_up"][torch.from_numpy(at.ravel()).cuda()].cpu().numpy().reshape(at.shape), ws)
    del params
    layer = MoELayer(cfg_for(wl), qp, training=False, device=torch.device("cuda"))
    routing = layer.new_routing()
    y = layer.forward(x, routing=routing)
    torch.cuda.synchronize()
    assert layer.status() == 0
    _check_routing(L, routing, idx)
    for name in ("Wgu", "Wdn", "Wgu_s", "Wdn_s"):
        oracle.mx_fakequant_bf16(L.arrays[name])
    L.set()
    toks = _sample_tokens(wl.T, 30, 4)
    hstat = check_mx_h(layer, L, idx, toks, routing["inv_perm"].cpu().numpy())
    yo = L.fwd(idx, w, tokens=toks)
    got = to_np(y[torch.from_numpy(toks).long().cuda()])
    err, worst = rel_rms_per_token(got, yo)
    print(f"dsv3_mxfp8: relative RMS of y {err:.3g} pooled, {worst:.3g} worst sampled token; h {hstat}")
    assert err <= 2e-2, err
    assert worst <= 2e-2, worst
    y2 = layer.forward(x)
    torch.cuda.synchronize()
    assert torch.equal(y2.view(torch.int16), y.view(torch.int16))


def test_mxfp8_backward_dsv3_expert_shape():
    """MXFP8 training step at the DeepSeek-V3 expert shape (H = 7168, I = 2048, top-8,
    one shared expert, grouped sigmoid routing) with 16 routed experts and 256 rows
    each on average: dx on sampled tokens, sampled entries of both weight gradients
    of the hottest routed and of the shared expert, and the router-gradient row of
    the lightest expert, each within 2e-2 relative RMS of the oracle's MXFP8
    backward; reruns bit-identical."""
    from mixture_experts_layer_persistent_b200 import quantize_mxfp8_weights_t
    wl = synth.scaled(synth.WORKLOADS["dsv3_mxfp8_e16"], backward=True)
    params, L, x, dy, idx, w = _case(wl, mx=True)
    qp = {k: params[k] for k in ("router_w", "e_bias", "logit_bias")}
    for name, sname, tname, tsname in (("w_gate_up", "s_gate_up", "wt_gate_up", "st_gate_up"),
                                       ("w_down", "s_down", "wt_down", "st_down"),
                                       ("ws_gate_up", "ss_gate_up", "wst_gate_up", "sst_gate_up"),
                                       ("ws_down", "ss_down", "wst_down", "sst_down")):
        qp[name], qp[sname] = quantize_mxfp8_weights(params[name])
        qp[tname], qp[tsname] = quantize_mxfp8_weights_t(params[name])
    del params
    layer = MoELayer(cfg_for(wl), qp, training=True, device=torch.device("cuda"))
    routing = layer.new_routing()
    layer.forward(x, routing=routing)
    grads = layer.backward(x, dy)
    torch.cuda.synchronize()
    assert layer.status() == 0
    counts = _check_routing(L, routing, idx)
    for name in ("Wgu", "Wdn", "Wgu_s", "Wdn_s"):
        b = L.arrays[name].copy()
        oracle.mx_fakequant_cols_bf16(b)
        oracle.mx_fakequant_bf16(L.arrays[name])
        L.set(**{name.replace("_s", "") + ("_sb" if name.endswith("_s") else "_b"): b})
    toks = _sample_tokens(wl.T, 24, 5)
    dxo, _, _ = L.bwd(idx, w, tokens=toks)
    edx, wdx = rel_rms_per_token(to_np(grads["dx"][torch.from_numpy(toks).long().cuda()]), dxo)
    rng = np.random.default_rng(6)
    order = np.argsort(-counts, kind="stable")
    errs = []
    for g, shared in ((int(order[0]), False), (0, True)):
        dgu = grads["dws_gate_up" if shared else "dw_gate_up"][g]
        ddn = grads["dws_down" if shared else "dw_down"][g]
        for which, M, N, got in ((0, 2 * wl.I, wl.H, dgu), (1, wl.H, wl.I, ddn)):
            r_, c_ = rng.integers(0, M, 12), rng.integers(0, N, 12)
            want = L.dw_entries(idx, w, g, shared, which, r_, c_)
            have = to_np(got[torch.from_numpy(r_).long().cuda(), torch.from_numpy(c_).long().cuda()])
            errs.append(float(np.sqrt(np.sum((have - want) ** 2) / np.sum(want ** 2))))
    light = [int(e) for e in order if counts[e] > 0][-1:]
    dro = L.drouter(idx, w, light)
    gdr = to_np(grads["drouter_w"][torch.tensor(light).cuda()])
    edr = float(np.sqrt(np.sum((gdr - dro) ** 2) / np.sum(dro ** 2)))
    print(f"{wl.name} backward: relative RMS dx {edx:.3g} (worst sampled token {wdx:.3g}), "
          f"dW entries {max(errs):.3g} (worst of {len(errs)}), dWr {edr:.3g}")
    for e in (edx, wdx, max(errs), edr):
        assert e <= 2e-2, (edx, wdx, errs, edr)
    g2 = layer.backward(x, dy)
    torch.cuda.synchronize()
    for k in ("dx", "dw_gate_up", "dw_down", "drouter_w"):
        a, b = g2[k], grads[k]
        vw = torch.int32 if a.dtype == torch.float32 else torch.int16
        assert torch.equal(a.view(vw), b.view(vw)), k
