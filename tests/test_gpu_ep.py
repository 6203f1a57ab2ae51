"""Expert parallelism: each rank's y and gradients against the one-GPU layer.

The ranks run on one device with one buffer set each (EPWorld), the phases in
stream order.  Rank r owns the routed experts [r E/world, (r+1) E/world); its
expert GEMMs read rows of every rank's tokens (pulled by index from that
rank's x) and push each output row into the slot rows of the token's rank.
Every output row depends only on its own input row and the expert's weights,
and the k-sum runs in slot order on the token's rank, so each rank's y must
equal moe_fwd of the same tokens with all E experts byte for byte, whatever
share of the rows each rank receives.  Rank 0's y is also checked against the
oracle at the layer tolerance.

Backward: the owner pulls dy rows like x rows and pushes dX rows and the
slot-gradient partials back to the tokens' ranks, so each rank's dx, router
gradient and shared-expert gradient equal moe_bwd on its tokens byte for byte;
an owner's expert weight gradients (summed over every rank's rows, in rank then
token order) equal moe_bwd's on the concatenated batch, byte for byte when that
batch routes its tokens the same way (the same router K split), else at the
layer tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_persistent_b200 import (EPWorld, MoELayer, abi, cfg_for, quantize_mxfp8_weights,
                                                   quantize_mxfp8_weights_t, split_params, synth)
from tests._support import assert_close, bits_to_bf16, oracle_layer, to_np

pytestmark = pytest.mark.gpu

CASES = [
    (1, synth.WORKLOADS["tiny"]),
    (2, synth.Workload("ep_softmax", T=300, H=512, E=16, k=4, I=256, S=1, Is=256, seed=51)),
    (4, synth.Workload("ep_sigmoid", T=260, H=512, E=16, k=4, I=256, S=1, Is=256, score_fn=1, n_group=4,
                       topk_group=2, seed=52)),
    # one expert per rank, two slots per token: a rank holds at most one slot of a token
    (8, synth.Workload("ep_one_expert_per_rank", T=200, H=256, E=8, k=2, I=128, seed=53)),
    # skewed routing: most rows go to the few ranks that own the favoured experts; two shared experts
    (4, synth.Workload("ep_zipf", T=500, H=512, E=16, k=4, I=256, S=2, Is=256, score_fn=1, n_group=4,
                       topk_group=2, zipf=3.0, seed=54)),
    # I = 384 (gate/up N tiles not a multiple of 2), softmax top-3 of 12 over 3 ranks
    (3, synth.Workload("ep_i384", T=333, H=768, E=12, k=3, I=384, S=1, Is=384, seed=55)),
]


def _rank_inputs(wl, world, dev, margins=True):
    """Parameters of the whole layer and one x per rank (top-k margins >= 1e-3)."""
    params = synth.draw_params(wl, dev)
    xs, bits = [], []
    for r in range(world):
        wr = synth.scaled(wl, seed=wl.seed * 100 + r)
        xb = synth.bf16_bits(synth.draw_x(wr, dev))
        if margins:
            L = oracle_layer(wl, params, xb)
            xb, _, _, _ = oracle.margin_reject(L, lambda a, wr=wr: synth.bf16_bits(synth.draw_x(wr, dev, attempt=a)))
        bits.append(xb)
        xs.append(bits_to_bf16(xb, dev))
    return params, xs, bits


def _margin_xs(wl, params, world, dev):
    """One x per rank with top-k margins >= 1e-3, routed by the oracle from the router
    parameters alone (no expert weight leaves the device)."""
    f32 = lambda t: None if t is None else t.detach().float().cpu().numpy()
    xs = []
    for r in range(world):
        wr = synth.scaled(wl, seed=wl.seed * 100 + r)
        L = oracle.Layer(wl.T, wl.H, wl.E, wl.k, wl.I, S=wl.S, Is=wl.Is, score_fn=wl.score_fn, n_group=wl.n_group,
                         topk_group=wl.topk_group, routed_scale=wl.routed_scale)
        L.set(x=synth.bf16_bits(synth.draw_x(wr, dev)), Wr=f32(params["router_w"]), bias=f32(params.get("e_bias")),
              lbias=f32(params.get("logit_bias")))
        xb, _, _, _ = oracle.margin_reject(L, lambda a, wr=wr: synth.bf16_bits(synth.draw_x(wr, dev, attempt=a)))
        xs.append(bits_to_bf16(xb, dev))
    return xs


def _same(a, b):
    return torch.equal(a.contiguous().view(torch.uint8), b.contiguous().view(torch.uint8))


@pytest.mark.parametrize("world,wl", CASES, ids=[f"{w.name}-w{n}" for n, w in CASES])
def test_each_rank_matches_the_one_gpu_layer(world, wl):
    dev = torch.device("cuda")
    params, xs, bits = _rank_inputs(wl, world, dev)
    cfg = cfg_for(wl)
    ep = EPWorld(cfg, world, [split_params(params, world, r, wl.E) for r in range(world)])
    ys = ep.forward(xs)
    ys2 = ep.forward(xs)                       # rerun on the same buffers
    torch.cuda.synchronize()
    assert abi.moe_status(torch.cuda.current_stream().cuda_stream) == 0
    layer = MoELayer(cfg, params, training=False)
    for r in range(world):
        y_ref = layer.forward(xs[r]).clone()
        torch.cuda.synchronize()
        assert _same(ys[r], y_ref), f"rank {r}: y differs from moe_fwd"
        assert _same(ys2[r], ys[r]), f"rank {r}: rerun differs"
    assert layer.status() == 0
    L = oracle_layer(wl, params, bits[0])
    idx, w, _ = L.route()
    assert_close(to_np(ys[0]), L.fwd(idx, w), f"{wl.name} rank 0 y vs oracle")


def test_dsv3_expert_shape_over_eight_ranks():
    """E = 256 experts of the DeepSeek-V3 shape over 8 ranks of 512 tokens each (the
    4096-token batch split 8 ways), sigmoid + group-limited routing, one shared
    expert; plus a skewed variant where a logit term sends most rows to the ranks
    owning the favoured experts.  Byte equality with moe_fwd per rank, no status."""
    dev = torch.device("cuda")
    world = 8
    for wl in (synth.scaled(synth.WORKLOADS["dsv3"], name="ep_dsv3", T=512, seed=56),
               synth.scaled(synth.WORKLOADS["dsv3"], name="ep_dsv3_zipf", T=512, zipf=1.2, seed=57)):
        params = synth.draw_params(wl, dev)
        xs = [synth.draw_x(synth.scaled(wl, seed=wl.seed * 100 + r), dev) for r in range(world)]
        cfg = cfg_for(wl)
        ep = EPWorld(cfg, world, [split_params(params, world, r, wl.E) for r in range(world)])
        ys = ep.forward(xs)
        torch.cuda.synchronize()
        assert abi.moe_status(torch.cuda.current_stream().cuda_stream) == 0
        layer = MoELayer(cfg, params, training=False)
        for r in range(world):
            y_ref = layer.forward(xs[r])
            torch.cuda.synchronize()
            assert _same(ys[r], y_ref), f"{wl.name} rank {r}: y differs from moe_fwd"
        del ep, layer, params, xs, ys
        torch.cuda.empty_cache()


def _rank_dys(wl, world, dev):
    return [synth.draw_dy(synth.scaled(wl, seed=wl.seed * 100 + 50 + r), dev) for r in range(world)]


@pytest.mark.parametrize("world,wl", CASES, ids=[f"{w.name}-w{n}" for n, w in CASES])
def test_backward_matches_the_one_gpu_layer(world, wl):
    dev = torch.device("cuda")
    params, xs, bits = _rank_inputs(wl, world, dev)
    dys = _rank_dys(wl, world, dev)
    cfg = cfg_for(wl)
    el = wl.E // world
    ep = EPWorld(cfg, world, [split_params(params, world, r, wl.E) for r in range(world)], training=True)
    ys = ep.forward(xs)
    grads = ep.backward(dys)
    torch.cuda.synchronize()
    assert abi.moe_status(torch.cuda.current_stream().cuda_stream) == 0
    # per rank: y, dx, the router gradient and the shared experts' gradient of its tokens
    layer = MoELayer(cfg, params, training=True)
    for r in range(world):
        y_ref = layer.forward(xs[r]).clone()
        g_ref = layer.backward(xs[r], dys[r])
        torch.cuda.synchronize()
        assert _same(ys[r], y_ref), f"rank {r}: y"
        for n in ("dx", "drouter_w", "dws_gate_up", "dws_down"):
            if g_ref.get(n) is not None:
                assert _same(grads[r][n], g_ref[n]), f"rank {r}: {n}"
    assert layer.status() == 0
    # the owners' expert gradients against the one-GPU layer on every rank's tokens
    whole = synth.scaled(wl, T=wl.T * world)
    big = MoELayer(cfg_for(whole), params, training=True)
    routing = big.new_routing()
    big.forward(torch.cat(xs), routing=routing)
    g_all = big.backward(torch.cat(xs), torch.cat(dys))
    torch.cuda.synchronize()
    assert big.status() == 0
    same_routing = True
    for r in range(world):                 # does the concatenated batch route each token as its rank did?
        rr = layer.new_routing()
        layer.forward(xs[r], routing=rr)
        sl = slice(r * wl.T, (r + 1) * wl.T)
        same_routing &= _same(rr["topk_idx"], routing["topk_idx"][sl]) and _same(rr["topk_w"], routing["topk_w"][sl])
    assert same_routing, "these cases keep the router's K split, so the routing must agree"
    for r in range(world):
        for n in ("dw_gate_up", "dw_down"):
            assert _same(grads[r][n], g_all[n][r * el:(r + 1) * el]), f"owner {r}: {n}"
    # rank 0's dx against the oracle
    L = oracle_layer(wl, params, bits[0], synth.bf16_bits(dys[0]))
    idx, w, _ = L.route()
    dxo, _, _ = L.bwd(idx, w)
    assert_close(to_np(grads[0]["dx"]), dxo, f"{wl.name} rank 0 dx vs oracle")


def test_backward_dsv3_expert_shape_over_eight_ranks():
    """The DeepSeek-V3 shape over 8 ranks of 256 tokens (32 experts per rank, about
    64 rows per expert): per-rank y, dx, router and shared-expert gradients byte-equal
    to moe_bwd of the rank's tokens; each owner's expert weight gradients byte-equal
    to moe_bwd's on all 2048 tokens.  At 256 and 2048 tokens the router splits its
    contraction the same way (8 K splits), so that batch routes every token as its
    rank did (checked); top-k margins of 1e-3 as everywhere."""
    dev = torch.device("cuda")
    world = 8
    wl = synth.scaled(synth.WORKLOADS["dsv3"], name="ep_dsv3_bwd", T=256, seed=58)
    el = wl.E // world
    params = synth.draw_params(wl, dev)
    xs = _margin_xs(wl, params, world, dev)
    dys = _rank_dys(wl, world, dev)
    cfg = cfg_for(wl)
    ep = EPWorld(cfg, world, [split_params(params, world, r, wl.E) for r in range(world)], training=True)
    ys = ep.forward(xs)
    grads = ep.backward(dys)
    torch.cuda.synchronize()
    assert abi.moe_status(torch.cuda.current_stream().cuda_stream) == 0
    layer = MoELayer(cfg, params, training=True)
    routings = []
    for r in range(world):
        rr = layer.new_routing()
        y_ref = layer.forward(xs[r], routing=rr)
        g_ref = layer.backward(xs[r], dys[r])
        torch.cuda.synchronize()
        assert _same(ys[r], y_ref), f"rank {r}: y"
        for n in ("dx", "drouter_w", "dws_gate_up", "dws_down"):
            assert _same(grads[r][n], g_ref[n]), f"rank {r}: {n}"
        routings.append(rr)
        del g_ref
    del layer
    torch.cuda.empty_cache()
    big = MoELayer(cfg_for(synth.scaled(wl, T=wl.T * world)), params, training=True)
    routing = big.new_routing()
    big.forward(torch.cat(xs), routing=routing)
    g_all = big.backward(torch.cat(xs), torch.cat(dys))
    torch.cuda.synchronize()
    assert big.status() == 0
    for r in range(world):
        sl = slice(r * wl.T, (r + 1) * wl.T)
        assert _same(routings[r]["topk_idx"], routing["topk_idx"][sl]), f"rank {r}: selection"
        assert _same(routings[r]["topk_w"], routing["topk_w"][sl]), f"rank {r}: routing weights"
    for r in range(world):
        for n in ("dw_gate_up", "dw_down"):
            assert _same(grads[r][n], g_all[n][r * el:(r + 1) * el]), f"owner {r}: {n}"


def _mx_params(params, world, E):
    """MXFP8 weights of the whole layer (for moe_fwd) and of each rank's experts (each
    rank quantises its own slice: the same codes, scales packed for the slice)."""
    full = {k: params[k] for k in ("router_w", "e_bias", "logit_bias")}
    for name, sname in (("w_gate_up", "s_gate_up"), ("w_down", "s_down"), ("ws_gate_up", "ss_gate_up"),
                        ("ws_down", "ss_down")):
        full[name], full[sname] = (quantize_mxfp8_weights(params[name]) if params.get(name) is not None
                                   else (None, None))
    el = E // world
    ranks = []
    for r in range(world):
        p = dict(full)
        for name, sname in (("w_gate_up", "s_gate_up"), ("w_down", "s_down")):
            p[name], p[sname] = quantize_mxfp8_weights(params[name][r * el:(r + 1) * el].contiguous())
        ranks.append(p)
    return full, ranks


MX_CASES = [
    (4, synth.Workload("ep_mx", T=300, H=512, E=16, k=4, I=256, S=1, Is=256, score_fn=1, n_group=4, topk_group=2,
                       mxfp8=True, backward=False, seed=61)),
    (3, synth.Workload("ep_mx_i384", T=211, H=768, E=12, k=3, I=384, S=2, Is=384, mxfp8=True, backward=False,
                       seed=62)),
    (8, synth.Workload("ep_mx_one_expert_per_rank", T=150, H=256, E=8, k=2, I=128, mxfp8=True, backward=False,
                       seed=63)),
]


@pytest.mark.parametrize("world,wl", MX_CASES, ids=[f"{w.name}-w{n}" for n, w in MX_CASES])
def test_mxfp8_forward_matches_the_one_gpu_layer(world, wl):
    """MXFP8: each rank quantises its x in the routing phase and the owners pull the
    e4m3 rows and their scales; each rank's y equals the one-GPU MXFP8 forward's on its
    tokens byte for byte."""
    dev = torch.device("cuda")
    params = synth.draw_params(wl, dev)
    xs = [synth.draw_x(synth.scaled(wl, seed=wl.seed * 100 + r), dev) for r in range(world)]
    full, ranks = _mx_params(params, world, wl.E)
    cfg = cfg_for(wl)
    ep = EPWorld(cfg, world, ranks)
    ys = ep.forward(xs)
    torch.cuda.synchronize()
    assert abi.moe_status(torch.cuda.current_stream().cuda_stream) == 0
    layer = MoELayer(cfg, full, training=False)
    for r in range(world):
        y_ref = layer.forward(xs[r]).clone()
        torch.cuda.synchronize()
        assert _same(ys[r], y_ref), f"rank {r}: y differs from the MXFP8 moe_fwd"
    assert layer.status() == 0


def test_mxfp8_dsv3_expert_shape_over_eight_ranks():
    dev = torch.device("cuda")
    world = 8
    wl = synth.scaled(synth.WORKLOADS["dsv3_mxfp8"], name="ep_mx_dsv3", T=1024, seed=64)
    params = synth.draw_params(wl, dev)
    xs = [synth.draw_x(synth.scaled(wl, seed=wl.seed * 100 + r), dev) for r in range(world)]
    full, ranks = _mx_params(params, world, wl.E)
    del params
    torch.cuda.empty_cache()
    cfg = cfg_for(wl)
    ep = EPWorld(cfg, world, ranks)
    ys = ep.forward(xs)
    torch.cuda.synchronize()
    assert abi.moe_status(torch.cuda.current_stream().cuda_stream) == 0
    layer = MoELayer(cfg, full, training=False)
    for r in range(world):
        y_ref = layer.forward(xs[r])
        torch.cuda.synchronize()
        assert _same(ys[r], y_ref), f"rank {r}: y differs from the MXFP8 moe_fwd"


def _mx_train_params(params, world, E):
    """_mx_params plus the transposed copies the MXFP8 backward reads, for the whole
    layer and for each rank's slice."""
    full, ranks = _mx_params(params, world, E)
    el = E // world
    for name in ("w_gate_up", "w_down", "ws_gate_up", "ws_down"):
        t = "wt" + name[1:] if name.startswith("w_") else "wst" + name[2:]
        ts = "st" + name[1:] if name.startswith("w_") else "sst" + name[2:]
        if params.get(name) is None:
            continue
        full[t], full[ts] = quantize_mxfp8_weights_t(params[name])
        for r in range(world):
            if name.startswith("ws"):
                ranks[r][t], ranks[r][ts] = full[t], full[ts]
            else:
                ranks[r][t], ranks[r][ts] = quantize_mxfp8_weights_t(params[name][r * el:(r + 1) * el].contiguous())
    return full, ranks


def test_mxfp8_training_matches_the_one_gpu_layer():
    """The MXFP8 training step over 4 ranks: every rank's y, dx, router and
    shared-expert gradients byte-equal to the one-GPU MXFP8 layer's (forward with saved
    state + MXFP8 backward) on its tokens; every owner's expert weight gradients
    byte-equal to the one-GPU layer's on the concatenated batch (same router K split,
    so the same routing, checked)."""
    dev = torch.device("cuda")
    world = 4
    wl = synth.Workload("ep_mx_train", T=300, H=512, E=16, k=4, I=256, S=1, Is=256, score_fn=1, n_group=4,
                        topk_group=2, mxfp8=True, seed=67)
    el = wl.E // world
    params = synth.draw_params(wl, dev)
    xs = [synth.draw_x(synth.scaled(wl, seed=wl.seed * 100 + r), dev) for r in range(world)]
    dys = _rank_dys(wl, world, dev)
    full, ranks = _mx_train_params(params, world, wl.E)
    cfg = cfg_for(wl)
    ep = EPWorld(cfg, world, ranks, training=True)
    ys = ep.forward(xs)
    grads = ep.backward(dys)
    torch.cuda.synchronize()
    assert abi.moe_status(torch.cuda.current_stream().cuda_stream) == 0
    layer = MoELayer(cfg, full, training=True)
    for r in range(world):
        y_ref = layer.forward(xs[r]).clone()
        g_ref = layer.backward(xs[r], dys[r])
        torch.cuda.synchronize()
        assert _same(ys[r], y_ref), f"rank {r}: y"
        for n in ("dx", "drouter_w", "dws_gate_up", "dws_down"):
            assert _same(grads[r][n], g_ref[n]), f"rank {r}: {n}"
    big = MoELayer(cfg_for(synth.scaled(wl, T=wl.T * world)), full, training=True)
    routing = big.new_routing()
    big.forward(torch.cat(xs), routing=routing)
    g_all = big.backward(torch.cat(xs), torch.cat(dys))
    torch.cuda.synchronize()
    assert big.status() == 0
    for r in range(world):
        rr = layer.new_routing()
        layer.forward(xs[r], routing=rr)
        sl = slice(r * wl.T, (r + 1) * wl.T)
        assert _same(rr["topk_idx"], routing["topk_idx"][sl]) and _same(rr["topk_w"], routing["topk_w"][sl])
    for r in range(world):
        for n in ("dw_gate_up", "dw_down"):
            assert _same(grads[r][n], g_all[n][r * el:(r + 1) * el]), f"owner {r}: {n}"


@pytest.mark.parametrize("mx,train", [(False, True), (True, False), (True, True)],
                         ids=["bf16_train", "mxfp8", "mxfp8_train"])
def test_persistent_and_split_experts_phase_agree(mx, train):
    """The owner's experts phases as one persistent launch each (the default) and as
    the split launches: y and, when training, every gradient of the backward that
    reads the forward's saved rows, byte for byte; one launch for the persistent
    forward experts phase."""
    dev = torch.device("cuda")
    world = 4
    wl = synth.Workload("ep_sched", T=300, H=512, E=16, k=4, I=256, S=1, Is=256, score_fn=1, n_group=4,
                        topk_group=2, mxfp8=mx, backward=train, seed=65)
    params = synth.draw_params(wl, dev)
    xs = [synth.draw_x(synth.scaled(wl, seed=wl.seed * 100 + r), dev) for r in range(world)]
    if mx:
        _, rank_params = (_mx_train_params if train else _mx_params)(params, world, wl.E)
    else:
        rank_params = [split_params(params, world, r, wl.E) for r in range(world)]
    dys = _rank_dys(wl, world, dev)
    out = {}
    for sched in (abi.MOK_SCHEDULE_PERSISTENT, abi.MOK_SCHEDULE_SPLIT):
        abi.moe_set_schedule(sched)
        try:
            ep = EPWorld(cfg_for(wl), world, rank_params, training=train)
            ys = ep.forward(xs)
            n = None
            if sched == abi.MOK_SCHEDULE_PERSISTENT:
                abi.moe_ep_experts(cfg_for(wl), world, world - 1, train, [x.data_ptr() for x in xs],
                                   [s.data_ptr() for s in ep.states], ep.cparams[world - 1],
                                   ep.scratch[world - 1].data_ptr(), ep.scratch_bytes,
                                   torch.cuda.current_stream().cuda_stream)
                n = abi.moe_launch_count()
            grads = ep.backward(dys) if train else None
            torch.cuda.synchronize()
        finally:
            abi.moe_set_schedule(abi.MOK_SCHEDULE_PERSISTENT)
        assert abi.moe_status(torch.cuda.current_stream().cuda_stream) == 0
        out[sched] = ([y.clone() for y in ys], grads, n)
    (yp, gp, n), (ys_, gs, _) = out[abi.MOK_SCHEDULE_PERSISTENT], out[abi.MOK_SCHEDULE_SPLIT]
    assert n == 1, "the persistent experts phase is one launch"
    for r in range(world):
        assert _same(yp[r], ys_[r]), f"rank {r}: y"
        if train:
            for k in gp[r]:
                if gp[r][k] is not None:
                    assert _same(gp[r][k], gs[r][k]), f"rank {r}: {k}"


def test_experts_phase_on_buffers_of_ones():
    """The persistent experts phase on state and scratch buffers filled with 0xFF bytes
    (what an int array of -1s leaves behind) before their first use: the grid
    barriers must not read leftover words as arrivals, so the result equals the one
    on zeroed buffers byte for byte and no status bit is set."""
    dev = torch.device("cuda")
    world = 4
    wl = synth.Workload("ep_ones", T=300, H=512, E=16, k=4, I=256, S=1, Is=256, score_fn=1, n_group=4,
                        topk_group=2, seed=66)
    params = synth.draw_params(wl, dev)
    xs = [synth.draw_x(synth.scaled(wl, seed=wl.seed * 100 + r), dev) for r in range(world)]
    dys = _rank_dys(wl, world, dev)
    rank_params = [split_params(params, world, r, wl.E) for r in range(world)]
    res = []
    for fill in (0x00, 0xFF):
        ep = EPWorld(cfg_for(wl), world, rank_params, training=True)
        for t in ep.states + ep.scratch + ep.bwd:
            t.fill_(fill)
        ys = ep.forward(xs)
        g = ep.backward(dys)
        torch.cuda.synchronize()
        assert abi.moe_status(torch.cuda.current_stream().cuda_stream) == 0, f"fill {fill:#x}"
        res.append(([y.clone() for y in ys], g))
    for r in range(world):
        assert _same(res[0][0][r], res[1][0][r]), f"rank {r}: y"
        for k in res[0][1][r]:
            if res[0][1][r][k] is not None:
                assert _same(res[0][1][r][k], res[1][1][r][k]), f"rank {r}: {k}"


def test_owner_with_no_routed_rows():
    """A logit term that rules out the experts of rank 1 (4..7): rank 1 receives no
    routed row, its experts phase runs only its shared expert on its own 77 tokens
    (a ragged count), and its experts' weight gradients are zero.  Every rank's y, dx,
    router and shared-expert gradients equal the one-GPU layer's byte for byte, in
    BF16 training."""
    dev = torch.device("cuda")
    world = 2
    wl = synth.Workload("ep_empty_owner", T=77, H=256, E=8, k=2, I=128, S=1, Is=128, seed=68)
    params = synth.draw_params(wl, dev)
    params["logit_bias"] = torch.tensor([0.0] * 4 + [-100.0] * 4, device=dev)
    xs = [synth.draw_x(synth.scaled(wl, seed=wl.seed * 100 + r), dev) for r in range(world)]
    dys = _rank_dys(wl, world, dev)
    cfg = cfg_for(wl)
    ep = EPWorld(cfg, world, [split_params(params, world, r, wl.E) for r in range(world)], training=True)
    ys = ep.forward(xs)
    grads = ep.backward(dys)
    torch.cuda.synchronize()
    assert abi.moe_status(torch.cuda.current_stream().cuda_stream) == 0
    layer = MoELayer(cfg, params, training=True)
    for r in range(world):
        routing = layer.new_routing()
        y_ref = layer.forward(xs[r], routing=routing).clone()
        g_ref = layer.backward(xs[r], dys[r])
        torch.cuda.synchronize()
        assert int(routing["counts"][4:].sum()) == 0, "the logit term keeps experts 4..7 empty"
        assert _same(ys[r], y_ref), f"rank {r}: y"
        for n in ("dx", "drouter_w", "dws_gate_up", "dws_down"):
            assert _same(grads[r][n], g_ref[n]), f"rank {r}: {n}"
    assert not grads[1]["dw_gate_up"].any() and not grads[1]["dw_down"].any(), "empty experts: zero weight gradients"
