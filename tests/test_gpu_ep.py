"""Expert parallelism: each rank's y against the one-GPU layer on its tokens.

The ranks run on one device with one buffer set each (EPWorld), the phases in
stream order.  Rank r owns the routed experts [r E/world, (r+1) E/world); its
expert GEMMs read rows of every rank's tokens (pulled by index from that
rank's x) and push each output row into the slot rows of the token's rank.
Every output row depends only on its own input row and the expert's weights,
and the k-sum runs in slot order on the token's rank, so each rank's y must
equal moe_fwd of the same tokens with all E experts byte for byte, whatever
share of the rows each rank receives.  Rank 0's y is also checked against the
oracle at the layer tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_persistent_b200 import EPWorld, MoELayer, abi, cfg_for, split_params, synth
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
