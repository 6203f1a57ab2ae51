"""Seeded synthetic inputs for the MoE layer workloads.

This module draws random numbers and nothing else: it holds none of the
layer's arithmetic (no routing, no expert math), so both the CUDA path and the
fp64 oracle can consume what it produces.  All tensors are drawn with
``torch.Generator`` streams keyed by (seed, tensor name[, attempt]); large
workloads are drawn on the GPU in per-expert chunks, small ones on the CPU.

Distributions (one reading of the workload descriptions, N(0, s) = std s):
  x, dy                ~ N(0, 1)            rounded to bf16
  router_w [E, H]      ~ N(0, 1/sqrt(H))    fp32
  e_bias [E]           = 0.01 * N(0, 1)     fp32, sigmoid-routed workloads only
  logit_bias [E]       = -1.2 * ln(pi(e)+1) for a seeded random permutation pi
                         (Zipf(1.2) popularity over a random expert order;
                         imbalanced workload only)
  expert / shared W    ~ N(0, 0.02)         rounded to bf16
"""
from __future__ import annotations

import dataclasses
import math
import zlib

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    E: int
    k: int
    I: int
    S: int = 0
    Is: int = 0
    score_fn: int = 0          # 0 softmax, 1 sigmoid + selection bias
    n_group: int = 1
    topk_group: int = 1
    zipf: float = 0.0          # >0: add -zipf*ln(rank) to the logits
    routed_scale: float = 1.0  # factor on the renormalised routing weights
    mxfp8: bool = False
    backward: bool = True
    seed: int = 0


WORKLOADS = {
    "tiny": Workload("tiny", T=64, H=256, E=8, k=2, I=128, seed=0),
    "small": Workload("small", T=2048, H=2048, E=64, k=6, I=1408, S=2, Is=1408,
                      backward=False, seed=1),
    "dsv3": Workload("dsv3", T=4096, H=7168, E=256, k=8, I=2048, S=1, Is=2048, score_fn=1,
                     n_group=8, topk_group=4, seed=2),
    "dsv3_mxfp8": Workload("dsv3_mxfp8", T=8192, H=7168, E=256, k=8, I=2048, S=1, Is=2048,
                           score_fn=1, n_group=8, topk_group=4, mxfp8=True, backward=False,
                           seed=3),
    "dsv3_zipf": Workload("dsv3_zipf", T=16384, H=7168, E=256, k=8, I=2048, S=1, Is=2048,
                          score_fn=1, n_group=8, topk_group=4, zipf=1.2, seed=4),
    # 16 routed experts of the DeepSeek-V3 shape, 128 rows each on average (as dsv3), for
    # per-kernel counter captures: about 3 GB on the device with gradients, every weight
    # tensor larger than L2
    "dsv3_e16_r128": Workload("dsv3_e16_r128", T=256, H=7168, E=16, k=8, I=2048, S=1, Is=2048,
                              score_fn=1, n_group=8, topk_group=4, seed=8),
    # the same with 512 rows per expert (the mean load of the skewed workload): every group
    # exceeds the resident kernel's 192 rows, so the streaming weight-gradient kernel does all the work
    "dsv3_e16_r512": Workload("dsv3_e16_r512", T=1024, H=7168, E=16, k=8, I=2048, S=1, Is=2048,
                              score_fn=1, n_group=8, topk_group=4, seed=10),
    # the MXFP8 forward of the same shape with 256 rows per routed expert (as dsv3_mxfp8)
    "dsv3_mxfp8_e16": Workload("dsv3_mxfp8_e16", T=512, H=7168, E=16, k=8, I=2048, S=1, Is=2048,
                               score_fn=1, n_group=8, topk_group=4, mxfp8=True, backward=False, seed=9),
}


def scaled(wl: Workload, **changes) -> Workload:
    """A copy of a workload with some shapes changed (for reduced-size tests)."""
    return dataclasses.replace(wl, **changes)


def _gen(device, seed: int, name: str, attempt: int = 0) -> torch.Generator:
    g = torch.Generator(device=device)
    key = zlib.crc32(f"{name}/{attempt}".encode())
    g.manual_seed((seed * 1_000_003 + key) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def _normal_bf16(shape, std, device, gen, chunk_rows=None):
    """N(0, std) drawn in fp32 and rounded to bf16, optionally per leading index."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    if chunk_rows is None or len(shape) == 1:
        out.copy_(torch.randn(shape, generator=gen, device=device).mul_(std))
        return out
    for i in range(shape[0]):
        out[i].copy_(torch.randn(shape[1:], generator=gen, device=device).mul_(std))
    return out


def draw_x(wl: Workload, device="cpu", attempt: int = 0) -> torch.Tensor:
    return _normal_bf16((wl.T, wl.H), 1.0, device, _gen(device, wl.seed, "x", attempt))


def draw_dy(wl: Workload, device="cpu") -> torch.Tensor:
    return _normal_bf16((wl.T, wl.H), 1.0, device, _gen(device, wl.seed, "dy"))


def draw_params(wl: Workload, device="cpu") -> dict:
    """Router and expert parameters of a workload."""
    p = {}
    p["router_w"] = (torch.randn((wl.E, wl.H), generator=_gen(device, wl.seed, "router_w"),
                                 device=device) / math.sqrt(wl.H)).contiguous()
    if wl.score_fn == 1:
        p["e_bias"] = 0.01 * torch.randn(wl.E, generator=_gen(device, wl.seed, "e_bias"),
                                         device=device)
    else:
        p["e_bias"] = None
    if wl.zipf > 0:
        pi = torch.randperm(wl.E, generator=_gen("cpu", wl.seed, "zipf_perm"))
        p["logit_bias"] = (-wl.zipf * torch.log((pi + 1).double())).float().to(device)
    else:
        p["logit_bias"] = None
    chunk = wl.E * wl.H * wl.I > (1 << 26)
    p["w_gate_up"] = _normal_bf16((wl.E, 2 * wl.I, wl.H), 0.02, device,
                                  _gen(device, wl.seed, "w_gate_up"), chunk)
    p["w_down"] = _normal_bf16((wl.E, wl.H, wl.I), 0.02, device,
                               _gen(device, wl.seed, "w_down"), chunk)
    if wl.S:
        p["ws_gate_up"] = _normal_bf16((wl.S, 2 * wl.Is, wl.H), 0.02, device,
                                       _gen(device, wl.seed, "ws_gate_up"), chunk)
        p["ws_down"] = _normal_bf16((wl.S, wl.H, wl.Is), 0.02, device,
                                    _gen(device, wl.seed, "ws_down"), chunk)
    else:
        p["ws_gate_up"] = p["ws_down"] = None
    return p


def bf16_bits(t: torch.Tensor):
    """numpy uint16 view of a bf16 tensor's bit patterns (copied to the host)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view("uint16")
