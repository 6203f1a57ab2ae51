"""Shared helpers of the tests: seeded cases, oracle set-up, tolerance checks."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from mixture_experts_layer_persistent_b200 import synth

RTOL = 1e-2
ATOL = 1e-2


def bits_to_bf16(bits: np.ndarray, device="cpu") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def oracle_layer(wl, params, x_bits, dy_bits=None, mx=False, pure=False, weights=None):
    """Oracle layer of a workload; params are torch tensors (any device)."""
    L = oracle.Layer(wl.T, wl.H, wl.E, wl.k, wl.I, S=wl.S, Is=wl.Is, score_fn=wl.score_fn,
                     n_group=wl.n_group, topk_group=wl.topk_group, routed_scale=wl.routed_scale, mx=mx,
                     pure=pure)
    f32 = lambda t: None if t is None else t.detach().float().cpu().numpy()
    w = weights or {}
    L.set(x=x_bits, Wr=f32(params["router_w"]), bias=f32(params.get("e_bias")),
          lbias=f32(params.get("logit_bias")),
          Wgu=w.get("Wgu", None) if "Wgu" in w else synth.bf16_bits(params["w_gate_up"]),
          Wdn=w.get("Wdn", None) if "Wdn" in w else synth.bf16_bits(params["w_down"]),
          Wgu_s=w.get("Wgu_s") if "Wgu_s" in w else (synth.bf16_bits(params["ws_gate_up"]) if wl.S else None),
          Wdn_s=w.get("Wdn_s") if "Wdn_s" in w else (synth.bf16_bits(params["ws_down"]) if wl.S else None),
          dy=dy_bits)
    return L


def make_case(wl, device="cpu", gen_device=None, mx=False):
    """Seeded inputs of a workload with top-k margins >= 1e-3 (x rows resampled).

    Returns dict: params (on `device`), x, dy (on `device`), x_bits, dy_bits,
    oracle layer L, idx, w (oracle routing), resamples.
    """
    gd = gen_device or device
    params = synth.draw_params(wl, gd)
    x_bits = synth.bf16_bits(synth.draw_x(wl, gd))
    dy_bits = synth.bf16_bits(synth.draw_dy(wl, gd)) if wl.backward else None
    L = oracle_layer(wl, params, x_bits, dy_bits, mx=mx)
    x_bits, idx, w, counts = oracle.margin_reject(
        L, lambda a: synth.bf16_bits(synth.draw_x(wl, gd, attempt=a)))
    params = {k: (v.to(device) if v is not None else None) for k, v in params.items()}
    return {
        "params": params,
        "x": bits_to_bf16(x_bits, device),
        "dy": bits_to_bf16(dy_bits, device) if dy_bits is not None else None,
        "x_bits": x_bits, "dy_bits": dy_bits, "L": L, "idx": idx, "w": w, "resamples": counts,
    }


def assert_close(got, want, what, rtol=RTOL, atol=ATOL):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    err = np.abs(got - want)
    bound = atol + rtol * np.abs(want)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())}/{bad.size} elements out of tolerance; worst at "
                             f"{i}: got {got[i]!r} want {want[i]!r} (|err| {err[i]:.3g} > {bound[i]:.3g})")


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def packed_scale_offsets(rows, kb32, total_rows):
    """Byte offsets [len(rows), kb32] of the scales of `rows` in the packed weight-scale
    layout of include/mok.h (moe_quantize_mxfp8_weights): (K/128) x (total_rows/128)
    tiles of 512 bytes; row r = 128 rb + 32 q + i, block j = 4 kb + s at byte
    (kb * total_rows/128 + rb) * 512 + 16 i + 4 q + s."""
    r = np.asarray(rows, dtype=np.int64)[:, None]
    j = np.arange(kb32, dtype=np.int64)[None, :]
    return ((j // 4) * (total_rows // 128) + r // 128) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (j % 4)


# ---------------------------------------------------------------- MXFP8 h check
# Relative bound on |h_gpu - h_oracle| / |h| before quantisation: the GPU forms
# g and u as fp32 tensor-core sums of K = H e4m3 products (K <= 7168) and
# silu with expf; the oracle in fp64.  2^-12 is a loose bound on that
# difference (fp32 accumulation over 7168 terms stays near 2^-17 relative).
MX_H_REL = 2.0 ** -12


def _e4m3_table():
    import oracle
    vals = np.array([oracle.e4m3_value(c) for c in range(256)])
    finite = np.sort(np.unique(vals[np.isfinite(vals)]))
    return vals, finite


def check_mx_h(layer, L, idx, tokens, inv_perm):
    """Compare the e4m3 codes and ue8m0 scales of h that the MXFP8 gate/up
    epilogue stored with the oracle's quantisation of its own h (h_mx) for the
    given tokens' slots.  A scale may differ by one only where the oracle's block
    amax lies within MX_H_REL of a scale boundary 448 * 2^e; a code may differ
    only to the adjacent e4m3 value, and only where h * 2^-e lies within
    MX_H_REL of the midpoint between the two.  Returns counts (blocks, scale
    differences, codes, code differences) and raises on any other difference."""
    from mixture_experts_layer_persistent_b200 import abi
    c = layer.cfg
    T, k, S, I = c.T, c.top_k, c.n_shared, c.I
    R = T * (k + S)
    hq = layer.saved(abi.MOK_SAVED_HQ).view(R, I)
    hs = layer.saved(abi.MOK_SAVED_HS).view(R, I // 32)
    tokens = np.asarray(tokens, np.int32)
    rows = np.zeros((len(tokens), k + S), np.int64)
    for a, t in enumerate(tokens):
        rows[a, :k] = inv_perm[t * k:(t + 1) * k]
        rows[a, k:] = T * k + np.arange(S) * T + t
    ridx = torch.from_numpy(rows.ravel()).to(hq.device)
    gq = hq[ridx].cpu().numpy().reshape(len(tokens), k + S, I)
    gs = hs[ridx].cpu().numpy().reshape(len(tokens), k + S, I // 32).astype(np.int64)
    hraw, oq, os_ = L.h_mx(idx, tokens)
    os_ = os_.astype(np.int64)
    vals, grid = _e4m3_table()
    # scales
    amax = np.abs(hraw[..., :I]).reshape(len(tokens), k + S, I // 32, 32).max(-1)
    eo = os_ - 127
    near = np.minimum(np.abs(amax / (448.0 * 2.0 ** (eo - 1)) - 1), np.abs(amax / (448.0 * 2.0 ** eo) - 1))
    sdiff = gs != os_
    bad_s = sdiff & ~((np.abs(gs - os_) == 1) & (near <= MX_H_REL))
    assert not bad_s.any(), f"{int(bad_s.sum())} h scale bytes differ away from a scale boundary"
    # codes of the blocks whose scales agree
    same = np.repeat(~sdiff, 32, axis=-1)
    vg, vo = vals[gq], vals[oq]
    v = hraw[..., :I] * 2.0 ** -np.repeat(eo, 32, axis=-1)
    cdiff = same & (gq != oq) & ~((vg == 0) & (vo == 0))
    pos_g, pos_o = np.searchsorted(grid, vg), np.searchsorted(grid, vo)
    adjacent = np.abs(pos_g - pos_o) == 1
    mid = 0.5 * (vg + vo)
    near_mid = np.abs(v - mid) <= MX_H_REL * np.abs(v) + 2.0 ** -40
    bad_c = cdiff & ~(adjacent & near_mid)
    assert not bad_c.any(), (f"{int(bad_c.sum())} h codes differ away from a rounding midpoint; first at "
                             f"{np.argwhere(bad_c)[0]}")
    return {"blocks": int(sdiff.size), "scale_diffs": int(sdiff.sum()), "codes": int(same.sum()),
            "code_diffs": int(cdiff.sum())}


def rel_rms_per_token(got, want):
    """(pooled relative RMS, largest per-token relative RMS) over rows of y."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    pooled = float(np.sqrt(np.mean((got - want) ** 2)) / np.sqrt(np.mean(want ** 2)))
    per = np.sqrt(np.mean((got - want) ** 2, axis=-1)) / np.sqrt(np.mean(want ** 2, axis=-1))
    return pooled, float(per.max())
