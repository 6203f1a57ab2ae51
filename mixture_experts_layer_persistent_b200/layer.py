"""Torch plumbing around the C ABI: device buffers, streams, pointer marshalling.

``MoELayer`` owns the ctx / scratch buffers (torch allocations on the current
CUDA device) and calls ``moe_fwd`` / ``moe_bwd`` of libmok.  All arithmetic of
the layer runs in libmok's kernels.
"""
from __future__ import annotations

import torch

from . import abi


def _ptr(t):
    return None if t is None else t.data_ptr()


def make_cfg(T, H, E, I, top_k, n_shared=0, I_shared=0, score_fn=0, n_group=1, topk_group=1,
             routed_scale=1.0, dtype=abi.MOK_DTYPE_BF16) -> abi.moe_cfg:
    return abi.moe_cfg(T, H, E, I, top_k, n_shared, I_shared if n_shared else 0, score_fn, n_group,
                       topk_group, routed_scale, dtype)


def cfg_for(wl, dtype=None) -> abi.moe_cfg:
    """C config of a synth.Workload."""
    if dtype is None:
        dtype = abi.MOK_DTYPE_MXFP8 if wl.mxfp8 else abi.MOK_DTYPE_BF16
    return make_cfg(wl.T, wl.H, wl.E, wl.I, wl.k, wl.S, wl.Is, wl.score_fn, wl.n_group,
                    wl.topk_group, wl.routed_scale, dtype)


def make_params(p: dict) -> abi.moe_params:
    """C parameter record of a dict of device tensors (missing keys: NULL)."""
    return abi.moe_params(
        _ptr(p.get("router_w")), _ptr(p.get("e_bias")), _ptr(p.get("logit_bias")),
        _ptr(p.get("w_gate_up")), _ptr(p.get("w_down")), _ptr(p.get("s_gate_up")), _ptr(p.get("s_down")),
        _ptr(p.get("ws_gate_up")), _ptr(p.get("ws_down")), _ptr(p.get("ss_gate_up")),
        _ptr(p.get("ss_down")), _ptr(p.get("wt_gate_up")), _ptr(p.get("wt_down")),
        _ptr(p.get("st_gate_up")), _ptr(p.get("st_down")), _ptr(p.get("wst_gate_up")),
        _ptr(p.get("wst_down")), _ptr(p.get("sst_gate_up")), _ptr(p.get("sst_down")))


class MoELayer:
    """One layer's parameters plus the buffers the C ABI needs.

    params: dict of device tensors (router_w, e_bias, logit_bias, w_gate_up,
    w_down, ws_gate_up, ws_down and, for MXFP8, the s_* scale tensors; the MXFP8
    backward also reads the transposed copies wt_*, st_*, wst_*, sst_* made by
    quantize_mxfp8_weights_t).
    """

    def __init__(self, cfg: abi.moe_cfg, params: dict, training: bool = True, device=None):
        self.cfg = cfg
        self.params = params
        self.device = torch.device(device or "cuda")
        self.ctx_bytes, self.fwd_bytes, self.bwd_bytes = abi.moe_workspace_size(cfg)
        self.training = training
        self.ctx = torch.empty(self.ctx_bytes if training else 0, dtype=torch.uint8, device=self.device)
        self.scratch = torch.empty(self.fwd_bytes if not training else 0, dtype=torch.uint8,
                                   device=self.device)
        self.bwd_scratch = torch.empty(self.bwd_bytes if training else 0, dtype=torch.uint8,
                                       device=self.device)
        self.cparams = make_params(params)

    def stream(self):
        return torch.cuda.current_stream(self.device).cuda_stream

    def new_routing(self):
        c = self.cfg
        d = self.device
        r = {
            "topk_idx": torch.empty((c.T, c.top_k), dtype=torch.int32, device=d),
            "topk_w": torch.empty((c.T, c.top_k), dtype=torch.float32, device=d),
            "counts": torch.empty(c.E, dtype=torch.int32, device=d),
            "offsets": torch.empty(c.E + 1, dtype=torch.int32, device=d),
            "perm": torch.empty(c.T * c.top_k, dtype=torch.int32, device=d),
            "inv_perm": torch.empty(c.T * c.top_k, dtype=torch.int32, device=d),
        }
        return r

    def forward(self, x: torch.Tensor, y: torch.Tensor = None, routing: dict = None):
        c = self.cfg
        if y is None:
            y = torch.empty((c.T, c.H), dtype=torch.bfloat16, device=self.device)
        cr = None
        if routing is not None:
            cr = abi.moe_routing(*(_ptr(routing.get(n)) for n in
                                   ("topk_idx", "topk_w", "counts", "offsets", "perm", "inv_perm")))
        if self.training:
            abi.moe_fwd(c, x.data_ptr(), self.cparams, y.data_ptr(), cr, self.ctx.data_ptr(),
                        self.ctx_bytes, 1, None, 0, self.stream())
        else:
            abi.moe_fwd(c, x.data_ptr(), self.cparams, y.data_ptr(), cr, None, 0, 0,
                        self.scratch.data_ptr(), self.fwd_bytes, self.stream())
        return y

    def new_grads(self):
        c = self.cfg
        d = self.device
        g = {
            "dx": torch.empty((c.T, c.H), dtype=torch.bfloat16, device=d),
            "dw_gate_up": torch.empty((c.E, 2 * c.I, c.H), dtype=torch.bfloat16, device=d),
            "dw_down": torch.empty((c.E, c.H, c.I), dtype=torch.bfloat16, device=d),
            "drouter_w": torch.empty((c.E, c.H), dtype=torch.float32, device=d),
            "dws_gate_up": None, "dws_down": None,
        }
        if c.n_shared:
            g["dws_gate_up"] = torch.empty((c.n_shared, 2 * c.I, c.H), dtype=torch.bfloat16, device=d)
            g["dws_down"] = torch.empty((c.n_shared, c.H, c.I), dtype=torch.bfloat16, device=d)
        return g

    def backward(self, x: torch.Tensor, dy: torch.Tensor, grads: dict = None):
        if not self.training:
            raise RuntimeError("layer was built without saved state (training=False)")
        grads = grads or self.new_grads()
        cg = abi.moe_grads(*(_ptr(grads.get(n)) for n in
                             ("dx", "dw_gate_up", "dw_down", "drouter_w", "dws_gate_up", "dws_down")))
        abi.moe_bwd(self.cfg, x.data_ptr(), dy.data_ptr(), self.cparams, self.ctx.data_ptr(),
                    self.ctx_bytes, cg, self.bwd_scratch.data_ptr(), self.bwd_bytes, self.stream())
        return grads

    def saved(self, which: int, dtype=torch.uint8) -> torch.Tensor:
        """A view of one tensor the last forward kept in this layer's buffer
        (abi.MOK_SAVED_*), flat, of the given dtype."""
        off, n = abi.moe_saved_tensor(self.cfg, self.training, which)
        buf = self.ctx if self.training else self.scratch
        return buf[off:off + n].view(dtype)

    def status(self) -> int:
        return abi.moe_status(self.stream())


def quantize_mxfp8(src: torch.Tensor):
    """bf16 [..., K] -> (e4m3 codes uint8 [..., K], ue8m0 scales uint8 [..., K/32]) via libmok."""
    K = src.shape[-1]
    rows = src.numel() // K
    q = torch.empty(src.shape, dtype=torch.uint8, device=src.device)
    s = torch.empty((*src.shape[:-1], K // 32), dtype=torch.uint8, device=src.device)
    abi.moe_quantize_mxfp8(src.data_ptr(), rows, K, q.data_ptr(), s.data_ptr(),
                           torch.cuda.current_stream(src.device).cuda_stream)
    return q, s


def quantize_mxfp8_weights(src: torch.Tensor):
    """Expert weights bf16 [..., K] -> (e4m3 codes uint8 [..., K], ue8m0 scales as a flat uint8
    tensor in the packed weight-scale layout of include/mok.h) via libmok."""
    K = src.shape[-1]
    rows = src.numel() // K
    q = torch.empty(src.shape, dtype=torch.uint8, device=src.device)
    s = torch.empty(rows * (K // 32), dtype=torch.uint8, device=src.device)
    abi.moe_quantize_mxfp8_weights(src.data_ptr(), rows, K, q.data_ptr(), s.data_ptr(),
                                   torch.cuda.current_stream(src.device).cuda_stream)
    return q, s


def quantize_mxfp8_weights_t(src: torch.Tensor):
    """Expert weights bf16 [batch, R, C] -> the MXFP8 backward's copy: e4m3 codes
    [batch, C, R] quantised along R and their scales (flat uint8, packed layout of
    the [batch*C, R] matrix) via libmok."""
    batch, R, C = src.shape
    q = torch.empty((batch, C, R), dtype=torch.uint8, device=src.device)
    s = torch.empty(batch * C * (R // 32), dtype=torch.uint8, device=src.device)
    abi.moe_quantize_mxfp8_weights_t(src.data_ptr(), batch, R, C, q.data_ptr(), s.data_ptr(),
                                     torch.cuda.current_stream(src.device).cuda_stream)
    return q, s


def quantize_mxfp8_weights_both(src: torch.Tensor, out=None):
    """Expert weights bf16 [batch, R, C] -> both MXFP8 copies from one read: (q, s) as
    quantize_mxfp8_weights and (qt, st) as quantize_mxfp8_weights_t, via libmok.
    out: optional (q, s, qt, st) tensors to write into (requantisation in place)."""
    batch, R, C = src.shape
    if out is None:
        out = (torch.empty((batch, R, C), dtype=torch.uint8, device=src.device),
               torch.empty(batch * R * (C // 32), dtype=torch.uint8, device=src.device),
               torch.empty((batch, C, R), dtype=torch.uint8, device=src.device),
               torch.empty(batch * C * (R // 32), dtype=torch.uint8, device=src.device))
    q, s, qt, st = out
    abi.moe_quantize_mxfp8_weights_both(src.data_ptr(), batch, R, C, q.data_ptr(), s.data_ptr(), qt.data_ptr(),
                                        st.data_ptr(), torch.cuda.current_stream(src.device).cuda_stream)
    return out
