"""The C-ABI library loads on a CPU-only host and exports every declared entry point."""
import ctypes
import os
import re

import pytest

from mixture_experts_layer_persistent_b200 import abi, build, make_cfg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "mok.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(moe_\w+)\s*\(", text, flags=re.M)))


def test_library_builds_and_exports_every_symbol():
    build.build()
    lib = ctypes.CDLL(abi.LIB_PATH)
    names = _declared()
    assert "moe_fwd" in names and "moe_bwd" in names and len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n


def test_workspace_sizes_and_argument_checks():
    c = make_cfg(4096, 7168, 256, 2048, 8, 1, 2048, 1, 8, 4)
    ctx, fwd, bwd = abi.moe_workspace_size(c)
    T, H, I, kk = 4096, 7168, 2048, 9
    R = T * kk
    # ctx holds at least g,u, h, w*h and the per-slot rows
    assert ctx >= R * 2 * I * 2 + 2 * R * I * 2 + T * kk * H * 4
    assert fwd >= R * I * 2 + T * kk * H * 4 and fwd < ctx
    assert bwd >= R * 2 * I * 2 + T * kk * H * 4
    bad = [make_cfg(64, 200, 8, 128, 2), make_cfg(64, 256, 8, 100, 2), make_cfg(64, 256, 8, 128, 9),
           make_cfg(64, 256, 300, 128, 2), make_cfg(0, 256, 8, 128, 2),
           make_cfg(64, 256, 8, 128, 2, score_fn=1, n_group=3, topk_group=1)]
    for c in bad:
        with pytest.raises(abi.MokError) as ei:
            abi.moe_workspace_size(c)
        assert ei.value.code == abi.MOK_ERR_INVALID
    with pytest.raises(abi.MokError) as ei:
        abi.moe_workspace_size(make_cfg(64, 256, 8, 128, 2, n_shared=1, I_shared=256))
    assert ei.value.code == abi.MOK_ERR_UNSUPPORTED
    assert abi.moe_strerror(abi.MOK_ERR_WORKSPACE).startswith("ctx or scratch")


def test_calls_fail_loudly_without_a_device():
    import torch
    if torch.cuda.is_available():
        pytest.skip("needs a host without a usable GPU")
    c = make_cfg(64, 256, 8, 128, 2)
    p = abi.moe_params()
    with pytest.raises(abi.MokError):
        abi.moe_fwd(c, 16, p, 16, None, None, 0, 0, 16, 1 << 30, None)


def test_mxfp8_backward_argument_checks():
    """moe_bwd with MOK_DTYPE_MXFP8 refuses, before touching any device, a call
    without the transposed weight copies (MOK_ERR_INVALID) and an I that is not a
    multiple of 256 (MOK_ERR_UNSUPPORTED).  The pointers are never dereferenced."""
    fake = 1 << 20                                    # aligned, never read
    g = abi.moe_grads(fake, fake, fake, fake, None, None)

    def params(with_t):
        p = abi.moe_params(router_w=fake, w_gate_up=fake, w_down=fake, s_gate_up=fake, s_down=fake)
        if with_t:
            p.wt_gate_up = p.wt_down = p.st_gate_up = p.st_down = fake
        return p

    c = make_cfg(64, 256, 8, 256, 2, dtype=abi.MOK_DTYPE_MXFP8)
    with pytest.raises(abi.MokError) as ei:
        abi.moe_bwd(c, fake, fake, params(False), fake, 1 << 30, g, fake, 1 << 30, None)
    assert ei.value.code == abi.MOK_ERR_INVALID
    c = make_cfg(64, 256, 8, 384, 2, dtype=abi.MOK_DTYPE_MXFP8)
    with pytest.raises(abi.MokError) as ei:
        abi.moe_bwd(c, fake, fake, params(True), fake, 1 << 30, g, fake, 1 << 30, None)
    assert ei.value.code == abi.MOK_ERR_UNSUPPORTED
    with pytest.raises(abi.MokError) as ei:      # the one-pass quantiser's shape rule
        abi.moe_quantize_mxfp8_weights_both(fake, 2, 256, 384, fake, fake, fake, fake, None)
    assert ei.value.code == abi.MOK_ERR_INVALID


def test_pipelined_host_step_argument_checks():
    """moe_step_host_async refuses missing host buffers (MOK_ERR_INVALID) and a scratch
    buffer smaller than moe_host_scratch_size(cfg, 3) (MOK_ERR_WORKSPACE) before it
    touches a device; the pipelined scratch holds two x and two dx slots more than
    moe_step_host's.  The pointers are never dereferenced."""
    c = make_cfg(64, 256, 8, 128, 2)
    io = 64 * 256 * 2
    n2, n3 = abi.moe_host_scratch_size(c, 2), abi.moe_host_scratch_size(c, 3)
    assert n3 - n2 == 2 * ((io + 255) // 256 * 256)
    p, g = abi.moe_params(), abi.moe_grads()
    args = dict(x_host=16, x_next_host=None, dy_host=16, y_host=16, dx_host=16)
    for missing in ("x_host", "dy_host", "y_host", "dx_host"):
        a = dict(args, **{missing: None})
        with pytest.raises(abi.MokError) as ei:
            abi.moe_step_host_async(c, a["x_host"], a["x_next_host"], a["dy_host"], p, a["y_host"], a["dx_host"], 16, 0,
                                    g, 16, n3, None)
        assert ei.value.code == abi.MOK_ERR_INVALID, missing
    with pytest.raises(abi.MokError) as ei:
        abi.moe_step_host_async(c, 16, None, 16, p, 16, 16, 16, 0, g, 16, n3 - 1, None)
    assert ei.value.code == abi.MOK_ERR_WORKSPACE


def test_expert_parallel_sizes_and_argument_checks():
    """moe_ep_size gives the per-rank state (the forward scratch: routing record and
    slot rows) and a receive scratch sized for the largest share a rank can get
    (world T min(k, E/world) expert rows plus the shared rows, world T pulled token
    rows); the EP calls refuse
    bad ranks, an E that world does not divide, MXFP8, row codes past 24 bits, NULL
    or short buffers -- all before touching a device (no pointer is dereferenced)."""
    T, H, E, I, k, W = 512, 7168, 256, 2048, 8, 8
    c = make_cfg(T, H, E, I, k, 1, I, 1, 8, 4)
    state, scratch, bwd = abi.moe_ep_size(c, W)
    _, scratch_t, _ = abi.moe_ep_size(c, W, True)
    assert state == abi.moe_workspace_size(c)[1]
    rr = W * T * min(k, E // W)          # expert rows: one per (token, slot) routed here
    rows = rr + T
    pulled = T + W * T                    # token rows: the own ones, then one per (rank, token) routed here
    assert scratch >= pulled * H * 2 + rows * I * 2 + rows * 12
    # training adds g/u, w h, the pulled dy rows, dGU and the slot-gradient partials
    assert scratch_t >= scratch + rows * (2 * I + I + 2 * I) * 2 + pulled * H * 2 + rr * (I // 128) * 4
    # the token side of the backward: dX slot rows and the slot-gradient partials others push
    assert bwd >= T * 9 * H * 4 + T * k * (I // 128) * 4
    # E/world < k: a token puts at most E/world of its k slots on one rank
    c2 = make_cfg(200, 256, 8, 128, 2)
    _, s8, _ = abi.moe_ep_size(c2, 8)
    _, s1, _ = abi.moe_ep_size(c2, 1)
    assert s8 >= (200 + 8 * 200) * 256 * 2 + 8 * 200 * 128 * 2 and s1 >= (200 + 200) * 256 * 2 + 400 * 128 * 2
    for world, cfg, code in ((0, c, abi.MOK_ERR_INVALID), (9, c, abi.MOK_ERR_INVALID),
                             (3, make_cfg(64, 256, 8, 128, 2), abi.MOK_ERR_INVALID),
                             (2, make_cfg(1 << 21, 256, 8, 128, 8), abi.MOK_ERR_INVALID)):
        with pytest.raises(abi.MokError) as ei:
            abi.moe_ep_size(cfg, world)
        assert ei.value.code == code, (world, code)
    # MXFP8: the forward without saved state only
    mxc = make_cfg(64, 256, 8, 128, 2, dtype=abi.MOK_DTYPE_MXFP8)
    mst, msc, _ = abi.moe_ep_size(mxc, 2)
    assert msc >= (64 + 2 * 64) * (256 + 8) + (2 * 64 * 2) * (128 + 4)
    with pytest.raises(abi.MokError) as ei:      # MXFP8 training needs I % 256 == 0
        abi.moe_ep_size(mxc, 2, True)
    assert ei.value.code == abi.MOK_ERR_UNSUPPORTED
    mxt = make_cfg(64, 256, 8, 256, 2, dtype=abi.MOK_DTYPE_MXFP8)
    _, msct, mbb = abi.moe_ep_size(mxt, 2, True)
    pm = abi.moe_params(router_w=16, w_gate_up=16, w_down=16)      # MXFP8 without weight scales
    with pytest.raises(abi.MokError) as ei:
        abi.moe_ep_experts(mxc, 2, 0, 0, [16, 16], [16, 16], pm, 16, msc, None)
    assert ei.value.code == abi.MOK_ERR_INVALID
    with pytest.raises(abi.MokError) as ei:
        abi.moe_ep_experts(mxc, 2, 0, 1, [16, 16], [16, 16], pm, 16, msc, None)
    assert ei.value.code == abi.MOK_ERR_UNSUPPORTED
    pms = abi.moe_params(router_w=16, w_gate_up=16, w_down=16, s_gate_up=16, s_down=16)   # no transposed copies
    with pytest.raises(abi.MokError) as ei:
        abi.moe_ep_bwd_experts(mxt, 2, 0, [16, 16], [16, 16], pms, abi.moe_grads(dx=16, dw_gate_up=16, dw_down=16,
                                                                                 drouter_w=16), 16, msct, None)
    assert ei.value.code == abi.MOK_ERR_INVALID
    small = make_cfg(64, 256, 8, 128, 2)
    st, sc, bb = abi.moe_ep_size(small, 2)
    _, sct, _ = abi.moe_ep_size(small, 2, True)
    p = abi.moe_params(router_w=16, w_gate_up=16, w_down=16)
    for rank in (-1, 2):
        with pytest.raises(abi.MokError) as ei:
            abi.moe_ep_route(small, 2, rank, 16, p, 16, st, None)
        assert ei.value.code == abi.MOK_ERR_INVALID
    with pytest.raises(abi.MokError) as ei:
        abi.moe_ep_route(small, 2, 0, 16, p, 16, st - 1, None)
    assert ei.value.code == abi.MOK_ERR_WORKSPACE
    with pytest.raises(abi.MokError) as ei:
        abi.moe_ep_route(small, 2, 0, None, p, 16, st, None)
    assert ei.value.code == abi.MOK_ERR_INVALID
    with pytest.raises(abi.MokError) as ei:
        abi.moe_ep_experts(small, 2, 0, 0, [16, 16], [16, 16], p, 16, sc - 1, None)
    assert ei.value.code == abi.MOK_ERR_WORKSPACE
    with pytest.raises(abi.MokError) as ei:
        abi.moe_ep_experts(small, 2, 0, 0, [16, None], [16, 16], p, 16, sc, None)
    assert ei.value.code == abi.MOK_ERR_INVALID
    with pytest.raises(abi.MokError) as ei:      # a training forward needs the larger scratch
        abi.moe_ep_experts(small, 2, 0, 1, [16, 16], [16, 16], p, 16, sct - 1, None)
    assert ei.value.code == abi.MOK_ERR_WORKSPACE
    g = abi.moe_grads(dx=16, dw_gate_up=16, dw_down=16, drouter_w=16)
    with pytest.raises(abi.MokError) as ei:
        abi.moe_ep_bwd_experts(small, 2, 0, [16, 16], [16, 16], p, g, 16, sct - 1, None)
    assert ei.value.code == abi.MOK_ERR_WORKSPACE
    with pytest.raises(abi.MokError) as ei:
        abi.moe_ep_bwd_experts(small, 2, 1, [16, None], [16, 16], p, g, 16, sct, None)
    assert ei.value.code == abi.MOK_ERR_INVALID
    with pytest.raises(abi.MokError) as ei:
        abi.moe_ep_bwd_combine(small, 2, 0, 16, p, 16, 16, bb - 1, g, None)
    assert ei.value.code == abi.MOK_ERR_WORKSPACE
    with pytest.raises(abi.MokError) as ei:
        abi.moe_ep_bwd_combine(small, 2, 0, 16, p, 16, 16, bb, abi.moe_grads(dx=16), None)
    assert ei.value.code == abi.MOK_ERR_INVALID
    with pytest.raises(abi.MokError) as ei:
        abi.moe_ep_combine(small, 2, 0, 16, None, None)
    assert ei.value.code == abi.MOK_ERR_INVALID
    with pytest.raises(abi.MokError) as ei:
        abi.moe_ep_ipc_handle(None)
    assert ei.value.code == abi.MOK_ERR_INVALID
    with pytest.raises(ValueError):
        abi.moe_ep_ipc_open(b"short", 0)
