"""ctypes binding of libmok.so -- argument marshalling only.

Every name here mirrors an entry point of include/mok.h.  Device pointers
are passed as integers (e.g. ``tensor.data_ptr()``), streams as
``torch.cuda.Stream.cuda_stream`` integers.  Nothing in this module computes
any part of the layer, and there is no fallback: if the library cannot be
loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmok.so")

MOK_OK = 0
MOK_ERR_INVALID = -1
MOK_ERR_DEVICE = -2
MOK_ERR_WORKSPACE = -3
MOK_ERR_LAUNCH = -4
MOK_ERR_UNSUPPORTED = -5
MOK_STATUS_TIMEOUT = 1
MOK_STATUS_BAD_INDEX = 2
MOK_SCORE_SOFTMAX = 0
MOK_SCORE_SIGMOID = 1
MOK_DTYPE_BF16 = 0
MOK_DTYPE_MXFP8 = 1
MOK_FWD_PHASES = 5
MOK_BWD_PHASES = 8
MOK_STATIC_SCRATCH_BYTES = 32 << 20
MOK_SCHEDULE_PERSISTENT = 0
MOK_SCHEDULE_SPLIT = 1
MOK_SCHEDULE_SPLIT_PDL = 2
MOK_TRACE_POINTS = 9
MOK_EP_MAX_RANKS = 8
MOK_EP_IPC_HANDLE_BYTES = 64
MOK_SAVED_H, MOK_SAVED_HQ, MOK_SAVED_HS, MOK_SAVED_GU, MOK_SAVED_HW, MOK_SAVED_ROW_TOKEN, MOK_SAVED_ROW_W = range(7)

_i32, _f32, _vp, _sz = ctypes.c_int32, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t


class moe_cfg(ctypes.Structure):
    _fields_ = [("T", _i32), ("H", _i32), ("E", _i32), ("I", _i32), ("top_k", _i32),
                ("n_shared", _i32), ("I_shared", _i32), ("score_fn", _i32), ("n_group", _i32),
                ("topk_group", _i32), ("routed_scale", _f32), ("dtype", _i32)]


class moe_params(ctypes.Structure):
    _fields_ = [(n, _vp) for n in ("router_w", "e_bias", "logit_bias", "w_gate_up", "w_down",
                                    "s_gate_up", "s_down", "ws_gate_up", "ws_down", "ss_gate_up",
                                    "ss_down", "wt_gate_up", "wt_down", "st_gate_up", "st_down",
                                    "wst_gate_up", "wst_down", "sst_gate_up", "sst_down")]


class moe_routing(ctypes.Structure):
    _fields_ = [(n, _vp) for n in ("topk_idx", "topk_w", "counts", "offsets", "perm", "inv_perm")]


class moe_grads(ctypes.Structure):
    _fields_ = [(n, _vp) for n in ("dx", "dw_gate_up", "dw_down", "drouter_w", "dws_gate_up",
                                    "dws_down")]


class MokError(RuntimeError):
    def __init__(self, fn, code):
        detail = lib().moe_last_error().decode()
        super().__init__(f"{fn} failed: {moe_strerror(code)} ({code})" + (f": {detail}" if detail else ""))
        self.code = code


_lib = None


def lib():
    """Load libmok.so (raises if it is missing: the layer has no other implementation)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m mixture_experts_layer_persistent_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER
        L.moe_workspace_size.argtypes = [P(moe_cfg), P(_sz), P(_sz), P(_sz)]
        L.moe_fwd.argtypes = [P(moe_cfg), _vp, P(moe_params), _vp, P(moe_routing), _vp, _sz, _i32, _vp,
                              _sz, _vp]
        L.moe_bwd.argtypes = [P(moe_cfg), _vp, _vp, P(moe_params), _vp, _sz, P(moe_grads), _vp, _sz,
                              _vp]
        L.moe_host_scratch_size.argtypes = [P(moe_cfg), _i32, P(_sz)]
        L.moe_fwd_host.argtypes = [P(moe_cfg), _vp, P(moe_params), _vp, _vp, _sz, _i32, _vp, _sz, _vp]
        L.moe_bwd_host.argtypes = [P(moe_cfg), _vp, _vp, P(moe_params), _vp, _sz, _vp, P(moe_grads),
                                   _vp, _sz, _vp]
        L.moe_step_host.argtypes = [P(moe_cfg), _vp, _vp, P(moe_params), _vp, _vp, _vp, _sz, P(moe_grads), _vp,
                                    _sz, _vp]
        L.moe_step_host_async.argtypes = [P(moe_cfg), _vp, _vp, _vp, P(moe_params), _vp, _vp, _vp, _sz,
                                          P(moe_grads), _vp, _sz, _vp]
        L.moe_step_host_sync.argtypes = [_vp]
        L.moe_quantize_mxfp8.argtypes = [_vp, ctypes.c_int64, ctypes.c_int64, _vp, _vp, _vp]
        L.moe_quantize_mxfp8_weights.argtypes = [_vp, ctypes.c_int64, ctypes.c_int64, _vp, _vp, _vp]
        L.moe_quantize_mxfp8_weights_t.argtypes = [_vp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, _vp, _vp,
                                                   _vp]
        L.moe_quantize_mxfp8_weights_both.argtypes = [_vp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, _vp, _vp,
                                                      _vp, _vp, _vp]
        L.moe_status.argtypes = [_vp, P(_i32)]
        L.moe_trace_events.argtypes = [P(_vp), ctypes.c_int, P(_vp), ctypes.c_int]
        L.moe_fwd_static.argtypes = [P(moe_cfg), _vp, P(moe_params), _vp, _vp]
        L.moe_test_drop_signal.argtypes = [ctypes.c_int]
        L.moe_launch_count.argtypes = [P(_i32)]
        L.moe_saved_tensor.argtypes = [P(moe_cfg), _i32, _i32, P(_sz), P(_sz)]
        L.moe_set_schedule.argtypes = [ctypes.c_int]
        L.moe_get_schedule.argtypes = [P(_i32)]
        L.moe_trace_device.argtypes = [_vp, _sz, _vp, _sz]
        L.moe_ep_size.argtypes = [P(moe_cfg), _i32, _i32, P(_sz), P(_sz), P(_sz)]
        L.moe_ep_route.argtypes = [P(moe_cfg), _i32, _i32, _vp, P(moe_params), _vp, _sz, _vp]
        L.moe_ep_experts.argtypes = [P(moe_cfg), _i32, _i32, _i32, P(_vp), P(_vp), P(moe_params), _vp, _sz, _vp]
        L.moe_ep_combine.argtypes = [P(moe_cfg), _i32, _i32, _vp, _vp, _vp]
        L.moe_ep_bwd_experts.argtypes = [P(moe_cfg), _i32, _i32, P(_vp), P(_vp), P(moe_params), P(moe_grads), _vp,
                                         _sz, _vp]
        L.moe_ep_bwd_combine.argtypes = [P(moe_cfg), _i32, _i32, _vp, P(moe_params), _vp, _vp, _sz, P(moe_grads),
                                         _vp]
        L.moe_ep_ipc_handle.argtypes = [_vp, _vp, P(_sz)]
        L.moe_ep_ipc_open.argtypes = [_vp, _sz, P(_vp)]
        L.moe_ep_ipc_close.argtypes = [_vp, _sz]
        L.moe_strerror.argtypes = [ctypes.c_int]
        L.moe_strerror.restype = ctypes.c_char_p
        L.moe_last_error.argtypes = []
        L.moe_last_error.restype = ctypes.c_char_p
        for name in ("moe_workspace_size", "moe_fwd", "moe_bwd", "moe_host_scratch_size",
                     "moe_fwd_host", "moe_bwd_host", "moe_step_host", "moe_step_host_async", "moe_step_host_sync",
                     "moe_quantize_mxfp8", "moe_quantize_mxfp8_weights",
                     "moe_quantize_mxfp8_weights_t", "moe_quantize_mxfp8_weights_both", "moe_status",
                     "moe_trace_events", "moe_fwd_static", "moe_test_drop_signal", "moe_saved_tensor",
                     "moe_set_schedule", "moe_get_schedule", "moe_trace_device", "moe_ep_size", "moe_ep_route",
                     "moe_ep_experts", "moe_ep_combine", "moe_ep_bwd_experts", "moe_ep_bwd_combine",
                     "moe_ep_ipc_handle", "moe_ep_ipc_open",
                     "moe_ep_ipc_close"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(fn, rc):
    if rc != MOK_OK:
        raise MokError(fn, rc)


def moe_strerror(code: int) -> str:
    return lib().moe_strerror(int(code)).decode()


def moe_workspace_size(cfg: moe_cfg):
    c, f, b = _sz(), _sz(), _sz()
    _check("moe_workspace_size", lib().moe_workspace_size(ctypes.byref(cfg), ctypes.byref(c),
                                                          ctypes.byref(f), ctypes.byref(b)))
    return c.value, f.value, b.value


def moe_set_schedule(schedule: int) -> None:
    _check("moe_set_schedule", lib().moe_set_schedule(int(schedule)))


def moe_get_schedule() -> int:
    v = _i32()
    _check("moe_get_schedule", lib().moe_get_schedule(ctypes.byref(v)))
    return v.value


def moe_trace_device(buf, nbytes: int, bwd_buf=None, bwd_nbytes: int = 0) -> None:
    _check("moe_trace_device", lib().moe_trace_device(buf, int(nbytes), bwd_buf, int(bwd_nbytes)))


def moe_saved_tensor(cfg: moe_cfg, save_for_backward: bool, which: int):
    """(byte offset, bytes) of a saved tensor inside the forward's buffer."""
    off, n = _sz(), _sz()
    _check("moe_saved_tensor", lib().moe_saved_tensor(ctypes.byref(cfg), int(save_for_backward), int(which),
                                                      ctypes.byref(off), ctypes.byref(n)))
    return off.value, n.value


def moe_host_scratch_size(cfg: moe_cfg, backward) -> int:
    """backward: False (moe_fwd_host), True (moe_bwd_host), 2 (moe_step_host) or 3 (moe_step_host_async)."""
    n = _sz()
    _check("moe_host_scratch_size", lib().moe_host_scratch_size(ctypes.byref(cfg), int(backward),
                                                                ctypes.byref(n)))
    return n.value


def moe_fwd(cfg, x, params, y, routing, ctx, ctx_bytes, save_for_backward, scratch, scratch_bytes,
            stream):
    rc = lib().moe_fwd(ctypes.byref(cfg), x, ctypes.byref(params), y,
                       ctypes.byref(routing) if routing is not None else None, ctx, ctx_bytes,
                       int(save_for_backward), scratch, scratch_bytes, stream)
    _check("moe_fwd", rc)


def moe_bwd(cfg, x, dy, params, ctx, ctx_bytes, grads, scratch, scratch_bytes, stream):
    rc = lib().moe_bwd(ctypes.byref(cfg), x, dy, ctypes.byref(params), ctx, ctx_bytes,
                       ctypes.byref(grads), scratch, scratch_bytes, stream)
    _check("moe_bwd", rc)


def moe_fwd_host(cfg, x_host, params, y_host, ctx, ctx_bytes, save_for_backward, scratch,
                 scratch_bytes, stream):
    rc = lib().moe_fwd_host(ctypes.byref(cfg), x_host, ctypes.byref(params), y_host, ctx, ctx_bytes,
                            int(save_for_backward), scratch, scratch_bytes, stream)
    _check("moe_fwd_host", rc)


def moe_bwd_host(cfg, x_host, dy_host, params, ctx, ctx_bytes, dx_host, grads, scratch,
                 scratch_bytes, stream):
    rc = lib().moe_bwd_host(ctypes.byref(cfg), x_host, dy_host, ctypes.byref(params), ctx,
                            ctx_bytes, dx_host, ctypes.byref(grads), scratch, scratch_bytes, stream)
    _check("moe_bwd_host", rc)


def moe_step_host(cfg, x_host, dy_host, params, y_host, dx_host, ctx, ctx_bytes, grads, scratch, scratch_bytes,
                  stream):
    _check("moe_step_host", lib().moe_step_host(ctypes.byref(cfg), x_host, dy_host, ctypes.byref(params), y_host,
                                                dx_host, ctx, ctx_bytes, ctypes.byref(grads), scratch, scratch_bytes,
                                                stream))


def moe_step_host_async(cfg, x_host, x_next_host, dy_host, params, y_host, dx_host, ctx, ctx_bytes, grads, scratch,
                        scratch_bytes, stream):
    _check("moe_step_host_async", lib().moe_step_host_async(ctypes.byref(cfg), x_host, x_next_host, dy_host,
                                                            ctypes.byref(params), y_host, dx_host, ctx, ctx_bytes,
                                                            ctypes.byref(grads), scratch, scratch_bytes, stream))


def moe_step_host_sync(stream):
    _check("moe_step_host_sync", lib().moe_step_host_sync(stream))


def moe_quantize_mxfp8(src, rows, K, q, scales, stream):
    _check("moe_quantize_mxfp8", lib().moe_quantize_mxfp8(src, rows, K, q, scales, stream))


def moe_quantize_mxfp8_weights(src, rows, K, q, scales, stream):
    _check("moe_quantize_mxfp8_weights", lib().moe_quantize_mxfp8_weights(src, rows, K, q, scales, stream))


def moe_quantize_mxfp8_weights_both(src, batch, R, C, q, scales, qt, scales_t, stream):
    _check("moe_quantize_mxfp8_weights_both",
           lib().moe_quantize_mxfp8_weights_both(src, batch, R, C, q, scales, qt, scales_t, stream))


def moe_quantize_mxfp8_weights_t(src, batch, R, C, q, scales, stream):
    _check("moe_quantize_mxfp8_weights_t", lib().moe_quantize_mxfp8_weights_t(src, batch, R, C, q, scales, stream))


def moe_status(stream) -> int:
    v = _i32()
    _check("moe_status", lib().moe_status(stream, ctypes.byref(v)))
    return v.value


def moe_trace_events(fwd_events, bwd_events):
    """fwd_events / bwd_events: lists of raw cudaEvent_t handles (ints), or None to stop."""
    fa = (_vp * len(fwd_events))(*fwd_events) if fwd_events else None
    ba = (_vp * len(bwd_events))(*bwd_events) if bwd_events else None
    _check("moe_trace_events", lib().moe_trace_events(fa, len(fwd_events or ()), ba,
                                                      len(bwd_events or ())))


def moe_fwd_static(cfg, x, params, y, stream):
    """Forward pass using the library's static scratch (no workspace argument)."""
    _check("moe_fwd_static", lib().moe_fwd_static(ctypes.byref(cfg), x, ctypes.byref(params), y, stream))


def moe_launch_count() -> int:
    """Kernels launched by the last forward or backward called on this thread."""
    n = _i32(0)
    _check("moe_launch_count", lib().moe_launch_count(ctypes.byref(n)))
    return n.value


def moe_test_drop_signal(enable: bool):
    """Fault injection for the bounded waits (see include/mok.h)."""
    _check("moe_test_drop_signal", lib().moe_test_drop_signal(int(enable)))


def moe_ep_size(cfg: moe_cfg, world: int, training: bool = False):
    """(state_bytes, scratch_bytes, bwd_bytes) of one rank of an expert-parallel layer."""
    a, b, c = _sz(), _sz(), _sz()
    _check("moe_ep_size", lib().moe_ep_size(ctypes.byref(cfg), int(world), int(training), ctypes.byref(a),
                                            ctypes.byref(b), ctypes.byref(c)))
    return a.value, b.value, c.value


def moe_ep_route(cfg, world, rank, x, params, state, state_bytes, stream):
    _check("moe_ep_route", lib().moe_ep_route(ctypes.byref(cfg), int(world), int(rank), x, ctypes.byref(params),
                                              state, state_bytes, stream))


def moe_ep_experts(cfg, world, rank, training, x_ranks, state_ranks, params, scratch, scratch_bytes, stream):
    xs = (_vp * len(x_ranks))(*x_ranks)
    ss = (_vp * len(state_ranks))(*state_ranks)
    _check("moe_ep_experts", lib().moe_ep_experts(ctypes.byref(cfg), int(world), int(rank), int(training), xs, ss,
                                                  ctypes.byref(params), scratch, scratch_bytes, stream))


def moe_ep_bwd_experts(cfg, world, rank, dy_ranks, bwd_ranks, params, grads, scratch, scratch_bytes, stream):
    ds = (_vp * len(dy_ranks))(*dy_ranks)
    bs = (_vp * len(bwd_ranks))(*bwd_ranks)
    _check("moe_ep_bwd_experts", lib().moe_ep_bwd_experts(ctypes.byref(cfg), int(world), int(rank), ds, bs,
                                                          ctypes.byref(params), ctypes.byref(grads), scratch,
                                                          scratch_bytes, stream))


def moe_ep_bwd_combine(cfg, world, rank, x, params, state, bwd, bwd_bytes, grads, stream):
    _check("moe_ep_bwd_combine", lib().moe_ep_bwd_combine(ctypes.byref(cfg), int(world), int(rank), x,
                                                          ctypes.byref(params), state, bwd, bwd_bytes,
                                                          ctypes.byref(grads), stream))


def moe_ep_combine(cfg, world, rank, state, y, stream):
    _check("moe_ep_combine", lib().moe_ep_combine(ctypes.byref(cfg), int(world), int(rank), state, y, stream))


def moe_ep_ipc_handle(dev_ptr):
    """(handle bytes, offset) of the device allocation holding dev_ptr."""
    h = ctypes.create_string_buffer(MOK_EP_IPC_HANDLE_BYTES)
    off = _sz()
    _check("moe_ep_ipc_handle", lib().moe_ep_ipc_handle(dev_ptr, h, ctypes.byref(off)))
    return h.raw, off.value


def moe_ep_ipc_open(handle: bytes, offset: int) -> int:
    if len(handle) != MOK_EP_IPC_HANDLE_BYTES:
        raise ValueError("an IPC handle is %d bytes" % MOK_EP_IPC_HANDLE_BYTES)
    p = _vp()
    _check("moe_ep_ipc_open", lib().moe_ep_ipc_open(handle, offset, ctypes.byref(p)))
    return p.value


def moe_ep_ipc_close(dev_ptr: int, offset: int) -> None:
    _check("moe_ep_ipc_close", lib().moe_ep_ipc_close(dev_ptr, offset))
