"""fp64 CPU oracle of the mixture-of-experts layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding) never imports, links or runs anything here, and this package never
imports the product.

``oracle.c`` holds all arithmetic; this module only builds it, marshals numpy
arrays into it and, for input generation, applies the top-k margin rule (resample
a token's x row until its selection scores are separated by at least 1e-3).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

BF16, F32, F64 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (plain gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O3", "-fopenmp", "-shared", "-fPIC", "-Wall",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class Cfg(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("H", ctypes.c_int), ("E", ctypes.c_int), ("k", ctypes.c_int),
                ("I", ctypes.c_int), ("S", ctypes.c_int), ("Is", ctypes.c_int),
                ("score_fn", ctypes.c_int), ("n_group", ctypes.c_int), ("topk_group", ctypes.c_int),
                ("routed_scale", ctypes.c_double), ("mx", ctypes.c_int), ("pure", ctypes.c_int),
                ("act_kind", ctypes.c_int), ("w_kind", ctypes.c_int), ("r_kind", ctypes.c_int)]


_INPUTS = ("x", "Wr", "bias", "lbias", "Wgu", "Wdn", "Wgu_s", "Wdn_s", "dy",
           "Wgu_b", "Wdn_b", "Wgu_sb", "Wdn_sb")


class Inputs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _INPUTS]


_lib = None

# Path of another build of the oracle to load instead of liboracle.so.  The
# planted-mistake tests set it to run the pins against a deliberately broken copy.
LIB_ENV = "MOK_ORACLE_LIB"


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(os.environ.get(LIB_ENV) or build())
        d, p, i, i64 = ctypes.c_double, ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        _lib.orc_round_bf16.restype = d
        _lib.orc_round_bf16.argtypes = [d]
        _lib.orc_bf16_bits.restype = ctypes.c_uint16
        _lib.orc_bf16_bits.argtypes = [d]
        _lib.orc_round_e4m3.restype = d
        _lib.orc_round_e4m3.argtypes = [d]
        _lib.orc_e4m3_bits.restype = ctypes.c_uint8
        _lib.orc_e4m3_bits.argtypes = [d]
        _lib.orc_e4m3_value.restype = d
        _lib.orc_e4m3_value.argtypes = [ctypes.c_uint8]
        _lib.orc_mx_scale_exp.restype = i
        _lib.orc_mx_scale_exp.argtypes = [d]
        _lib.orc_mx_quantize.argtypes = [p, i64, i64, p, p]
        _lib.orc_mx_fakequant_bf16.argtypes = [p, i64, i64]
        _lib.orc_mx_fakequant_cols_bf16.argtypes = [p, i64, i64, i64]
        cp = ctypes.POINTER(Cfg)
        ip = ctypes.POINTER(Inputs)
        _lib.orc_route.argtypes = [cp, p, p, p, p, p, i, p, p, p, p, p]
        _lib.orc_dispatch.argtypes = [cp, p, p, p, p, p]
        _lib.orc_fwd_tokens.argtypes = [cp, ip, p, p, p, i, p, p, p]
        _lib.orc_h_mx.argtypes = [cp, ip, p, p, i, p, p, p]
        _lib.orc_bwd_tokens.argtypes = [cp, ip, p, p, p, i, p, p, p]
        _lib.orc_drouter.argtypes = [cp, ip, p, p, p, i, p]
        _lib.orc_dw_entries.argtypes = [cp, ip, p, p, i, i, i, p, p, i, p]
        _lib.orc_dw_full.argtypes = [cp, ip, p, p, i, i, p, p]
        _lib.orc_num_threads.restype = i
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _kind(a):
    if a is None:
        return BF16
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.float64:
        return F64
    raise TypeError(a.dtype)


class Layer:
    """Holds one layer's shapes and inputs (numpy, C-contiguous).

    x, dy, expert weights: uint16 bf16 bit patterns (or float64 for finite
    differences); router_w, e_bias, logit_bias: float32 (or float64).
    MXFP8 backward: Wgu_b, Wdn_b (Wgu_sb, Wdn_sb) are the weight copies
    fake-quantised along the data-gradient contraction axis
    (mx_fakequant_cols_bf16), needed by bwd, drouter and the dw functions.
    """

    def __init__(self, T, H, E, k, I, S=0, Is=0, score_fn=0, n_group=1, topk_group=1,
                 routed_scale=1.0, mx=False, pure=False):
        self.cfg = Cfg(T, H, E, k, I, S, Is, score_fn, n_group, topk_group, routed_scale,
                       int(mx), int(pure), BF16, BF16, F32)
        self.arrays = {}
        self.inp = Inputs()

    def set(self, **arrays):
        for name, a in arrays.items():
            if a is not None:
                a = np.ascontiguousarray(a)
            self.arrays[name] = a
        x = self.arrays.get("x")
        self.cfg.act_kind = _kind(x)
        self.cfg.w_kind = _kind(self.arrays.get("Wgu"))
        self.cfg.r_kind = _kind(self.arrays.get("Wr"))
        for name in _INPUTS:
            setattr(self.inp, name, _ptr(self.arrays.get(name)))
        return self

    # -- routing -----------------------------------------------------------
    def route(self, tokens=None, want_logits=False, into=None):
        """Route all tokens (or the listed ones, updating ``into`` = (idx, w, gap))."""
        c = self.cfg
        if into is None:
            idx = np.zeros((c.T, c.k), np.int32)
            w = np.zeros((c.T, c.k), np.float64)
            gap = np.full(c.T, np.inf)
        else:
            idx, w, gap = into
        lg = np.zeros((c.T, c.E)) if want_logits else None
        pr = np.zeros((c.T, c.E)) if want_logits else None
        tk = None if tokens is None else np.ascontiguousarray(tokens, np.int32)
        a = self.arrays
        rc = lib().orc_route(ctypes.byref(c), _ptr(a["x"]), _ptr(a["Wr"]), _ptr(a.get("bias")),
                             _ptr(a.get("lbias")), _ptr(tk), 0 if tk is None else len(tk),
                             _ptr(idx), _ptr(w), _ptr(gap), _ptr(lg), _ptr(pr))
        assert rc == 0
        if want_logits:
            return idx, w, gap, lg, pr
        return idx, w, gap

    def dispatch(self, idx):
        c = self.cfg
        counts = np.zeros(c.E, np.int32)
        offsets = np.zeros(c.E + 1, np.int32)
        perm = np.zeros(c.T * c.k, np.int32)
        inv = np.zeros(c.T * c.k, np.int32)
        rc = lib().orc_dispatch(ctypes.byref(c), _ptr(np.ascontiguousarray(idx, np.int32)),
                                _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(inv))
        assert rc == 0
        return counts, offsets, perm, inv

    # -- forward / backward --------------------------------------------------
    def fwd(self, idx, w, tokens=None, want_slots=False):
        c = self.cfg
        tokens = np.arange(c.T, dtype=np.int32) if tokens is None else np.asarray(tokens, np.int32)
        n = len(tokens)
        kk = c.k + c.S
        y = np.zeros((n, c.H))
        O = np.zeros((n, kk, c.H)) if want_slots else None
        hm = max(c.I, c.Is)
        h = np.zeros((n, kk, hm)) if want_slots else None
        idx = np.ascontiguousarray(idx, np.int32)
        w = np.ascontiguousarray(w, np.float64)
        lib().orc_fwd_tokens(ctypes.byref(c), ctypes.byref(self.inp), _ptr(idx), _ptr(w),
                             _ptr(tokens), n, _ptr(y), _ptr(O), _ptr(h))
        return (y, O, h) if want_slots else y

    def h_mx(self, idx, tokens):
        """MXFP8 mode: (h unrounded [n, k+S, Im] fp64, e4m3 codes [n, k+S, Im] uint8,
        ue8m0 scales [n, k+S, Im/32] uint8) of the listed tokens' slots."""
        c = self.cfg
        tokens = np.ascontiguousarray(tokens, np.int32)
        n, kk, Im = len(tokens), c.k + c.S, max(c.I, c.Is)
        hraw = np.zeros((n, kk, Im))
        hq = np.zeros((n, kk, Im), np.uint8)
        hs = np.zeros((n, kk, Im // 32), np.uint8)
        rc = lib().orc_h_mx(ctypes.byref(c), ctypes.byref(self.inp),
                            _ptr(np.ascontiguousarray(idx, np.int32)), _ptr(tokens), n, _ptr(hraw),
                            _ptr(hq), _ptr(hs))
        assert rc == 0
        return hraw, hq, hs

    def bwd(self, idx, w, tokens=None):
        c = self.cfg
        tokens = np.arange(c.T, dtype=np.int32) if tokens is None else np.asarray(tokens, np.int32)
        n = len(tokens)
        dx = np.zeros((n, c.H))
        dl = np.zeros((n, c.k))
        G = np.zeros((n, c.k))
        idx = np.ascontiguousarray(idx, np.int32)
        w = np.ascontiguousarray(w, np.float64)
        rc = lib().orc_bwd_tokens(ctypes.byref(c), ctypes.byref(self.inp), _ptr(idx), _ptr(w),
                                  _ptr(tokens), n, _ptr(dx), _ptr(dl), _ptr(G))
        assert rc == 0, "MXFP8 backward needs the weight copies Wgu_b, Wdn_b (Wgu_sb, Wdn_sb)"
        return dx, dl, G

    def drouter(self, idx, w, experts):
        c = self.cfg
        experts = np.asarray(experts, np.int32)
        out = np.zeros((len(experts), c.H))
        lib().orc_drouter(ctypes.byref(c), ctypes.byref(self.inp),
                          _ptr(np.ascontiguousarray(idx, np.int32)),
                          _ptr(np.ascontiguousarray(w, np.float64)), _ptr(experts), len(experts),
                          _ptr(out))
        return out

    def dw_full(self, idx, w, group, shared=False):
        c = self.cfg
        I = c.Is if shared else c.I
        dgu = np.zeros((2 * I, c.H))
        ddn = np.zeros((c.H, I))
        rc = lib().orc_dw_full(ctypes.byref(c), ctypes.byref(self.inp),
                               _ptr(np.ascontiguousarray(idx, np.int32)),
                               _ptr(np.ascontiguousarray(w, np.float64)), group, int(shared),
                               _ptr(dgu), _ptr(ddn))
        assert rc >= 0
        return dgu, ddn

    def dw_entries(self, idx, w, group, shared, which, rows, cols):
        c = self.cfg
        rows = np.ascontiguousarray(rows, np.int32)
        cols = np.ascontiguousarray(cols, np.int32)
        out = np.zeros(len(rows))
        rc = lib().orc_dw_entries(ctypes.byref(c), ctypes.byref(self.inp),
                                  _ptr(np.ascontiguousarray(idx, np.int32)),
                                  _ptr(np.ascontiguousarray(w, np.float64)), group, int(shared), which,
                                  _ptr(rows), _ptr(cols), len(rows), _ptr(out))
        assert rc >= 0
        return out


# ---------------------------------------------------------------- scalars
def round_bf16(v: float) -> float:
    return lib().orc_round_bf16(float(v))


def round_e4m3(v: float) -> float:
    return lib().orc_round_e4m3(float(v))


def e4m3_bits(v: float) -> int:
    return lib().orc_e4m3_bits(float(v))


def e4m3_value(b: int) -> float:
    return lib().orc_e4m3_value(int(b))


def mx_scale_exp(amax: float) -> int:
    return lib().orc_mx_scale_exp(float(amax))


def mx_quantize(src_bits: np.ndarray):
    """bf16 bits [rows, K] -> (e4m3 codes uint8 [rows, K], ue8m0 uint8 [rows, K/32])."""
    src = np.ascontiguousarray(src_bits, np.uint16)
    rows, K = src.shape
    q = np.zeros((rows, K), np.uint8)
    s = np.zeros((rows, K // 32), np.uint8)
    assert lib().orc_mx_quantize(_ptr(src), rows, K, _ptr(q), _ptr(s)) == 0
    return q, s


def mx_fakequant_bf16(bits: np.ndarray) -> None:
    """In place: replace bf16 bits [rows, K] by their MXFP8-dequantised values."""
    assert bits.dtype == np.uint16 and bits.flags.c_contiguous
    K = bits.shape[-1]
    rows = bits.size // K
    assert lib().orc_mx_fakequant_bf16(_ptr(bits), rows, K) == 0


def mx_fakequant_cols_bf16(bits: np.ndarray) -> None:
    """In place: bf16 bits [..., R, C] -> MXFP8-dequantised values with blocks of 32
    consecutive rows of each column (quantisation along R)."""
    assert bits.dtype == np.uint16 and bits.flags.c_contiguous and bits.ndim >= 2
    R, C = bits.shape[-2:]
    batch = bits.size // (R * C)
    assert lib().orc_mx_fakequant_cols_bf16(_ptr(bits), batch, R, C) == 0


def num_threads() -> int:
    return lib().orc_num_threads()


# ---------------------------------------------------------------- margins
def margin_reject(layer: Layer, redraw, min_gap: float = 1e-3, max_rounds: int = 64):
    """Resample x rows whose top-k selection is not separated by min_gap.

    ``redraw(attempt)`` returns a fresh x matrix (same shape and dtype) drawn
    from the next seeded stream; rejected rows take their values from it.
    Returns (x, idx, w, resample_counts).
    """
    c = layer.cfg
    x = layer.arrays["x"].copy()
    layer.set(x=x)
    idx, w, gap = layer.route()
    counts = np.zeros(c.T, np.int32)
    bad = np.nonzero(gap < min_gap)[0]
    attempt = 0
    while len(bad) and attempt < max_rounds:
        attempt += 1
        fresh = redraw(attempt)
        x[bad] = fresh[bad]
        counts[bad] += 1
        layer.set(x=x)
        layer.route(tokens=bad, into=(idx, w, gap))
        bad = np.nonzero(gap < min_gap)[0]
    if len(bad):
        raise RuntimeError(f"margin rejection did not converge for {len(bad)} tokens")
    return x, idx, w, counts
