"""CPU oracle (fp64, plain C) for the group-scale search path -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg may import this package.  The product path (the CUDA library and
its Python binding) never loads it.

This module is argument marshalling around ``tq_oracle.c``: numpy arrays in,
numpy arrays out.  Every function of the method lives in the C file, which
cites the pages it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tq_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile tq_oracle.c with gcc (no fast-math, no FMA contraction)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i64, i32, f64, f32 = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_float
        sig = {
            "orc_imatrix": (None, [P, i64, i64, i64, P]),
            "orc_hessian": (None, [P, i64, i64, i64, P]),
            "orc_e4m3_rne": (i32, [f32]),
            "orc_lloyd_max_g32": (None, [P, i64, i64, i64, i64, i64, P, i64, i32, P, P, P, P, P]),
            "orc_lloyd_max_assign": (None, [P, i64, i64, i64, i64, i64, P, P, P]),
            "orc_pack_lm2": (None, [P, i64, i64, P]),
            "orc_dequant_lm2": (None, [P, i64, i64, P, P, P]),
            "orc_fp8_scale": (f32, [i32, f64, f64, i32, f32]),
            "orc_search_fp8": (None, [P, i64, i64, i64, i64, i64, P, i64, i32, f64, f64, P, P, P, P, P]),
            "orc_dequant_fp8": (None, [P, i64, i64, P, P]),
            "orc_hessian_entry": (f64, [P, i64, i64, i64, i64]),
            "orc_proxy_error_full": (None, [P, P, i64, i64, P, P, P]),
            "orc_gptq_sweep": (None, [P, i64, i64, i32, i32, P, P, P, i64, P, P]),
            "orc_nvfp4_quant_act": (None, [P, i64, i64, P, P, P]),
            "orc_gemm_nvfp4": (None, [P, P, f32, i64, P, P, f32, i64, i64, P]),
            "orc_sym_stage1_ratio": (f32, [i32, f64, f64, i32]),
            "orc_sym_stage2_ratio": (f32, [i32, i32, f64, f64, i32, i32]),
            "orc_sym_loss": (f64, [P, P, i32, f32, P]),
            "orc_search_sym_group": (i32, [P, P, i32, i32, i32, f64, f64, P, P, P]),
            "orc_asym_scale_factor": (f32, [i32, f64, f64, i32]),
            "orc_asym_zero": (i32, [i32, i32]),
            "orc_asym_loss": (f64, [P, P, i32, f32, i32, P]),
            "orc_search_asym_group": (i32, [P, P, i32, i32, i32, f64, f64, P, P, P, P]),
            "orc_e4m3_decode": (f64, [i32]),
            "orc_e2m1_rne_mag": (i32, [f32]),
            "orc_nvfp4_global": (f32, [P, i64]),
            "orc_nvfp4_window": (None, [f32, f32, i32, P]),
            "orc_nvfp4_loss": (f64, [P, P, i32, f32, P]),
            "orc_search_nvfp4_block": (i32, [P, P, i32, f32, i32, P, P]),
            "orc_search_sym_int3": (None, [P, i64, i64, i64, i64, i64, P, i64, i32, i32, f64, f64,
                                           P, P, P, P]),
            "orc_search_asym_int4": (None, [P, i64, i64, i64, i64, i64, P, i64, i32, i32, f64, f64,
                                            P, P, P, P, P, i32]),
            "orc_search_nvfp4": (None, [P, i64, i64, i64, i64, i64, P, i64, P, i32, P, P, P, P]),
            "orc_rtn_int3": (None, [P, i64, i64, P, P]),
            "orc_rtn_int4": (None, [P, i64, i64, P, P, P, i32]),
            "orc_rtn_nvfp4": (None, [P, i64, i64, i64, P, P, P]),
            "orc_pack_int3": (None, [P, i64, i64, P]),
            "orc_unpack_int3": (None, [P, i64, i64, P]),
            "orc_pack_nibbles": (None, [P, i64, i64, i32, P, P]),
            "orc_unpack_nibbles": (None, [P, i64, i64, i32, P]),
            "orc_dequant_int3": (None, [P, i64, i64, P, P]),
            "orc_dequant_int4": (None, [P, i64, i64, P, P, P, i32]),
            "orc_dequant_nvfp4": (None, [P, i64, i64, i64, P, P, P]),
            "orc_proxy_error": (None, [P, P, i64, i64, P, P, P]),
            "orc_rowwise_int4": (None, [P, i64, i64, P]),
            "orc_num_threads": (i32, []),
            "orc_loss_given_int3": (None, [P, i64, i64, i64, i64, i64, P, i64, P, P]),
            "orc_loss_given_int4": (None, [P, i64, i64, i64, i64, i64, P, i64, P, P, P, i32]),
            "orc_loss_given_nvfp4": (None, [P, i64, i64, i64, i64, i64, P, i64, P, P, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


# ---------------------------------------------------------------- helpers

def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(a) -> np.ndarray:
    a = _to_numpy(a)
    return np.ascontiguousarray(a, dtype=np.float32)


def _to_numpy(a):
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return a.detach().to("cpu", torch.float32).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(a)


# Default grids (the workloads' settings): symmetric stage 1 = 32 magnitudes of
# [0.5, 1.2] x maxabs/4 with both signs, stage 2 = 32 refinements; asymmetric =
# 64 scales x 32 zero-points; NVFP4 = 16 E4M3 codes.
SYM = dict(n1=32, n2=32, lo=0.5, hi=1.2)
ASYM = dict(ns=64, nz=32, lo=0.5, hi=1.2)
FP4_WINDOW = 16


# ---------------------------------------------------------------- imatrix

def imatrix(X) -> np.ndarray:
    """[T, I] (or [n, T, I]) activations -> fp64 per-column mean of squares."""
    X = _f32(X)
    if X.ndim == 3:
        return np.stack([imatrix(x) for x in X])
    T, I = X.shape
    m = np.empty(I, dtype=np.float64)
    lib().orc_imatrix(_p(X), T, I, I, _p(m))
    return m


def hessian(X) -> np.ndarray:
    """[T, I] activations -> fp64 H = X^T X (both triangles)."""
    X = _f32(X)
    T, I = X.shape
    H = np.empty((I, I), dtype=np.float64)
    lib().orc_hessian(_p(X), T, I, I, _p(H))
    return H


def hessian_entry(X, i: int, j: int) -> float:
    X = _f32(X)
    T, I = X.shape
    return lib().orc_hessian_entry(_p(X), T, I, int(i), int(j))


def proxy_error_full(W, What, H) -> Tuple[float, float]:
    """(num, den) for one O x I matrix with a full Hessian: tr(E H E^T), tr(W H W^T)."""
    W = _f32(W); What = _f32(What); H = np.ascontiguousarray(H, np.float64)
    O, I = W.shape
    num = ctypes.c_double(); den = ctypes.c_double()
    lib().orc_proxy_error_full(_p(W), _p(What), O, I, _p(H), ctypes.byref(num), ctypes.byref(den))
    return num.value, den.value


def gptq_sweep(W, fmt: int, scales, zeros, U, g=None):
    """GPTQ/LDLQ column sweep of W [rows, I] (or [n, O, I], one U for all)
    with fixed group scales (and zeros): fmt 3 = int3-g64, 4 = int4 (g = 128
    by default, or 64).  U: fp32 [I, I] upper factor with H^-1 = U^T U.
    Returns (codes int8 [.., I], loss fp64 [rows])."""
    W = _f32(W)
    I = W.shape[-1]; rows = W.size // I
    g = g or (64 if fmt == 3 else 128)
    U = _f32(U)
    codes = np.empty(W.shape, np.int8)
    loss = np.empty(rows, np.float64)
    z = None if zeros is None else np.ascontiguousarray(zeros, np.uint8)
    lib().orc_gptq_sweep(_p(W), rows, I, int(fmt), int(g), _p(_f32(scales)), _p(z), _p(U), U.shape[-1],
                         _p(codes), _p(loss))
    return codes, loss


def nvfp4_quant_act(X):
    """NVFP4 activations X [rows, I] -> (global scale, E4M3 block-scale codes
    [rows, ceil(I/16)], E2M1 codes [rows, I] with the sign in bit 3)."""
    X = _f32(X)
    rows, I = X.shape
    g = ctypes.c_float()
    sc = np.empty((rows, (I + 15) // 16), np.uint8)
    c = np.empty((rows, I), np.uint8)
    lib().orc_nvfp4_quant_act(_p(X), rows, I, ctypes.byref(g), _p(sc), _p(c))
    return g.value, sc, c


def gemm_nvfp4(cw, ew, gw, cx, ex, gx):
    """W4A4 product y [B, O] (fp64) of NVFP4 weight codes cw [O, I] / block
    scales ew [O, G] / global gw and activation codes cx [B, I] / ex [B, G] / gx."""
    cw = np.ascontiguousarray(cw, np.uint8); cx = np.ascontiguousarray(cx, np.uint8)
    ew = np.ascontiguousarray(ew, np.uint8); ex = np.ascontiguousarray(ex, np.uint8)
    O, I = cw.shape
    B = cx.shape[0]
    y = np.empty((B, O), np.float64)
    lib().orc_gemm_nvfp4(_p(cw), _p(ew), float(gw), O, _p(cx), _p(ex), float(gx), B, I, _p(y))
    return y


def e4m3_rne(y: float) -> int:
    return lib().orc_e4m3_rne(float(np.float32(y)))


def fp8_scale(n: int, lo: float, hi: float, k: int, amax: float) -> float:
    return lib().orc_fp8_scale(n, lo, hi, k, float(np.float32(amax)))


def search_fp8(W, m, n=64, lo=0.5, hi=1.2, codes=True):
    """W [n_mat, O, I] (or [O, I]), m [n_mat, I] or [I] -> (scales[n_mat], idx, loss, losses[n_mat, n], codes)."""
    W = _f32(W)
    if W.ndim == 2:
        W = W[None]
    E, O, I = W.shape
    m = _f32(m)
    ms = I if m.ndim == 2 else 0
    scales = np.empty(E, np.float32)
    idx = np.empty(E, np.int32)
    loss = np.empty(E, np.float64)
    losses = np.empty((E, n), np.float64)
    c = np.empty((E, O, I), np.uint8) if codes else None
    lib().orc_search_fp8(_p(W), E, O, I, I, O * I, _p(m), ms, n, lo, hi, _p(scales), _p(idx), _p(loss),
                         _p(losses), _p(c))
    return scales, idx, loss, losses, c


LM_START = (-0.75, -0.25, 0.25, 0.75)


def lloyd_max_g32(W, m, n_iter=16, start=LM_START, codes=True):
    """W [n_mat, O, I], m [n_mat, I] or [I] -> (codebook[4], scales[n_mat, O, G32], codes, loss, history)."""
    W = _f32(W)
    if W.ndim == 2:
        W = W[None]
    E, O, I = W.shape
    m = _f32(m)
    ms = I if m.ndim == 2 else 0
    cb = np.array(start, np.float32)
    sc = np.empty((E, O, (I + 31) // 32), np.float32)
    c = np.empty((E, O, I), np.uint8) if codes else None
    loss = ctypes.c_double()
    hist = np.empty(n_iter + 1, np.float64)
    lib().orc_lloyd_max_g32(_p(W), E, O, I, I, O * I, _p(m), ms, n_iter, _p(cb), _p(sc), _p(c),
                            ctypes.byref(loss), _p(hist))
    return cb, sc, c, loss.value, hist


def lloyd_max_assign(W, codebook):
    W = _f32(W)
    if W.ndim == 2:
        W = W[None]
    E, O, I = W.shape
    sc = np.empty((E, O, (I + 31) // 32), np.float32)
    c = np.empty((E, O, I), np.uint8)
    lib().orc_lloyd_max_assign(_p(W), E, O, I, I, O * I, _p(_f32(codebook)), _p(sc), _p(c))
    return sc, c


def pack_lm2(codes) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8); I = codes.shape[-1]; rows = codes.size // I
    out = np.empty(rows * ((I + 31) // 32) * 8, np.uint8)
    lib().orc_pack_lm2(_p(codes), rows, I, _p(out))
    return out


def dequant_lm2(codes, scales, codebook) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8); I = codes.shape[-1]; rows = codes.size // I
    out = np.empty(codes.shape, np.float32)
    lib().orc_dequant_lm2(_p(codes), rows, I, _p(_f32(scales)), _p(_f32(codebook)), _p(out))
    return out


def dequant_fp8(c, scales) -> np.ndarray:
    c = np.ascontiguousarray(c, np.uint8)
    if c.ndim == 2:
        c = c[None]
    E = c.shape[0]
    out = np.empty(c.shape, np.float32)
    lib().orc_dequant_fp8(_p(c), E, c[0].size, _p(_f32(scales)), _p(out))
    return out


# ---------------------------------------------------------------- searches

def search_sym_int3(W, m, n1=32, n2=32, lo=0.5, hi=1.2, codes=True):
    """W [n_mat, O, I], m [n_mat, I] or [I] -> (scales, idx, loss, codes)."""
    W = _f32(W)
    if W.ndim == 2:
        W = W[None]
    E, O, I = W.shape
    m = _f32(m)
    ms = I if m.ndim == 2 else 0
    G = (I + 63) // 64
    scales = np.empty((E, O, G), np.float32)
    idx = np.empty((E, O, G), np.int32)
    loss = np.empty((E, O, G), np.float64)
    v = np.empty((E, O, I), np.int8) if codes else None
    lib().orc_search_sym_int3(_p(W), E, O, I, I, O * I, _p(m), ms, n1, n2, lo, hi,
                              _p(scales), _p(idx), _p(loss), _p(v))
    return scales, idx, loss, v


def search_asym_int4(W, m, ns=64, nz=32, lo=0.5, hi=1.2, codes=True, g=128):
    W = _f32(W)
    if W.ndim == 2:
        W = W[None]
    E, O, I = W.shape
    m = _f32(m)
    ms = I if m.ndim == 2 else 0
    G = (I + g - 1) // g
    scales = np.empty((E, O, G), np.float32)
    zeros = np.empty((E, O, G), np.uint8)
    idx = np.empty((E, O, G), np.int32)
    loss = np.empty((E, O, G), np.float64)
    q = np.empty((E, O, I), np.uint8) if codes else None
    lib().orc_search_asym_int4(_p(W), E, O, I, I, O * I, _p(m), ms, ns, nz, lo, hi,
                               _p(scales), _p(zeros), _p(idx), _p(loss), _p(q), g)
    return scales, zeros, idx, loss, q


def nvfp4_global(W) -> np.ndarray:
    W = _f32(W)
    if W.ndim == 2:
        W = W[None]
    return np.array([lib().orc_nvfp4_global(_p(np.ascontiguousarray(w)), w.size) for w in W],
                    dtype=np.float32)


def search_nvfp4(W, m, gscale=None, window=16, codes=True):
    W = _f32(W)
    if W.ndim == 2:
        W = W[None]
    E, O, I = W.shape
    m = _f32(m)
    ms = I if m.ndim == 2 else 0
    if gscale is None:
        gscale = nvfp4_global(W)
    gscale = _f32(gscale).reshape(E)
    G = (I + 15) // 16
    sc = np.empty((E, O, G), np.uint8)
    idx = np.empty((E, O, G), np.int32)
    loss = np.empty((E, O, G), np.float64)
    c = np.empty((E, O, I), np.uint8) if codes else None
    lib().orc_search_nvfp4(_p(W), E, O, I, I, O * I, _p(m), ms, _p(gscale), window,
                           _p(sc), _p(idx), _p(loss), _p(c))
    return gscale, sc, idx, loss, c


# ---------------------------------------------------------------- per-group

def sym_group(w, m, n1=32, n2=32, lo=0.5, hi=1.2):
    w, m = _f32(w).ravel(), _f32(m).ravel()
    s = ctypes.c_float(); L = ctypes.c_double(); v = np.empty(w.size, np.int8)
    c = lib().orc_search_sym_group(_p(w), _p(m), w.size, n1, n2, lo, hi,
                                   ctypes.byref(s), ctypes.byref(L), _p(v))
    return c, s.value, L.value, v


def sym_loss(w, m, s) -> float:
    w, m = _f32(w).ravel(), _f32(m).ravel()
    return lib().orc_sym_loss(_p(w), _p(m), w.size, float(np.float32(s)), None)


def asym_group(w, m, ns=64, nz=32, lo=0.5, hi=1.2):
    w, m = _f32(w).ravel(), _f32(m).ravel()
    s = ctypes.c_float(); z = ctypes.c_uint8(); L = ctypes.c_double(); q = np.empty(w.size, np.uint8)
    c = lib().orc_search_asym_group(_p(w), _p(m), w.size, ns, nz, lo, hi, ctypes.byref(s),
                                    ctypes.byref(z), ctypes.byref(L), _p(q))
    return c, s.value, z.value, L.value, q


def asym_loss(w, m, s, z) -> float:
    w, m = _f32(w).ravel(), _f32(m).ravel()
    return lib().orc_asym_loss(_p(w), _p(m), w.size, float(np.float32(s)), int(z), None)


def nvfp4_block(w, m, g, window=16):
    w, m = _f32(w).ravel(), _f32(m).ravel()
    L = ctypes.c_double(); c = np.empty(w.size, np.uint8)
    e = lib().orc_search_nvfp4_block(_p(w), _p(m), w.size, float(np.float32(g)), window,
                                     ctypes.byref(L), _p(c))
    return e, L.value, c


def nvfp4_loss(w, m, S) -> float:
    w, m = _f32(w).ravel(), _f32(m).ravel()
    return lib().orc_nvfp4_loss(_p(w), _p(m), w.size, float(np.float32(S)), None)


def sym_stage1_ratio(k, n1=32, lo=0.5, hi=1.2) -> float:
    return lib().orc_sym_stage1_ratio(n1, lo, hi, k)


def sym_stage2_ratio(kstar, i, n1=32, n2=32, lo=0.5, hi=1.2) -> float:
    return lib().orc_sym_stage2_ratio(n1, n2, lo, hi, kstar, i)


def asym_scale_factor(k, ns=64, lo=0.5, hi=1.2) -> float:
    return lib().orc_asym_scale_factor(ns, lo, hi, k)


def asym_zero(i, nz=32) -> int:
    return lib().orc_asym_zero(nz, i)


def e4m3_decode(code: int) -> float:
    return lib().orc_e4m3_decode(int(code))


def e2m1_rne_mag(y: float) -> int:
    return lib().orc_e2m1_rne_mag(float(np.float32(y)))


def nvfp4_window(a: float, g: float, window=16):
    """Window codes for block amax a under global scale g."""
    out = np.empty(window, np.int32)
    lib().orc_nvfp4_window(float(np.float32(a)), float(np.float32(g)), window, _p(out))
    return out


# ---------------------------------------------------------------- RTN / pack / dequant

def rtn_int3(W, scales):
    W = _f32(W); I = W.shape[-1]; rows = W.size // I
    v = np.empty(W.shape, np.int8)
    lib().orc_rtn_int3(_p(W), rows, I, _p(_f32(scales)), _p(v))
    return v


def rtn_int4(W, scales, zeros, g=128):
    W = _f32(W); I = W.shape[-1]; rows = W.size // I
    q = np.empty(W.shape, np.uint8)
    lib().orc_rtn_int4(_p(W), rows, I, _p(_f32(scales)), _p(np.ascontiguousarray(zeros, np.uint8)), _p(q), g)
    return q


def rtn_nvfp4(W, scale_codes, gscale):
    W = _f32(W)
    if W.ndim == 2:
        W = W[None]
    E, O, I = W.shape
    c = np.empty(W.shape, np.uint8)
    lib().orc_rtn_nvfp4(_p(W), E * O, O, I, _p(np.ascontiguousarray(scale_codes, np.uint8)),
                        _p(_f32(gscale)), _p(c))
    return c


def pack_int3(v) -> np.ndarray:
    v = np.ascontiguousarray(v, np.int8); I = v.shape[-1]; rows = v.size // I
    G = (I + 63) // 64
    out = np.empty(rows * G * 24, np.uint8)
    lib().orc_pack_int3(_p(v), rows, I, _p(out))
    return out


def unpack_int3(packed, rows, I) -> np.ndarray:
    packed = np.ascontiguousarray(packed, np.uint8)
    v = np.empty((rows, I), np.int8)
    lib().orc_unpack_int3(_p(packed), rows, I, _p(v))
    return v


def pack_nibbles(c, g, pad_per_group=None) -> np.ndarray:
    c = np.ascontiguousarray(c, np.uint8); I = c.shape[-1]; rows = c.size // I
    G = (I + g - 1) // g
    out = np.empty(rows * G * (g // 2), np.uint8)
    pad = None if pad_per_group is None else np.ascontiguousarray(pad_per_group, np.uint8)
    lib().orc_pack_nibbles(_p(c), rows, I, g, _p(pad), _p(out))
    return out


def unpack_nibbles(packed, rows, I, g) -> np.ndarray:
    packed = np.ascontiguousarray(packed, np.uint8)
    c = np.empty((rows, I), np.uint8)
    lib().orc_unpack_nibbles(_p(packed), rows, I, g, _p(c))
    return c


def dequant_int3(v, scales) -> np.ndarray:
    v = np.ascontiguousarray(v, np.int8); I = v.shape[-1]; rows = v.size // I
    out = np.empty(v.shape, np.float32)
    lib().orc_dequant_int3(_p(v), rows, I, _p(_f32(scales)), _p(out))
    return out


def dequant_int4(q, scales, zeros, g=128) -> np.ndarray:
    q = np.ascontiguousarray(q, np.uint8); I = q.shape[-1]; rows = q.size // I
    out = np.empty(q.shape, np.float32)
    lib().orc_dequant_int4(_p(q), rows, I, _p(_f32(scales)), _p(np.ascontiguousarray(zeros, np.uint8)), _p(out), g)
    return out


def dequant_nvfp4(c, scale_codes, gscale) -> np.ndarray:
    c = np.ascontiguousarray(c, np.uint8)
    if c.ndim == 2:
        c = c[None]
    E, O, I = c.shape
    out = np.empty(c.shape, np.float32)
    lib().orc_dequant_nvfp4(_p(c), E * O, O, I, _p(np.ascontiguousarray(scale_codes, np.uint8)),
                            _p(_f32(gscale)), _p(out))
    return out


def proxy_error(W, What, m) -> Tuple[float, float]:
    """(num, den) for one O x I matrix: tr(E H E^T), tr(W H W^T), H = diag(m)."""
    W, What, m = _f32(W), _f32(What), _f32(m)
    I = W.shape[-1]; O = W.size // I
    a = ctypes.c_double(); b = ctypes.c_double()
    lib().orc_proxy_error(_p(W), _p(What), O, I, _p(m), ctypes.byref(a), ctypes.byref(b))
    return a.value, b.value


def rowwise_int4(W) -> np.ndarray:
    W = _f32(W); I = W.shape[-1]; rows = W.size // I
    out = np.empty(W.shape, np.float32)
    lib().orc_rowwise_int4(_p(W), rows, I, _p(out))
    return out


def _batch(W, m):
    W = _f32(W)
    if W.ndim == 2:
        W = W[None]
    m = _f32(m)
    E, O, I = W.shape
    return W, m, E, O, I, (I if m.ndim == 2 else 0)


def loss_given_int3(W, m, scales) -> np.ndarray:
    """fp64 loss of given int3 scales for every group of W [n_mat, O, I]."""
    W, m, E, O, I, ms = _batch(W, m)
    out = np.empty((E, O, (I + 63) // 64), np.float64)
    lib().orc_loss_given_int3(_p(W), E, O, I, I, O * I, _p(m), ms, _p(_f32(scales)), _p(out))
    return out


def loss_given_int4(W, m, scales, zeros, g=128) -> np.ndarray:
    W, m, E, O, I, ms = _batch(W, m)
    out = np.empty((E, O, (I + g - 1) // g), np.float64)
    lib().orc_loss_given_int4(_p(W), E, O, I, I, O * I, _p(m), ms, _p(_f32(scales)),
                              _p(np.ascontiguousarray(zeros, np.uint8)), _p(out), g)
    return out


def loss_given_nvfp4(W, m, scale_codes, gscale) -> np.ndarray:
    W, m, E, O, I, ms = _batch(W, m)
    out = np.empty((E, O, (I + 15) // 16), np.float64)
    lib().orc_loss_given_nvfp4(_p(W), E, O, I, I, O * I, _p(m), ms,
                               _p(np.ascontiguousarray(scale_codes, np.uint8)), _p(_f32(gscale)), _p(out))
    return out


def num_threads() -> int:
    return lib().orc_num_threads()
