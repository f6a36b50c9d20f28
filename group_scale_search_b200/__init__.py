"""Python binding of the tq C ABI (include/tq.h): group-scale search, RTN,
low-bit packing, dequantization and imatrix-weighted reconstruction error on
NVIDIA B200 (sm_100a).

This module only marshals arguments: torch tensors supply device memory and
the current CUDA stream; every step runs in the CUDA kernels of libtq.so.
There is no CPU fallback -- importing works without a GPU (so the library's
exports can be inspected), but every call needs CUDA tensors and the built
library, and raises otherwise.

Function names match the C entry points:

    tq_imatrix(X)                      -> m            (per-column mean of x^2)
    tq_amax(W)                         -> amax per matrix
    tq_search_groups(W, m, fmt)        -> SearchResult (scales, zeros, global scale,
                                                        candidate index, loss, packed)
    tq_pack(W, fmt, scales, ...)       -> packed bytes
    tq_pack_codes / tq_unpack_codes    -> packed bytes / codes
    tq_dequant(packed, fmt, ...)       -> What
    tq_proxy_error(W, packed, fmt, ..) -> (num, den) per matrix
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional, Tuple

import torch

__all__ = [
    "INT3_G64_SYM", "INT4_G128_ASYM", "INT4_G64_ASYM", "INT4_G32_ASYM", "NVFP4_G16", "SearchParams", "SearchResult", "TQError",
    "lib", "lib_path", "tq_version", "tq_group_size", "tq_num_groups", "tq_packed_bytes", "search_result_empty",
    "tq_imatrix", "tq_amax", "tq_search_groups", "tq_pack", "tq_pack_batch", "tq_pack_codes", "tq_unpack_codes",
    "tq_dequant", "tq_dequant_batch", "tq_proxy_error_batch", "proxy_batch_workspace_bytes", "MAX_BATCH", "tq_dequant_gemv", "tq_hessian", "tq_search_fp8", "tq_pack_fp8", "tq_dequant_fp8", "Fp8Result",
    "tq_lloyd_max_g32", "tq_dequant_lm2", "LloydResult", "tq_proxy_error", "tq_proxy_error_full", "tq_gptq_sweep", "tq_sync", "tq_debug_set_wait_limit", "tq_selftest_e2m1",
    "tq_quant_nvfp4_act", "Nvfp4Act", "tq_nvfp4_scales_to_mma", "tq_gemm_nvfp4", "FORMATS", "EXPORTS",
]

INT4_G128_ASYM = 4
INT4_G64_ASYM = 6
INT4_G32_ASYM = 7
INT3_G64_SYM = 5
NVFP4_G16 = 16
FORMATS = {"int3_g64_sym": INT3_G64_SYM, "int4_g128_asym": INT4_G128_ASYM, "int4_g64_asym": INT4_G64_ASYM,
           "int4_g32_asym": INT4_G32_ASYM, "nvfp4_g16": NVFP4_G16}
_GROUP = {INT3_G64_SYM: 64, INT4_G128_ASYM: 128, INT4_G64_ASYM: 64, INT4_G32_ASYM: 32, NVFP4_G16: 16}
_INT4 = (INT4_G128_ASYM, INT4_G64_ASYM, INT4_G32_ASYM)
_F32, _BF16 = 0, 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libtq.so")
_lib = None

# every symbol include/tq.h declares
EXPORTS = [
    "tq_default_params", "tq_last_error_string", "tq_version", "tq_group_size", "tq_num_groups",
    "tq_packed_bytes", "tq_imatrix_workspace_bytes", "tq_imatrix", "tq_amax", "tq_search_groups",
    "tq_pack", "tq_pack_batch", "tq_pack_codes", "tq_unpack_codes", "tq_dequant", "tq_dequant_batch",
    "tq_proxy_workspace_bytes", "tq_proxy_batch_workspace_bytes", "tq_proxy_error_batch",
    "tq_proxy_error", "tq_sync", "tq_imatrix_static_capacity", "tq_imatrix_static", "tq_selftest_e2m1",
    "tq_dequant_gemv", "tq_hessian", "tq_fp8_workspace_bytes", "tq_search_fp8", "tq_pack_fp8", "tq_dequant_fp8",
    "tq_lloyd_workspace_bytes", "tq_lloyd_max_g32", "tq_dequant_lm2", "tq_proxy_full_workspace_bytes",
    "tq_proxy_error_full", "tq_gptq_workspace_bytes", "tq_gptq_sweep", "tq_debug_set_wait_limit",
    "tq_quant_nvfp4_act", "tq_nvfp4_scales_mma_bytes", "tq_nvfp4_scales_to_mma", "tq_gemm_nvfp4",
]


class TQError(RuntimeError):
    """A tq_* call returned a non-zero status."""


class _Mat(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("n_mat", ctypes.c_int64), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("ld", ctypes.c_int64), ("mat_stride", ctypes.c_int64)]


class _Params(ctypes.Structure):
    _fields_ = [("sym_n1", ctypes.c_int32), ("sym_n2", ctypes.c_int32), ("sym_lo", ctypes.c_double),
                ("sym_hi", ctypes.c_double), ("asym_n_scale", ctypes.c_int32),
                ("asym_n_zero", ctypes.c_int32), ("asym_lo", ctypes.c_double),
                ("asym_hi", ctypes.c_double), ("fp4_window", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


@dataclasses.dataclass
class SearchParams:
    """Candidate grids (defaults: the workloads' 32+32 symmetric, 64x32
    asymmetric and 16-code NVFP4 grids)."""
    sym_n1: int = 32
    sym_n2: int = 32
    sym_lo: float = 0.5
    sym_hi: float = 1.2
    asym_n_scale: int = 64
    asym_n_zero: int = 32
    asym_lo: float = 0.5
    asym_hi: float = 1.2
    fp4_window: int = 16

    def _c(self) -> _Params:
        return _Params(self.sym_n1, self.sym_n2, self.sym_lo, self.sym_hi, self.asym_n_scale,
                       self.asym_n_zero, self.asym_lo, self.asym_hi, self.fp4_window, 0)


@dataclasses.dataclass
class SearchResult:
    fmt: int
    scales: torch.Tensor                  # f32 [n_mat, O, G] (int3/int4) or u8 E4M3 codes (NVFP4)
    zeros: Optional[torch.Tensor]         # u8 [n_mat, O, G] (int4)
    global_scale: Optional[torch.Tensor]  # f32 [n_mat] (NVFP4)
    cand_idx: Optional[torch.Tensor]      # int32 [n_mat, O, G]
    loss: Optional[torch.Tensor]          # f64 [n_mat, O, G]
    packed: Optional[torch.Tensor]        # u8 [n_mat * O * G * record bytes]


def lib_path() -> str:
    return _LIB_PATH


def lib():
    """The loaded libtq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"{_LIB_PATH} is missing: build it with "
                              "`python -m group_scale_search_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(_LIB_PATH)
        P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        Mp = ctypes.POINTER(_Mat)
        sig = {
            "tq_default_params": (None, [ctypes.POINTER(_Params)]),
            "tq_last_error_string": (ctypes.c_char_p, []),
            "tq_version": (ctypes.c_char_p, []),
            "tq_group_size": (i64, [i32]),
            "tq_num_groups": (i64, [i32, i64, i64]),
            "tq_packed_bytes": (sz, [i32, i64, i64]),
            "tq_imatrix_workspace_bytes": (sz, [Mp]),
            "tq_imatrix": (i32, [Mp, P, i64, ctypes.c_float, i32, P, sz, P]),
            "tq_hessian": (i32, [Mp, P, i64, i64, ctypes.c_float, i32, P]),
            "tq_fp8_workspace_bytes": (sz, [Mp]),
            "tq_lloyd_workspace_bytes": (sz, [Mp]),
            "tq_lloyd_max_g32": (i32, [Mp, P, i64, i32, P, P, P, P, P, P, sz, P]),
            "tq_dequant_lm2": (i32, [P, P, P, i64, i64, i64, P, i32, P]),
            "tq_search_fp8": (i32, [Mp, P, i64, i32, ctypes.c_double, ctypes.c_double, P, P, P, P, P, P, sz, P]),
            "tq_pack_fp8": (i32, [Mp, P, P, P]),
            "tq_dequant_fp8": (i32, [P, P, i64, i64, i64, P, i32, P]),
            "tq_amax": (i32, [Mp, P, P]),
            "tq_search_groups": (i32, [Mp, P, i64, i32, ctypes.POINTER(_Params), P, P, P, P, P, P, P]),
            "tq_pack": (i32, [Mp, i32, P, P, P, P, P]),
            "tq_pack_batch": (i32, [i32, Mp, i32, P, P, P, P, P]),
            "tq_dequant_batch": (i32, [i32, P, i32, P, P, P, P, P, P, P, i32, P]),
            "tq_proxy_batch_workspace_bytes": (sz, [i32, Mp, i32]),
            "tq_proxy_error_batch": (i32, [i32, Mp, P, i32, P, P, P, P, P, P, P, P, sz, P]),
            "tq_pack_codes": (i32, [P, i32, i64, i64, P, P, P]),
            "tq_unpack_codes": (i32, [P, i32, i64, i64, P, P]),
            "tq_dequant": (i32, [P, i32, P, P, P, i64, i64, i64, P, i32, P]),
            "tq_proxy_workspace_bytes": (sz, [Mp, i32]),
            "tq_proxy_error": (i32, [Mp, P, i32, P, P, P, P, i64, P, P, P, sz, P]),
            "tq_proxy_full_workspace_bytes": (sz, [Mp, Mp]),
            "tq_gptq_workspace_bytes": (sz, [Mp]),
            "tq_gptq_sweep": (i32, [Mp, i32, P, P, P, i64, i64, P, P, P, sz, P]),
            "tq_proxy_error_full": (i32, [Mp, Mp, P, i32, P, P, P, P, P, P, sz, P]),
            "tq_sync": (i32, [P]),
            "tq_debug_set_wait_limit": (i32, [i64]),
            "tq_quant_nvfp4_act": (i32, [Mp, P, P, P, P]),
            "tq_nvfp4_scales_mma_bytes": (sz, [i64, i64, i64]),
            "tq_nvfp4_scales_to_mma": (i32, [P, i64, i64, i64, P, P]),
            "tq_gemm_nvfp4": (i32, [P, P, P, P, P, P, i64, i64, i64, i64, P, P]),
            "tq_imatrix_static_capacity": (sz, []),
            "tq_imatrix_static": (i32, [Mp, P, i64, ctypes.c_float, i32, P]),
            "tq_selftest_e2m1": (i32, [P, P, P]),
            "tq_dequant_gemv": (i32, [P, i32, P, P, P, i64, i64, i64, P, i32, i64, i64, P, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


# ---------------------------------------------------------------- marshalling

def _check(status: int, what: str) -> None:
    if status != 0:
        msg = lib().tq_last_error_string().decode(errors="replace")
        raise TQError(f"{what} failed (status {status}): {msg}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _cuda(t: torch.Tensor, name: str) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TQError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    return t


def _mat(t: torch.Tensor, name: str) -> _Mat:
    _cuda(t, name)
    if t.dtype == torch.bfloat16:
        dt = _BF16
    elif t.dtype == torch.float32:
        dt = _F32
    else:
        raise TQError(f"{name}: dtype {t.dtype} not supported (bf16 or fp32)")
    if t.dim() == 2:
        t3 = t.unsqueeze(0)
    elif t.dim() == 3:
        t3 = t
    else:
        raise TQError(f"{name}: expected [O, I] or [n_mat, O, I]")
    if t3.stride(2) != 1:
        raise TQError(f"{name}: the last dimension must be contiguous")
    E, O, I = t3.shape
    return _Mat(t3.data_ptr(), dt, 0, E, O, I, t3.stride(1), t3.stride(0) if E > 1 else 0)


def _m_stride(m: torch.Tensor) -> int:
    return m.stride(0) if m.dim() == 2 and m.shape[0] > 1 else 0


def _check_m(m: torch.Tensor, n_mat: int, cols: int, name: str = "m", shared_ok: bool = True) -> torch.Tensor:
    """An imatrix the kernels may read or write in place: fp32 on the GPU,
    [cols] (one vector for every matrix, where allowed) or [n_mat, cols]
    ([1, cols] for one matrix), unit column stride and rows at least cols
    apart -- anything else would make a kernel touch memory outside the
    tensor, so it is refused here."""
    _cuda(m, name)
    if m.dtype != torch.float32:
        raise TQError(f"{name} must be float32, not {m.dtype}")
    if m.dim() == 1:
        if not shared_ok and n_mat > 1:
            raise TQError(f"{name} must be [n_mat={n_mat}, {cols}]")
        if m.shape[0] != cols:
            raise TQError(f"{name} has {m.shape[0]} columns, expected {cols}")
    elif m.dim() == 2:
        if m.shape[1] != cols or m.shape[0] not in ((n_mat, 1) if shared_ok else (n_mat,)):
            raise TQError(f"{name} is {tuple(m.shape)}, expected ({n_mat}, {cols})")
        if m.shape[0] > 1 and m.stride(0) < cols:
            raise TQError(f"{name}: rows overlap (stride {m.stride(0)} < {cols})")
    else:
        raise TQError(f"{name} must be [cols] or [n_mat, cols]")
    if m.stride(-1) != 1:
        raise TQError(f"{name} must have unit column stride")
    return m


def _groups(W: torch.Tensor, fmt: int):
    E, O, I = (W.unsqueeze(0) if W.dim() == 2 else W).shape
    g = _GROUP[fmt]
    return E, O, I, (I + g - 1) // g


# ---------------------------------------------------------------- API

def tq_version() -> str:
    return lib().tq_version().decode()


def tq_group_size(fmt: int) -> int:
    return int(lib().tq_group_size(fmt))


def tq_num_groups(fmt: int, rows: int, cols: int) -> int:
    return int(lib().tq_num_groups(fmt, rows, cols))


def tq_packed_bytes(fmt: int, rows: int, cols: int) -> int:
    return int(lib().tq_packed_bytes(fmt, rows, cols))


def tq_sync(stream=None) -> None:
    _check(lib().tq_sync(_stream(stream)), "tq_sync")


def tq_debug_set_wait_limit(rounds: int) -> None:
    """Testing aid: try-wait rounds after which the copy/MMA ring waits of
    later tq_hessian / tq_proxy_error_full launches give up (< 0: default)."""
    _check(lib().tq_debug_set_wait_limit(int(rounds)), "tq_debug_set_wait_limit")


def tq_selftest_e2m1(stream=None) -> Tuple[int, int]:
    """(mismatches, first failing pattern) of the GPU's E2M1 conversion
    instructions against the E2M1 round-half-to-even definition; (0,
    0xffffffff) on a conforming GPU.  Synchronises the stream."""
    n = ctypes.c_uint64(0)
    first = ctypes.c_uint32(0)
    _check(lib().tq_selftest_e2m1(ctypes.byref(n), ctypes.byref(first), _stream(stream)), "tq_selftest_e2m1")
    return int(n.value), int(first.value)


def tq_imatrix(X: torch.Tensor, m: Optional[torch.Tensor] = None, alpha: Optional[float] = None,
               accumulate: bool = False, workspace: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    """m[e, j] = alpha * sum_t X[e, t, j]^2 (alpha defaults to 1/T): the
    activation imatrix.  X: [T, I] or [n_mat, T, I] bf16/fp32 on the GPU."""
    d = _mat(X, "X")
    if alpha is None:
        alpha = 1.0 / d.rows
    if m is None:
        m = torch.zeros((d.n_mat, d.cols), dtype=torch.float32, device=X.device)
    _check_m(m, d.n_mat, d.cols, shared_ok=False)
    ws_bytes = int(lib().tq_imatrix_workspace_bytes(ctypes.byref(d)))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=X.device)
    _check(lib().tq_imatrix(ctypes.byref(d), _ptr(m), _m_stride(m) if m.dim() == 2 else 0,
                            ctypes.c_float(alpha), int(accumulate), _ptr(workspace),
                            workspace.numel(), _stream(stream)), "tq_imatrix")
    return m


def tq_hessian(X: torch.Tensor, out: Optional[torch.Tensor] = None, alpha: float = 1.0,
               accumulate: bool = False, stream=None) -> torch.Tensor:
    """H[e] = alpha * X[e]^T X[e] (+ H[e] when accumulate), fp32, on the tensor
    cores.  X: [T, I] or [n_mat, T, I] bf16 on the GPU; returns [I, I] or
    [n_mat, I, I] (both triangles, exactly symmetric)."""
    d = _mat(X, "X")
    shape = (d.cols, d.cols) if X.dim() == 2 else (d.n_mat, d.cols, d.cols)
    if out is None:
        out = (torch.zeros if accumulate else torch.empty)(shape, dtype=torch.float32, device=X.device)
    _cuda(out, "out")
    if out.dtype != torch.float32 or tuple(out.shape) != shape or out.stride(-1) != 1:
        raise ValueError(f"out must be float32 {shape} with unit column stride")
    ldh = out.stride(-2)
    hms = out.stride(0) if out.dim() == 3 else 0
    _check(lib().tq_hessian(ctypes.byref(d), _ptr(out), ldh, hms, ctypes.c_float(alpha), int(accumulate),
                            _stream(stream)), "tq_hessian")
    return out


@dataclasses.dataclass
class Fp8Result:
    scales: torch.Tensor               # f32 [n_mat]
    cand_idx: Optional[torch.Tensor]   # i32 [n_mat]
    loss: Optional[torch.Tensor]       # f64 [n_mat]
    losses: Optional[torch.Tensor]     # f64 [n_mat, n_cand]
    packed: Optional[torch.Tensor]     # u8 [n_mat, O, I] E4M3 codes


def tq_search_fp8(W: torch.Tensor, m: torch.Tensor, n_cand: int = 64, lo: float = 0.5, hi: float = 1.2,
                  pack: bool = True, out: Optional[Fp8Result] = None, workspace: Optional[torch.Tensor] = None,
                  stream=None) -> Fp8Result:
    """FP8 (E4M3) with one scale per matrix, the scale searched over n_cand
    candidates fl32(r amax / 448) by the imatrix-weighted squared error; with
    pack=True the E4M3 codes of the chosen scale are written too."""
    d = _mat(W, "W")
    _check_m(m, d.n_mat, d.cols)
    E, O, I = d.n_mat, d.rows, d.cols
    dev = W.device
    if out is None:
        out = Fp8Result(scales=torch.empty(E, dtype=torch.float32, device=dev),
                        cand_idx=torch.empty(E, dtype=torch.int32, device=dev),
                        loss=torch.empty(E, dtype=torch.float64, device=dev),
                        losses=torch.empty((E, n_cand), dtype=torch.float64, device=dev),
                        packed=torch.empty((E, O, I), dtype=torch.uint8, device=dev) if pack else None)
    ws = int(lib().tq_fp8_workspace_bytes(ctypes.byref(d)))
    if workspace is None:
        workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=dev)
    _check(lib().tq_search_fp8(ctypes.byref(d), _ptr(m), _m_stride(m), n_cand, lo, hi, _ptr(out.scales),
                               _ptr(out.cand_idx), _ptr(out.loss), _ptr(out.losses), _ptr(out.packed),
                               _ptr(workspace), workspace.numel(), _stream(stream)), "tq_search_fp8")
    return out


def tq_pack_fp8(W: torch.Tensor, scales: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    d = _mat(W, "W")
    _cuda(scales, "scales")
    if out is None:
        out = torch.empty((d.n_mat, d.rows, d.cols), dtype=torch.uint8, device=W.device)
    _check(lib().tq_pack_fp8(ctypes.byref(d), _ptr(scales), _ptr(out), _stream(stream)), "tq_pack_fp8")
    return out


def tq_dequant_fp8(packed: torch.Tensor, scales: torch.Tensor, n_mat: int, O: int, I: int,
                   out_dtype=torch.float32, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _cuda(packed, "packed")
    if out is None:
        out = torch.empty((n_mat, O, I), dtype=out_dtype, device=packed.device)
    _check(lib().tq_dequant_fp8(_ptr(packed), _ptr(scales), n_mat, O, I, _ptr(out),
                                _BF16 if out.dtype == torch.bfloat16 else _F32, _stream(stream)), "tq_dequant_fp8")
    return out


@dataclasses.dataclass
class LloydResult:
    codebook: torch.Tensor            # f32 [4]
    scales: torch.Tensor              # f32 [n_mat, O, ceil(I/32)]
    packed: Optional[torch.Tensor]    # u8 2-bit codes, 8 bytes per 32-weight group
    loss: torch.Tensor                # f64 [1]
    history: torch.Tensor             # f64 [n_iter + 1]


LM_START = (-0.75, -0.25, 0.25, 0.75)   # the data-free Lloyd-Max levels of a uniform source on [-1, 1]


def tq_lloyd_max_g32(W: torch.Tensor, m: torch.Tensor, n_iter: int = 16, start=LM_START, pack: bool = True,
                     workspace: Optional[torch.Tensor] = None, stream=None) -> LloydResult:
    """imatrix-weighted Lloyd-Max 2-bit codebook on absmax-normalised 32-weight
    groups, shared by every matrix of W, and the 2-bit codes."""
    d = _mat(W, "W")
    _check_m(m, d.n_mat, d.cols)
    E, O, I = d.n_mat, d.rows, d.cols
    dev = W.device
    G = (I + 31) // 32
    res = LloydResult(codebook=torch.tensor(start, dtype=torch.float32, device=dev),
                      scales=torch.empty((E, O, G), dtype=torch.float32, device=dev),
                      packed=torch.empty(E * O * G * 8, dtype=torch.uint8, device=dev) if pack else None,
                      loss=torch.empty(1, dtype=torch.float64, device=dev),
                      history=torch.empty(n_iter + 1, dtype=torch.float64, device=dev))
    ws = int(lib().tq_lloyd_workspace_bytes(ctypes.byref(d)))
    if workspace is None:
        workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=dev)
    _check(lib().tq_lloyd_max_g32(ctypes.byref(d), _ptr(m), _m_stride(m), n_iter, _ptr(res.codebook),
                                  _ptr(res.scales), _ptr(res.packed), _ptr(res.loss), _ptr(res.history),
                                  _ptr(workspace), workspace.numel(), _stream(stream)), "tq_lloyd_max_g32")
    return res


def tq_dequant_lm2(packed: torch.Tensor, codebook: torch.Tensor, scales: torch.Tensor, n_mat: int, O: int, I: int,
                   out_dtype=torch.float32, stream=None) -> torch.Tensor:
    _cuda(packed, "packed")
    out = torch.empty((n_mat, O, I), dtype=out_dtype, device=packed.device)
    _check(lib().tq_dequant_lm2(_ptr(packed), _ptr(codebook), _ptr(scales), n_mat, O, I, _ptr(out),
                                _BF16 if out_dtype == torch.bfloat16 else _F32, _stream(stream)), "tq_dequant_lm2")
    return out


def tq_imatrix_static(X: torch.Tensor, m: Optional[torch.Tensor] = None, alpha: Optional[float] = None,
                      accumulate: bool = False, stream=None) -> torch.Tensor:
    """tq_imatrix without a caller workspace: the library's fixed device
    scratch is used instead (see include/tq.h for its limits and the rule
    that calls must not overlap on the GPU)."""
    d = _mat(X, "X")
    if alpha is None:
        alpha = 1.0 / d.rows
    if m is None:
        m = torch.zeros((d.n_mat, d.cols), dtype=torch.float32, device=X.device)
    _check_m(m, d.n_mat, d.cols, shared_ok=False)
    _check(lib().tq_imatrix_static(ctypes.byref(d), _ptr(m), _m_stride(m) if m.dim() == 2 else 0,
                                   ctypes.c_float(alpha), int(accumulate), _stream(stream)), "tq_imatrix_static")
    return m


def tq_imatrix_static_capacity() -> int:
    return int(lib().tq_imatrix_static_capacity())


def tq_amax(W: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    d = _mat(W, "W")
    if out is None:
        out = torch.empty(d.n_mat, dtype=torch.float32, device=W.device)
    _check(lib().tq_amax(ctypes.byref(d), _ptr(out), _stream(stream)), "tq_amax")
    return out


def search_result_empty(W: torch.Tensor, fmt: int, pack: bool = True, want_idx: bool = True,
                        want_loss: bool = True) -> SearchResult:
    """Uninitialised outputs of tq_search_groups for W and fmt (for callers
    that preallocate: pass the result as `out`)."""
    E, O, I, G = _groups(W, fmt)
    dev = W.device
    sdt = torch.uint8 if fmt == NVFP4_G16 else torch.float32
    return SearchResult(
        fmt=fmt,
        scales=torch.empty((E, O, G), dtype=sdt, device=dev),
        zeros=torch.empty((E, O, G), dtype=torch.uint8, device=dev) if fmt in _INT4 else None,
        global_scale=torch.empty(E, dtype=torch.float32, device=dev) if fmt == NVFP4_G16 else None,
        cand_idx=torch.empty((E, O, G), dtype=torch.int32, device=dev) if want_idx else None,
        loss=torch.empty((E, O, G), dtype=torch.float64, device=dev) if want_loss else None,
        packed=torch.empty(tq_packed_bytes(fmt, E * O, I), dtype=torch.uint8, device=dev) if pack else None,
    )


def tq_search_groups(W: torch.Tensor, m: torch.Tensor, fmt: int, params: Optional[SearchParams] = None,
                     pack: bool = True, want_idx: bool = True, want_loss: bool = True,
                     out: Optional[SearchResult] = None, stream=None) -> SearchResult:
    """imatrix-weighted per-group scale (and zero-point) search; with
    pack=True the chosen codes are rounded and packed in the same kernel.
    m: [I] (shared) or [n_mat, I] fp32 imatrix."""
    d = _mat(W, "W")
    _check_m(m, d.n_mat, d.cols)
    if out is None:
        out = search_result_empty(W, fmt, pack, want_idx, want_loss)
    p = (params or SearchParams())._c()
    _check(lib().tq_search_groups(ctypes.byref(d), _ptr(m), _m_stride(m), fmt, ctypes.byref(p),
                                  _ptr(out.scales), _ptr(out.zeros), _ptr(out.global_scale),
                                  _ptr(out.cand_idx), _ptr(out.loss), _ptr(out.packed),
                                  _stream(stream)), "tq_search_groups")
    return out


def tq_pack(W: torch.Tensor, fmt: int, scales: torch.Tensor, zeros: Optional[torch.Tensor] = None,
            global_scale: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
            stream=None) -> torch.Tensor:
    d = _mat(W, "W")
    E, O, I, G = _groups(W, fmt)
    if out is None:
        out = torch.empty(tq_packed_bytes(fmt, E * O, I), dtype=torch.uint8, device=W.device)
    _check(lib().tq_pack(ctypes.byref(d), fmt, _ptr(scales), _ptr(zeros), _ptr(global_scale), _ptr(out),
                         _stream(stream)), "tq_pack")
    return out


def tq_pack_codes(codes: torch.Tensor, fmt: int, zeros: Optional[torch.Tensor] = None,
                  out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """codes: [rows, cols] (any leading dims are flattened into rows) int8/uint8."""
    _cuda(codes, "codes")
    c = codes.reshape(-1, codes.shape[-1]).contiguous()
    if c.dtype == torch.int8:
        c = c.view(torch.uint8)
    rows, cols = c.shape
    if out is None:
        out = torch.empty(tq_packed_bytes(fmt, rows, cols), dtype=torch.uint8, device=codes.device)
    _check(lib().tq_pack_codes(_ptr(c), fmt, rows, cols, _ptr(zeros), _ptr(out), _stream(stream)),
           "tq_pack_codes")
    return out


def tq_unpack_codes(packed: torch.Tensor, fmt: int, rows: int, cols: int, stream=None) -> torch.Tensor:
    _cuda(packed, "packed")
    out = torch.empty((rows, cols), dtype=torch.uint8, device=packed.device)
    _check(lib().tq_unpack_codes(_ptr(packed), fmt, rows, cols, _ptr(out), _stream(stream)),
           "tq_unpack_codes")
    return out.view(torch.int8) if fmt == INT3_G64_SYM else out


def tq_dequant(packed: torch.Tensor, fmt: int, scales: torch.Tensor, zeros: Optional[torch.Tensor],
               global_scale: Optional[torch.Tensor], n_mat: int, O: int, I: int,
               out_dtype=torch.float32, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _cuda(packed, "packed")
    if out is None:
        out = torch.empty((n_mat, O, I), dtype=out_dtype, device=packed.device)
    odt = _BF16 if out.dtype == torch.bfloat16 else _F32
    _check(lib().tq_dequant(_ptr(packed), fmt, _ptr(scales), _ptr(zeros), _ptr(global_scale), n_mat, O, I,
                            _ptr(out), odt, _stream(stream)), "tq_dequant")
    return out


def tq_dequant_gemv(packed: torch.Tensor, fmt: int, scales: torch.Tensor, zeros: Optional[torch.Tensor],
                    global_scale: Optional[torch.Tensor], n_mat: int, O: int, I: int, x: torch.Tensor,
                    out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """y[e, b, o] = sum_j What[e, o, j] x[e, b, j] (fp32) for x of shape [B, I] (shared by every matrix) or
    [n_mat, B, I], B <= 8, What dequantized as tq_dequant defines it."""
    _cuda(packed, "packed")
    _cuda(x, "x")
    if x.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("x must be float32 or bfloat16")
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")
    if x.dim() == 2:
        B, xms = x.shape[0], 0
    elif x.dim() == 3 and x.shape[0] == n_mat:
        B, xms = x.shape[1], x.shape[1] * x.shape[2]
    else:
        raise ValueError("x must be [B, I] or [n_mat, B, I]")
    if x.shape[-1] != I:
        raise ValueError("x's last dimension must be I")
    if out is None:
        out = torch.empty((n_mat, B, O), dtype=torch.float32, device=packed.device)
    _check(lib().tq_dequant_gemv(_ptr(packed), fmt, _ptr(scales), _ptr(zeros), _ptr(global_scale), n_mat, O, I,
                                 _ptr(x), _BF16 if x.dtype == torch.bfloat16 else _F32, B, xms, _ptr(out),
                                 _stream(stream)), "tq_dequant_gemv")
    return out


def tq_proxy_error(W: torch.Tensor, packed: torch.Tensor, fmt: int, scales: torch.Tensor,
                   zeros: Optional[torch.Tensor], global_scale: Optional[torch.Tensor], m: torch.Tensor,
                   out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None,
                   workspace: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """(num, den) fp64 per matrix: tr(E H E^T), tr(W H W^T) with H = diag(m)."""
    d = _mat(W, "W")
    _check_m(m, d.n_mat, d.cols)
    if out is None:
        out = (torch.empty(d.n_mat, dtype=torch.float64, device=W.device),
               torch.empty(d.n_mat, dtype=torch.float64, device=W.device))
    ws = int(lib().tq_proxy_workspace_bytes(ctypes.byref(d), fmt))
    if workspace is None:
        workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=W.device)
    _check(lib().tq_proxy_error(ctypes.byref(d), _ptr(packed), fmt, _ptr(scales), _ptr(zeros),
                                _ptr(global_scale), _ptr(m), _m_stride(m), _ptr(out[0]), _ptr(out[1]),
                                _ptr(workspace), workspace.numel(), _stream(stream)), "tq_proxy_error")
    return out


# ---------------------------------------------------------------- grouped launches

MAX_BATCH = 16   # TQ_MAX_BATCH


def _ptrs(ts) -> ctypes.Array:
    """A host array of device pointers (NULL for None entries)."""
    return (ctypes.c_void_p * len(ts))(*[None if t is None else t.data_ptr() for t in ts])


def _opt_ptrs(ts):
    return None if ts is None or all(t is None for t in ts) else _ptrs(ts)


def _mats(Ws, name: str):
    ds = [_mat(W, f"{name}[{i}]") for i, W in enumerate(Ws)]
    if not 1 <= len(ds) <= MAX_BATCH:
        raise TQError(f"{name}: {len(ds)} units, expected 1..{MAX_BATCH}")
    return (_Mat * len(ds))(*ds)


def tq_pack_batch(Ws, fmt: int, scales, zeros=None, global_scale=None, out=None, stream=None):
    """tq_pack of several units (matrix batches of any shapes, one format and
    weight dtype) in one launch; lists of tensors per unit."""
    arr = _mats(Ws, "Ws")
    if out is None:
        out = [torch.empty(tq_packed_bytes(fmt, d.n_mat * d.rows, d.cols), dtype=torch.uint8, device=W.device)
               for W, d in zip(Ws, arr)]
    _check(lib().tq_pack_batch(len(Ws), arr, fmt, _ptrs(scales), _opt_ptrs(zeros), _opt_ptrs(global_scale),
                               _ptrs(out), _stream(stream)), "tq_pack_batch")
    return out


def tq_dequant_batch(packed, fmt: int, scales, zeros, global_scale, shapes, out_dtype=torch.float32, out=None,
                     stream=None):
    """tq_dequant of several units in one launch; shapes = [(n_mat, O, I), ...]."""
    n = len(packed)
    if not 1 <= n <= MAX_BATCH:
        raise TQError(f"tq_dequant_batch: {n} units, expected 1..{MAX_BATCH}")
    for i, t in enumerate(packed):
        _cuda(t, f"packed[{i}]")
    if out is None:
        out = [torch.empty(tuple(sh), dtype=out_dtype, device=packed[0].device) for sh in shapes]
    odt = _BF16 if out[0].dtype == torch.bfloat16 else _F32
    if any(o.dtype != out[0].dtype for o in out):
        raise TQError("tq_dequant_batch: outputs of different dtypes")
    i64 = ctypes.c_int64 * n
    _check(lib().tq_dequant_batch(n, _ptrs(packed), fmt, _ptrs(scales), _opt_ptrs(zeros), _opt_ptrs(global_scale),
                                  i64(*[s[0] for s in shapes]), i64(*[s[1] for s in shapes]),
                                  i64(*[s[2] for s in shapes]), _ptrs(out), odt, _stream(stream)),
           "tq_dequant_batch")
    return out


def proxy_batch_workspace_bytes(Ws, fmt: int) -> int:
    arr = _mats(Ws, "Ws")
    return int(lib().tq_proxy_batch_workspace_bytes(len(Ws), arr, fmt))


def tq_proxy_error_batch(Ws, packed, fmt: int, scales, zeros, global_scale, ms, out=None, workspace=None,
                         stream=None):
    """tq_proxy_error of several units in one launch: [(num, den), ...]."""
    arr = _mats(Ws, "Ws")
    for d, m in zip(arr, ms):
        _check_m(m, d.n_mat, d.cols)
    n = len(Ws)
    if out is None:
        out = [(torch.empty(d.n_mat, dtype=torch.float64, device=W.device),
                torch.empty(d.n_mat, dtype=torch.float64, device=W.device)) for W, d in zip(Ws, arr)]
    ws = int(lib().tq_proxy_batch_workspace_bytes(n, arr, fmt))
    if workspace is None:
        workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=Ws[0].device)
    _check(lib().tq_proxy_error_batch(n, arr, _ptrs(packed), fmt, _ptrs(scales), _opt_ptrs(zeros),
                                      _opt_ptrs(global_scale), _ptrs(ms),
                                      (ctypes.c_int64 * n)(*[_m_stride(m) for m in ms]),
                                      _ptrs([o[0] for o in out]), _ptrs([o[1] for o in out]), _ptr(workspace),
                                      workspace.numel(), _stream(stream)), "tq_proxy_error_batch")
    return out


def tq_proxy_error_full(X: torch.Tensor, W: torch.Tensor, packed: torch.Tensor, fmt: int, scales: torch.Tensor,
                        zeros: Optional[torch.Tensor], global_scale: Optional[torch.Tensor],
                        out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None,
                        workspace: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """(num, den) fp64 per matrix with the full Hessian H = X^T X, never
    formed: ||X (W - What)^T||_F^2 and ||X W^T||_F^2 on the tensor cores.
    X: [T, I] or [n_mat, T, I] bf16 activations of each matrix's input;
    W: [O, I] or [n_mat, O, I] bf16."""
    dx, dw = _mat(X, "X"), _mat(W, "W")
    if out is None:
        out = (torch.empty(dw.n_mat, dtype=torch.float64, device=W.device),
               torch.empty(dw.n_mat, dtype=torch.float64, device=W.device))
    ws = int(lib().tq_proxy_full_workspace_bytes(ctypes.byref(dx), ctypes.byref(dw)))
    if workspace is None:
        workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=W.device)
    _check(lib().tq_proxy_error_full(ctypes.byref(dx), ctypes.byref(dw), _ptr(packed), fmt, _ptr(scales),
                                     _ptr(zeros), _ptr(global_scale), _ptr(out[0]), _ptr(out[1]),
                                     _ptr(workspace), workspace.numel(), _stream(stream)), "tq_proxy_error_full")
    return out


def tq_gptq_sweep(W: torch.Tensor, fmt: int, scales: torch.Tensor, zeros: Optional[torch.Tensor], U: torch.Tensor,
                  out: Optional[Tuple[torch.Tensor, Optional[torch.Tensor]]] = None, want_loss: bool = True,
                  workspace: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """GPTQ/LDLQ column sweep of W ([O, I] or [n_mat, O, I]) with the given
    group scales (and zeros) held fixed.  U: fp32 [I, I] (one factor for all
    matrices) or [n_mat, I, I] upper triangular with H^-1 = U^T U (unit column
    stride).  Returns (codes int8 [n_mat, O, I], per-row loss fp64 [n_mat, O])."""
    d = _mat(W, "W")
    _cuda(U, "U")
    if U.dtype != torch.float32 or U.stride(-1) != 1 or U.dim() not in (2, 3):
        raise ValueError("U must be float32 [I, I] or [n_mat, I, I] with unit column stride")
    E, O, I = d.n_mat, d.rows, d.cols
    ums = U.stride(0) if U.dim() == 3 and U.shape[0] > 1 else 0
    if out is None:
        out = (torch.empty((E, O, I), dtype=torch.int8, device=W.device),
               torch.empty((E, O), dtype=torch.float64, device=W.device) if want_loss else None)
    ws = int(lib().tq_gptq_workspace_bytes(ctypes.byref(d)))
    if workspace is None:
        workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=W.device)
    _check(lib().tq_gptq_sweep(ctypes.byref(d), fmt, _ptr(scales), _ptr(zeros), _ptr(U), U.stride(-2), ums,
                               _ptr(out[0]), _ptr(out[1]), _ptr(workspace), workspace.numel(), _stream(stream)),
           "tq_gptq_sweep")
    return out


@dataclasses.dataclass
class Nvfp4Act:
    packed: torch.Tensor        # u8 [n_mat, T, ceil(I/16) * 8] NVFP4 records
    scales: torch.Tensor        # u8 [n_mat, T, ceil(I/16)] E4M3 block-scale codes
    global_scale: torch.Tensor  # f32 [n_mat]


def tq_quant_nvfp4_act(X: torch.Tensor, out: Optional[Nvfp4Act] = None, stream=None) -> Nvfp4Act:
    """NVFP4 activations (the weights' recipe without the search): per matrix
    g = amax / 2688, per 16-block the nearest E4M3 scale, E2M1 codes.
    X: [T, I] or [n_mat, T, I] bf16/fp32 on the GPU."""
    d = _mat(X, "X")
    E, T, I = d.n_mat, d.rows, d.cols
    G = (I + 15) // 16
    if out is None:
        out = Nvfp4Act(packed=torch.empty((E, T, G * 8), dtype=torch.uint8, device=X.device),
                       scales=torch.empty((E, T, G), dtype=torch.uint8, device=X.device),
                       global_scale=torch.empty(E, dtype=torch.float32, device=X.device))
    for t, n, shape in ((out.packed, "packed", (E, T, G * 8)), (out.scales, "scales", (E, T, G))):
        _cuda(t, n)
        if t.dtype != torch.uint8 or not t.is_contiguous() or t.numel() != E * T * shape[2]:
            raise TQError(f"{n} must be a contiguous uint8 tensor of {E * T * shape[2]} bytes")
    _check(lib().tq_quant_nvfp4_act(ctypes.byref(d), _ptr(out.packed), _ptr(out.scales), _ptr(out.global_scale),
                                    _stream(stream)), "tq_quant_nvfp4_act")
    return out


def tq_nvfp4_scales_mma_bytes(n_mat: int, rows: int, cols: int) -> int:
    return int(lib().tq_nvfp4_scales_mma_bytes(n_mat, rows, cols))


def tq_nvfp4_scales_to_mma(scales: torch.Tensor, n_mat: int, rows: int, cols: int,
                           out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """E4M3 block-scale codes [n_mat, rows, ceil(cols/16)] in the tensor core's
    scale tiles (include/tq.h)."""
    _cuda(scales, "scales")
    G = (cols + 15) // 16
    if scales.dtype != torch.uint8 or not scales.is_contiguous() or scales.numel() != n_mat * rows * G:
        raise TQError(f"scales must be contiguous uint8 [{n_mat}, {rows}, {G}]")
    nb = tq_nvfp4_scales_mma_bytes(n_mat, rows, cols)
    if out is None:
        out = torch.empty(nb, dtype=torch.uint8, device=scales.device)
    _cuda(out, "out")
    if out.numel() < nb:
        raise TQError(f"out needs {nb} bytes")
    _check(lib().tq_nvfp4_scales_to_mma(_ptr(scales), n_mat, rows, cols, _ptr(out), _stream(stream)),
           "tq_nvfp4_scales_to_mma")
    return out


def tq_gemm_nvfp4(x_packed: torch.Tensor, x_scales_mma: torch.Tensor, x_global: torch.Tensor,
                  w_packed: torch.Tensor, w_scales_mma: torch.Tensor, w_global: torch.Tensor,
                  n_mat: int, T: int, O: int, I: int, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """W4A4 product y [n_mat, T, O] (fp32) of NVFP4 activations and weights on
    the block-scaled tensor cores; scales in the tiles of tq_nvfp4_scales_to_mma."""
    G = (I + 15) // 16
    for t, n, need in ((x_packed, "x_packed", n_mat * T * G * 8), (w_packed, "w_packed", n_mat * O * G * 8),
                       (x_scales_mma, "x_scales_mma", tq_nvfp4_scales_mma_bytes(n_mat, T, I)),
                       (w_scales_mma, "w_scales_mma", tq_nvfp4_scales_mma_bytes(n_mat, O, I))):
        _cuda(t, n)
        if t.dtype != torch.uint8 or not t.is_contiguous() or t.numel() < need:
            raise TQError(f"{n} must be contiguous uint8 with at least {need} bytes")
    for t, n in ((x_global, "x_global"), (w_global, "w_global")):
        _cuda(t, n)
        if t.dtype != torch.float32 or t.numel() < n_mat:
            raise TQError(f"{n} must be float32 [{n_mat}]")
    if out is None:
        out = torch.empty((n_mat, T, O), dtype=torch.float32, device=x_packed.device)
    _cuda(out, "out")
    if out.dtype != torch.float32 or not out.is_contiguous() or out.numel() != n_mat * T * O:
        raise TQError(f"out must be contiguous float32 [{n_mat}, {T}, {O}]")
    _check(lib().tq_gemm_nvfp4(_ptr(x_packed), _ptr(x_scales_mma), _ptr(x_global), _ptr(w_packed),
                               _ptr(w_scales_mma), _ptr(w_global), n_mat, T, O, I, _ptr(out), _stream(stream)),
           "tq_gemm_nvfp4")
    return out


def gptq_workspace_bytes(W: torch.Tensor) -> int:
    return int(lib().tq_gptq_workspace_bytes(ctypes.byref(_mat(W, "W"))))


def proxy_full_workspace_bytes(X: torch.Tensor, W: torch.Tensor) -> int:
    return int(lib().tq_proxy_full_workspace_bytes(ctypes.byref(_mat(X, "X")), ctypes.byref(_mat(W, "W"))))


def imatrix_workspace_bytes(X: torch.Tensor) -> int:
    d = _mat(X, "X")
    return int(lib().tq_imatrix_workspace_bytes(ctypes.byref(d)))


def proxy_workspace_bytes(W: torch.Tensor, fmt: int) -> int:
    d = _mat(W, "W")
    return int(lib().tq_proxy_workspace_bytes(ctypes.byref(d), fmt))
