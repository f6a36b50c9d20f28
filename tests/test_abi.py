"""C-ABI library checks that need no GPU: it loads, exports every symbol
include/tq.h declares, and its host-side size/validation logic answers."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def tq():
    from group_scale_search_b200 import build
    build.build()
    import group_scale_search_b200 as g
    g.lib()
    return g


def test_exports_every_declared_symbol(tq):
    declared = _declared()
    assert len(declared) >= 15
    L = ctypes.CDLL(tq.lib_path())
    for name in declared:
        assert hasattr(L, name), name
    assert sorted(tq.EXPORTS) == declared


def test_library_targets_sm100a(tq):
    assert "sm_100a" in tq.tq_version()


def test_sizes(tq):
    assert tq.tq_group_size(tq.INT3_G64_SYM) == 64
    assert tq.tq_group_size(tq.INT4_G128_ASYM) == 128
    assert tq.tq_group_size(tq.NVFP4_G16) == 16
    assert tq.tq_group_size(tq.INT4_G64_ASYM) == 64
    assert tq.tq_packed_bytes(tq.INT4_G64_ASYM, 5, 200) == 5 * 4 * 32   # 32-byte records, ragged last group
    assert tq.tq_group_size(tq.INT4_G32_ASYM) == 32
    assert tq.tq_packed_bytes(tq.INT4_G32_ASYM, 5, 200) == 5 * 7 * 16   # 16-byte records, ragged last group
    assert tq.tq_num_groups(tq.INT4_G32_ASYM, 5, 200) == 35
    assert tq.tq_group_size(99) == 0
    # int3-g64: 24 bytes per 64 weights + f32 scale = 3.5 bits/weight
    assert tq.tq_packed_bytes(tq.INT3_G64_SYM, 2048, 7168) == 2048 * 112 * 24
    assert tq.tq_packed_bytes(tq.INT3_G64_SYM, 2048, 7208) == 2048 * 113 * 24
    assert tq.tq_packed_bytes(tq.INT4_G128_ASYM, 4096, 4096) == 4096 * 32 * 64
    assert tq.tq_packed_bytes(tq.NVFP4_G16, 1856, 2688) == 1856 * 168 * 8
    assert tq.tq_num_groups(tq.NVFP4_G16, 3, 17) == 6


def test_default_params(tq):
    p = tq._Params()
    tq.lib().tq_default_params(ctypes.byref(p))
    assert (p.sym_n1, p.sym_n2, p.sym_lo, p.sym_hi) == (32, 32, 0.5, 1.2)
    assert (p.asym_n_scale, p.asym_n_zero, p.asym_lo, p.asym_hi, p.fp4_window) == (64, 32, 0.5, 1.2, 16)


def test_invalid_arguments_are_rejected_before_any_launch(tq):
    L = tq.lib()
    m = tq._Mat(None, 1, 0, 1, 4, 64, 64, 0)
    p = tq._Params()
    L.tq_default_params(ctypes.byref(p))
    st = L.tq_search_groups(ctypes.byref(m), None, 0, tq.INT3_G64_SYM, ctypes.byref(p),
                            None, None, None, None, None, None, None)
    assert st == 1 and b"null" in L.tq_last_error_string()
    fake = ctypes.c_void_p(0x1000)   # never dereferenced: validation fails first
    m = tq._Mat(fake, 1, 0, 1, 4, 64, 32, 0)    # ld < cols
    st = L.tq_search_groups(ctypes.byref(m), fake, 0, tq.INT3_G64_SYM, None, fake, None, None,
                            None, None, None, None)
    assert st == 1 and b"ld" in L.tq_last_error_string()
    m = tq._Mat(ctypes.c_void_p(0x1008), 1, 0, 1, 4, 64, 64, 0)    # misaligned
    st = L.tq_search_groups(ctypes.byref(m), fake, 0, tq.INT3_G64_SYM, None, fake, None, None,
                            None, None, None, None)
    assert st == 1 and b"aligned" in L.tq_last_error_string()
    m = tq._Mat(fake, 7, 0, 1, 4, 64, 64, 0)    # unknown dtype
    assert L.tq_amax(ctypes.byref(m), fake, None) == 2
    m = tq._Mat(fake, 1, 0, 1, 4, 64, 64, 0)
    assert L.tq_search_groups(ctypes.byref(m), fake, 0, 99, None, fake, None, None,
                              None, None, None, None) == 2
    # int4 needs zeros; others must not get them
    assert L.tq_search_groups(ctypes.byref(m), fake, 0, tq.INT4_G128_ASYM, None, fake, None, None,
                              None, None, None, None) == 1
    assert L.tq_search_groups(ctypes.byref(m), fake, 0, tq.INT3_G64_SYM, None, fake, fake, None,
                              None, None, None, None) == 1
    # unsupported grid sizes
    p2 = tq._Params()
    L.tq_default_params(ctypes.byref(p2))
    p2.asym_n_scale = 257
    assert L.tq_search_groups(ctypes.byref(m), fake, 0, tq.INT4_G128_ASYM, ctypes.byref(p2), fake, fake,
                              None, None, None, None, None) == 2
    p.sym_n1 = 40
    assert L.tq_search_groups(ctypes.byref(m), fake, 0, tq.INT3_G64_SYM, ctypes.byref(p), fake, None,
                              None, None, None, None, None) == 2
    # workspace too small
    x = tq._Mat(fake, 0, 0, 1, 1024, 512, 512, 0)
    need = L.tq_imatrix_workspace_bytes(ctypes.byref(x))
    assert need > 0
    assert L.tq_imatrix(ctypes.byref(x), fake, 512, ctypes.c_float(1.0), 0, fake, need - 8, None) == 1
    # dequant-GEMV: (packed, fmt, scales, zeros, gs, n_mat, O, I, x, x_dtype, B, x_mat_stride, y, stream)
    gemv = L.tq_dequant_gemv
    assert gemv(None, tq.INT3_G64_SYM, fake, None, None, 1, 8, 64, fake, 0, 1, 0, fake, None) == 1
    assert gemv(fake, 99, fake, None, None, 1, 8, 64, fake, 0, 1, 0, fake, None) == 2
    assert gemv(fake, tq.INT3_G64_SYM, fake, None, None, 1, 8, 64, fake, 7, 1, 0, fake, None) == 2
    for B in (0, 9):
        assert gemv(fake, tq.INT3_G64_SYM, fake, None, None, 1, 8, 64, fake, 0, B, 0, fake, None) == 1
        assert b"B must" in L.tq_last_error_string()
    assert gemv(fake, tq.INT3_G64_SYM, fake, None, None, 2, 8, 64, fake, 0, 2, 100, fake, None) == 1
    assert gemv(fake, tq.INT3_G64_SYM, fake, None, None, 1, 0, 64, fake, 0, 1, 0, fake, None) == 1
    assert gemv(ctypes.c_void_p(0x1008), tq.INT3_G64_SYM, fake, None, None, 1, 8, 64, fake, 0, 1, 0, fake,
                None) == 1
    assert b"aligned" in L.tq_last_error_string()
    assert gemv(fake, tq.INT4_G128_ASYM, fake, None, None, 1, 8, 64, fake, 0, 1, 0, fake, None) == 1
    assert gemv(fake, tq.NVFP4_G16, fake, None, None, 1, 8, 64, fake, 0, 1, 0, fake, None) == 1
    # FP8 per tensor: (W, m, m_stride, n_cand, lo, hi, scales, idx, loss, losses, packed, ws, ws_bytes, stream)
    w8 = tq._Mat(fake, 1, 0, 1, 16, 64, 64, 0)
    need8 = L.tq_fp8_workspace_bytes(ctypes.byref(w8))
    assert need8 > 0
    f8 = L.tq_search_fp8
    assert f8(ctypes.byref(w8), fake, 0, 65, 0.5, 1.2, fake, None, None, None, None, fake, need8, None) == 2
    assert f8(ctypes.byref(w8), fake, 0, 64, 0.5, 1.2, fake, None, None, None, None, fake, need8 - 8, None) == 1
    assert f8(ctypes.byref(w8), fake, 0, 64, 1.2, 0.5, fake, None, None, None, None, fake, need8, None) == 1
    assert f8(ctypes.byref(w8), None, 0, 64, 0.5, 1.2, fake, None, None, None, None, fake, need8, None) == 1
    assert L.tq_dequant_fp8(fake, fake, 1, 4, 64, fake, 7, None) == 2
    # Hessian: (X, H, ldh, h_mat_stride, alpha, accumulate, stream)
    hs = L.tq_hessian
    x = tq._Mat(fake, 1, 0, 1, 256, 128, 128, 0)
    x = tq._Mat(fake, 0, 0, 1, 256, 128, 128, 0)   # fp32 X
    assert hs(ctypes.byref(x), fake, 128, 0, ctypes.c_float(1.0), 0, None) == 2
    x = tq._Mat(fake, 1, 0, 1, 256, 128, 128, 0)
    assert hs(ctypes.byref(x), fake, 100, 0, ctypes.c_float(1.0), 0, None) == 1   # ldh < I
    assert hs(ctypes.byref(x), None, 128, 0, ctypes.c_float(1.0), 0, None) == 1
    x = tq._Mat(fake, 1, 0, 1, 256, 100, 100, 0)   # row stride 200 B
    assert hs(ctypes.byref(x), fake, 100, 0, ctypes.c_float(1.0), 0, None) == 1
    x = tq._Mat(ctypes.c_void_p(0x1008), 1, 0, 1, 256, 128, 128, 0)
    assert hs(ctypes.byref(x), fake, 128, 0, ctypes.c_float(1.0), 0, None) == 1

    # proxy error with the full Hessian: (X, W, packed, fmt, scales, zeros, gs, num, den, ws, ws_bytes, stream)
    pf = L.tq_proxy_error_full
    xa = tq._Mat(fake, 1, 0, 1, 300, 200, 200, 0)
    wa = tq._Mat(fake, 1, 0, 1, 300, 200, 200, 0)
    needf = L.tq_proxy_full_workspace_bytes(ctypes.byref(xa), ctypes.byref(wa))
    assert needf >= 300 * 2 * 256 * 2 + 2 * 3 * 2 * 8     # two bf16 pieces of E, I padded to 256; tile partials
    args = (tq.INT3_G64_SYM, fake, None, None, fake, fake, fake, needf, None)
    assert pf(ctypes.byref(xa), ctypes.byref(wa), None, *args) == 1
    assert pf(ctypes.byref(xa), ctypes.byref(wa), fake, 99, *args[1:]) == 2
    assert pf(ctypes.byref(xa), ctypes.byref(wa), fake, *args[:-2], needf - 8, None) == 1
    assert b"workspace" in L.tq_last_error_string()
    x32 = tq._Mat(fake, 0, 0, 1, 300, 200, 200, 0)
    assert pf(ctypes.byref(x32), ctypes.byref(wa), fake, *args) == 2
    xb = tq._Mat(fake, 1, 0, 1, 300, 208, 208, 0)            # I differs
    assert pf(ctypes.byref(xb), ctypes.byref(wa), fake, *args) == 1
    assert pf(ctypes.byref(xa), ctypes.byref(wa), fake, tq.INT4_G128_ASYM, *args[1:]) == 1   # int4 needs zeros
    assert pf(ctypes.byref(xa), ctypes.byref(wa), fake, tq.NVFP4_G16, *args[1:]) == 1        # needs global scale

    # GPTQ sweep: (W, fmt, scales, zeros, U, ldu, u_mat_stride, codes, loss, ws, ws_bytes, stream)
    gq = L.tq_gptq_sweep
    wg = tq._Mat(fake, 1, 0, 2, 40, 200, 200, 40 * 200)
    needg = L.tq_gptq_workspace_bytes(ctypes.byref(wg))
    assert needg == 2 * 40 * 200 * 4
    assert gq(ctypes.byref(wg), tq.NVFP4_G16, fake, None, fake, 200, 0, fake, None, fake, needg, None) == 2
    assert gq(ctypes.byref(wg), tq.INT4_G128_ASYM, fake, None, fake, 200, 0, fake, None, fake, needg, None) == 1
    assert gq(ctypes.byref(wg), tq.INT3_G64_SYM, fake, None, fake, 199, 0, fake, None, fake, needg, None) == 1
    assert gq(ctypes.byref(wg), tq.INT3_G64_SYM, fake, None, fake, 200, 100, fake, None, fake, needg, None) == 1
    assert gq(ctypes.byref(wg), tq.INT3_G64_SYM, fake, None, None, 200, 0, fake, None, fake, needg, None) == 1
    assert gq(ctypes.byref(wg), tq.INT3_G64_SYM, fake, None, fake, 200, 0, fake, None, fake, needg - 4, None) == 1
    assert b"workspace" in L.tq_last_error_string()


def test_binding_refuses_cpu_tensors(tq):
    import torch
    with pytest.raises(tq.TQError):
        tq.tq_imatrix(torch.zeros(8, 64))
    W = torch.zeros(8, 64, dtype=torch.bfloat16)
    with pytest.raises(tq.TQError):
        tq.tq_proxy_error_full(torch.zeros(4, 64, dtype=torch.bfloat16), W, torch.zeros(256, dtype=torch.uint8),
                               tq.INT3_G64_SYM, torch.zeros(8), None, None)
    with pytest.raises(tq.TQError):
        tq.tq_gptq_sweep(W, tq.INT3_G64_SYM, torch.zeros(8), None, torch.eye(64))
    with pytest.raises(tq.TQError):
        tq.tq_hessian(torch.zeros(4, 64, dtype=torch.bfloat16))


def test_grouped_calls_validate_before_any_launch(tq):
    """tq_pack_batch / tq_dequant_batch / tq_proxy_error_batch: unit counts,
    mixed dtypes, missing zero-points and bad shapes are refused on the host;
    the workspace query follows the units' shapes."""
    L = tq.lib()
    fake = ctypes.c_void_p(0x1000)   # never dereferenced: validation fails first
    V = ctypes.c_void_p
    mats = (tq._Mat * 2)(tq._Mat(fake, 1, 0, 1, 8, 64, 64, 0), tq._Mat(fake, 0, 0, 1, 8, 64, 64, 0))
    ptrs = (V * 2)(0x1000, 0x2000)
    for n in (0, tq.MAX_BATCH + 1):
        assert L.tq_pack_batch(n, mats, tq.INT3_G64_SYM, ptrs, None, None, ptrs, None) == 1
        assert b"outside" in L.tq_last_error_string()
    assert L.tq_pack_batch(2, mats, tq.INT3_G64_SYM, ptrs, None, None, ptrs, None) == 1   # bf16 + fp32
    assert b"dtypes" in L.tq_last_error_string()
    assert L.tq_pack_batch(1, mats, tq.INT4_G128_ASYM, ptrs, None, None, ptrs, None) == 1  # no zeros
    assert L.tq_pack_batch(1, mats, 99, ptrs, None, None, ptrs, None) == 2
    i64 = ctypes.c_int64 * 2
    assert L.tq_dequant_batch(2, ptrs, tq.INT3_G64_SYM, ptrs, None, None, i64(1, 1), i64(8, 0), i64(64, 64),
                              ptrs, 1, None) == 1   # empty shape in unit 1
    assert b"empty" in L.tq_last_error_string()
    assert L.tq_dequant_batch(1, ptrs, tq.NVFP4_G16, ptrs, None, None, i64(1, 1), i64(8, 8), i64(64, 64),
                              ptrs, 1, None) == 1   # NVFP4 without global scales
    one = L.tq_proxy_batch_workspace_bytes(1, mats, tq.INT3_G64_SYM)
    assert one == L.tq_proxy_workspace_bytes(mats, tq.INT3_G64_SYM) and one > 0
    assert L.tq_proxy_batch_workspace_bytes(2, mats, tq.INT3_G64_SYM) > one
    assert L.tq_proxy_batch_workspace_bytes(tq.MAX_BATCH + 1, mats, tq.INT3_G64_SYM) == 0
    assert L.tq_proxy_error_batch(1, mats, ptrs, tq.INT3_G64_SYM, ptrs, None, None, ptrs, i64(0, 0), ptrs, ptrs,
                                  fake, 8, None) == 1   # workspace too small
    assert b"workspace" in L.tq_last_error_string()
