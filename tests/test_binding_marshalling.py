"""The Python binding's marshalling on the CPU: a fake library records the
arguments each call passes through the C ABI (descriptor shapes and strides,
factor strides, output shapes, workspace sizing).  The binding's own GPU
check is bypassed only here, so no kernel is involved."""

import pytest
import torch

import group_scale_search_b200 as tq


class _FakeLib:
    """Records calls; size queries return fixed byte counts, calls return TQ_OK."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append((name, args))
            if name == "tq_packed_bytes":
                return 1234
            return 4096 if name.endswith("_workspace_bytes") else 0
        return fn


def _desc(arg):
    d = arg._obj if hasattr(arg, "_obj") else arg
    return (d.dtype, d.n_mat, d.rows, d.cols, d.ld, d.mat_stride)


@pytest.fixture
def fake(monkeypatch):
    lib = _FakeLib()
    monkeypatch.setattr(tq, "lib", lambda: lib)
    monkeypatch.setattr(tq, "_cuda", lambda t, name: t)
    monkeypatch.setattr(tq, "_stream", lambda stream=None: None)
    return lib


def _last(lib, name):
    return [a for n, a in lib.calls if n == name][-1]


def test_matrix_descriptors(fake):
    W = torch.zeros((3, 40, 264), dtype=torch.bfloat16)[:, 2:34, :256]      # padded rows and a matrix stride
    assert _desc(tq._mat(W, "W")) == (1, 3, 32, 256, 264, 40 * 264)
    W2 = torch.zeros((32, 136))[:, :128]                                    # one fp32 matrix, ld 136
    assert _desc(tq._mat(W2, "W")) == (0, 1, 32, 128, 136, 0)
    with pytest.raises(tq.TQError):
        tq._mat(torch.zeros((4, 8), dtype=torch.float16), "W")
    with pytest.raises(tq.TQError):
        tq._mat(torch.zeros((8, 4)).t(), "W")                               # last dimension not contiguous


def test_gptq_marshalling(fake):
    W = torch.zeros((2, 16, 128), dtype=torch.bfloat16)
    U1 = torch.zeros((128, 132))[:, :128]                                   # one factor, rows of 132
    codes, loss = tq.tq_gptq_sweep(W, tq.INT4_G128_ASYM, torch.zeros(2 * 16), torch.zeros(2 * 16, dtype=torch.uint8),
                                   U1)
    args = _last(fake, "tq_gptq_sweep")
    assert _desc(args[0]) == (1, 2, 16, 128, 128, 16 * 128)
    assert args[1] == tq.INT4_G128_ASYM and args[5] == 132 and args[6] == 0
    assert codes.shape == (2, 16, 128) and codes.dtype == torch.int8
    assert loss.shape == (2, 16) and loss.dtype == torch.float64
    assert args[10] == 4096                                                 # the size the library asked for
    U3 = torch.zeros((2, 128, 128))                                         # one factor per matrix
    tq.tq_gptq_sweep(W, tq.INT3_G64_SYM, torch.zeros(64), None, U3, want_loss=False)
    args = _last(fake, "tq_gptq_sweep")
    assert args[5] == 128 and args[6] == 128 * 128 and args[8] is None
    with pytest.raises(ValueError):
        tq.tq_gptq_sweep(W, tq.INT3_G64_SYM, torch.zeros(64), None, torch.zeros((128, 128), dtype=torch.float64))


def test_proxy_full_marshalling(fake):
    X = torch.zeros((2, 300, 200), dtype=torch.bfloat16)
    W = torch.zeros((2, 48, 208), dtype=torch.bfloat16)[:, :, :200]
    num, den = tq.tq_proxy_error_full(X, W, torch.zeros(16, dtype=torch.uint8), tq.INT3_G64_SYM, torch.zeros(8),
                                      None, None)
    args = _last(fake, "tq_proxy_error_full")
    assert _desc(args[0]) == (1, 2, 300, 200, 200, 300 * 200)
    assert _desc(args[1]) == (1, 2, 48, 200, 208, 48 * 208)
    assert args[3] == tq.INT3_G64_SYM and args[10] == 4096
    assert num.shape == (2,) and den.dtype == torch.float64


def test_hessian_marshalling(fake):
    X = torch.zeros((3, 100, 64), dtype=torch.bfloat16)
    H = tq.tq_hessian(X, alpha=0.5, accumulate=True)
    args = _last(fake, "tq_hessian")
    assert H.shape == (3, 64, 64) and H.dtype == torch.float32 and not H.any()      # accumulate starts from zeros
    assert args[2] == 64 and args[3] == 64 * 64 and abs(args[4].value - 0.5) < 1e-7 and args[5] == 1
    with pytest.raises(ValueError):
        tq.tq_hessian(X, out=torch.zeros((3, 64, 65)))


def test_search_marshalling(fake):
    """Output shapes and dtypes per format (from the group sizes), the packed
    buffer sized by the library's answer, the imatrix stride (per matrix or
    shared) and the grid parameters."""
    W = torch.zeros((2, 8, 300), dtype=torch.bfloat16)
    m2 = torch.zeros((2, 304))[:, :300]
    for fmt, g in [(tq.INT3_G64_SYM, 64), (tq.INT4_G128_ASYM, 128), (tq.INT4_G64_ASYM, 64), (tq.INT4_G32_ASYM, 32),
                   (tq.NVFP4_G16, 16)]:
        r = tq.tq_search_groups(W, m2, fmt)
        args = _last(fake, "tq_search_groups")
        G = -(-300 // g)
        assert r.scales.shape == (2, 8, G)
        assert r.scales.dtype == (torch.uint8 if fmt == tq.NVFP4_G16 else torch.float32)
        assert (r.zeros is not None) == (fmt in (tq.INT4_G128_ASYM, tq.INT4_G64_ASYM, tq.INT4_G32_ASYM))
        assert (r.global_scale is not None) == (fmt == tq.NVFP4_G16)
        assert r.cand_idx.shape == (2, 8, G) and r.loss.dtype == torch.float64
        assert r.packed.numel() == 1234
        assert args[2] == 304 and args[3] == fmt
        p = args[4]._obj
        assert (p.sym_n1, p.sym_n2, p.asym_n_scale, p.asym_n_zero, p.fp4_window) == (32, 32, 64, 32, 16)
    tq.tq_search_groups(W, torch.zeros(300), tq.INT3_G64_SYM, params=tq.SearchParams(sym_n1=16), pack=False)
    args = _last(fake, "tq_search_groups")
    assert args[2] == 0 and args[4]._obj.sym_n1 == 16 and args[10] is None


def test_gemv_marshalling(fake):
    """x shared by every matrix ([B, I], matrix stride 0) or one per matrix
    ([n_mat, B, I]); the output [n_mat, B, O]; shapes that do not fit are refused."""
    packed = torch.zeros(64, dtype=torch.uint8)
    x = torch.zeros((3, 256), dtype=torch.bfloat16)
    y = tq.tq_dequant_gemv(packed, tq.INT4_G128_ASYM, torch.zeros(4), torch.zeros(4, dtype=torch.uint8), None,
                           2, 10, 256, x)
    args = _last(fake, "tq_dequant_gemv")
    assert y.shape == (2, 3, 10) and args[9] == 1 and args[10] == 3 and args[11] == 0
    x3 = torch.zeros((2, 5, 256))
    tq.tq_dequant_gemv(packed, tq.INT3_G64_SYM, torch.zeros(4), None, None, 2, 10, 256, x3)
    args = _last(fake, "tq_dequant_gemv")
    assert args[9] == 0 and args[10] == 5 and args[11] == 5 * 256
    with pytest.raises(ValueError):
        tq.tq_dequant_gemv(packed, tq.INT3_G64_SYM, torch.zeros(4), None, None, 2, 10, 255, x)
    with pytest.raises(ValueError):
        tq.tq_dequant_gemv(packed, tq.INT3_G64_SYM, torch.zeros(4), None, None, 3, 10, 256, x3)


@pytest.mark.parametrize("bad", [
    torch.zeros((2, 64), dtype=torch.float64),               # not fp32
    torch.zeros((2, 63)),                                    # too few columns
    torch.zeros((3, 64)),                                    # wrong matrix count
    torch.zeros(10),                                         # a short vector
    torch.zeros((64, 2)).t(),                                # non-unit column stride
    torch.zeros((2, 64, 1)),                                 # wrong rank
])
def test_imatrix_outputs_refused_before_any_call(fake, bad):
    """tq_imatrix / tq_imatrix_static write m in place: a tensor of the wrong
    dtype, shape or strides is refused on the host, and nothing is called."""
    X = torch.zeros((2, 16, 64), dtype=torch.bfloat16)
    for fn in (tq.tq_imatrix, tq.tq_imatrix_static):
        with pytest.raises(tq.TQError):
            fn(X, m=bad)
    assert not [n for n, _ in fake.calls if n in ("tq_imatrix", "tq_imatrix_static")]


def test_imatrix_output_rows_must_not_overlap(fake):
    X = torch.zeros((2, 16, 64), dtype=torch.bfloat16)
    m = torch.zeros(128).as_strided((2, 64), (32, 1))        # rows 32 floats apart: overlapping
    with pytest.raises(tq.TQError):
        tq.tq_imatrix(X, m=m)
    m_ok = torch.zeros((2, 80))[:, :64]                      # padded rows are fine
    tq.tq_imatrix(X, m=m_ok)
    assert _last(fake, "tq_imatrix")[2] == 80


@pytest.mark.parametrize("bad", [torch.zeros(63), torch.zeros((3, 64)), torch.zeros(64, dtype=torch.bfloat16)])
def test_imatrix_inputs_refused(fake, bad):
    """The search, proxy error, FP8 search and Lloyd-Max read m: the same
    checks, with one shared [I] vector (or [1, I]) also allowed."""
    W = torch.zeros((2, 8, 64), dtype=torch.bfloat16)
    with pytest.raises(tq.TQError):
        tq.tq_search_groups(W, bad, tq.INT3_G64_SYM)
    with pytest.raises(tq.TQError):
        tq.tq_proxy_error(W, torch.zeros(16, dtype=torch.uint8), tq.INT3_G64_SYM, torch.zeros(16), None, None, bad)
    with pytest.raises(tq.TQError):
        tq.tq_search_fp8(W, bad)
    with pytest.raises(tq.TQError):
        tq.tq_lloyd_max_g32(W, bad)
    for ok in (torch.zeros(64), torch.zeros((1, 64)), torch.zeros((2, 64))):
        tq.tq_search_groups(W, ok, tq.INT3_G64_SYM)
