"""The allocation-free imatrix entry point, for callers that cannot allocate
device memory where they call it (an engine hook handed only its buffers, or
memory fully planned by an arena): through the C ABI it must give the same
imatrix as tq_imatrix with a caller workspace, call after call, while its
scratch lives in the library.  Collected last on purpose."""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("group_scale_search_b200")

import synth  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    tq.lib()


def _rel(a, b):
    return ((a.double() - b.double()).abs() / b.double().abs().clamp_min(1e-30)).max().item()


@pytest.mark.parametrize("name,scale", [("c1", 0.125), ("c2", 0.05), ("c0", 1.0)])
def test_static_scratch_matches_workspace_version_twice(name, scale):
    wl = synth.make(name, "cuda", scale=scale)
    for site in wl.sites.values():
        X = site.X
        ref = tq.tq_imatrix(X)
        got1 = tq.tq_imatrix_static(X)
        got2 = tq.tq_imatrix_static(X)      # second call reuses the scratch left by the first
        torch.cuda.synchronize()
        assert _rel(got1, ref) <= 1e-5
        assert _rel(got2, ref) <= 1e-5


def test_static_scratch_accumulates_and_rejects_oversize():
    X = synth.make("c1", "cuda", scale=0.125).sites["x"].X[0]
    T = X.shape[0]
    m = tq.tq_imatrix_static(X[: T // 2], alpha=1.0)
    tq.tq_imatrix_static(X[T // 2:], m=m, alpha=1.0, accumulate=True)
    ref = tq.tq_imatrix(X, alpha=1.0)
    torch.cuda.synchronize()
    assert _rel(m, ref) <= 1e-5
    cap = tq.tq_imatrix_static_capacity()
    # A shape whose fp64 token-slice partials exceed the fixed scratch: one
    # column tile more than a wave of blocks, over 2^24 tokens, splits into
    # many slices.  The call is refused on the host, before any launch, so
    # the descriptor's pointer is never read.
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    cols = (4 * sms + 1) * 256
    L = tq.lib()
    fake = ctypes.c_void_p(0x1000)
    d = tq._Mat(fake, 1, 0, 1, 1 << 24, cols, cols, 0)   # bf16 [1, 2^24, cols], never dereferenced
    assert L.tq_imatrix_workspace_bytes(ctypes.byref(d)) > cap
    m_dev = torch.empty(cols, dtype=torch.float32, device="cuda")
    st = L.tq_imatrix_static(ctypes.byref(d), ctypes.c_void_p(m_dev.data_ptr()), cols, ctypes.c_float(1.0), 0, None)
    assert st == 1 and b"scratch" in L.tq_last_error_string()
