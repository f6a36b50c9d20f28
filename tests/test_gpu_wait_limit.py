"""The give-up path of the tensor-core pipelines (tq_hessian,
tq_proxy_error_full), run on the GPU without stalling anything: the ring
waits' limit is set to zero rounds, so every CTA gives up at its first wait,
before it has issued any copy or MMA.  The call must then leave its outputs
as the give-up rule says (H untouched; num/den NaN), the next tq_sync must
report the timeout, and the next call with the default limit must be
correct again.  The limit is restored whatever happens."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("group_scale_search_b200")
import oracle  # noqa: E402

DEV = "cuda"


@pytest.fixture(autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    oracle.build()
    tq.lib()
    yield
    tq.tq_debug_set_wait_limit(-1)


def _x(T, I, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    return (torch.randn((T, I), generator=g, device=DEV) * 0.5).bfloat16()


def test_hessian_gives_up_and_recovers():
    X = _x(256, 320, 1)
    H = torch.full((320, 320), 7.0, dtype=torch.float32, device=DEV)
    tq.tq_sync()
    tq.tq_debug_set_wait_limit(0)
    tq.tq_hessian(X, out=H)
    with pytest.raises(tq.TQError, match="tq_hessian pipeline wait timed out"):
        tq.tq_sync()
    assert torch.all(H == 7.0)                 # a launch that gave up stores nothing
    tq.tq_debug_set_wait_limit(-1)
    tq.tq_hessian(X, out=H)
    tq.tq_sync()                               # the timeout was reported once; this launch is clean
    Xh = X.float().cpu().numpy()
    ref = oracle.hessian(Xh)
    bound = (256 / 16 + 32) * 2.0 ** -22 * (np.abs(Xh).T.astype(np.float64) @ np.abs(Xh).astype(np.float64))
    assert np.all(np.abs(H.cpu().numpy().astype(np.float64) - ref) <= bound)


def test_proxy_full_gives_up_and_recovers():
    E, T, O, I = 2, 200, 96, 256
    W = (synth.student_t((E, O, I), 4, torch.Generator(device=DEV).manual_seed(2), DEV) * 0.02).bfloat16()
    X = torch.stack([_x(T, I, 3 + e) for e in range(E)])
    m = tq.tq_imatrix(X)
    res = tq.tq_search_groups(W, m, tq.INT4_G128_ASYM)
    ok = tq.tq_proxy_error_full(X, W, res.packed, tq.INT4_G128_ASYM, res.scales, res.zeros, None)
    tq.tq_sync()
    ok = (ok[0].clone(), ok[1].clone())
    tq.tq_debug_set_wait_limit(0)
    bad = tq.tq_proxy_error_full(X, W, res.packed, tq.INT4_G128_ASYM, res.scales, res.zeros, None)
    with pytest.raises(tq.TQError, match="tq_proxy_error_full pipeline wait timed out"):
        tq.tq_sync()
    assert torch.isnan(bad[0]).all() and torch.isnan(bad[1]).all()
    tq.tq_debug_set_wait_limit(-1)
    again = tq.tq_proxy_error_full(X, W, res.packed, tq.INT4_G128_ASYM, res.scales, res.zeros, None)
    tq.tq_sync()
    assert torch.equal(again[0], ok[0]) and torch.equal(again[1], ok[1])   # deterministic, as before


def test_limit_applies_to_later_launches_only():
    """The limit is read when a call is enqueued: setting it after the launch
    does not touch a launch already queued."""
    X = _x(128, 192, 5)
    H1 = tq.tq_hessian(X)
    tq.tq_debug_set_wait_limit(0)
    tq.tq_debug_set_wait_limit(-1)
    tq.tq_sync()
    H2 = tq.tq_hessian(X)
    tq.tq_sync()
    assert torch.equal(H1, H2)
