"""The seeded synthetic workloads follow their recipe: shapes, dtypes, the
outlier structure of each configuration, LogNormal per-channel activation
scales, and determinism in the seed (CPU; small scales where the full size
would be heavy)."""
import numpy as np
import torch

import synth


def test_c0_shapes():
    """(Its two outlier rows sit inside a heavy-tailed t(4) body, so they are
    checked through the int3-vs-per-row-int4 pin, not by a statistic here.)"""
    wl = synth.make("c0", "cpu")
    W = wl.units[0].W[0]
    assert W.shape == (256, 512) and W.dtype == torch.float32 and wl.units[0].fmt == "int3_g64_sym"
    assert wl.sites["x"].X.shape == (1, 128, 512) and wl.sites["x"].X.dtype == torch.float32


def test_c1_shapes_and_outlier_columns():
    wl = synth.make("c1", "cpu")
    W = wl.units[0].W[0].float()
    assert W.shape == (4096, 4096) and wl.units[0].W.dtype == torch.bfloat16
    assert wl.sites["x"].X.shape == (1, 2048, 4096) and wl.sites["x"].X.dtype == torch.bfloat16
    col_std = W.std(dim=0)
    assert int((col_std > 0.1).sum()) == round(0.001 * 4096)     # columns scaled x10 (std 0.2 vs 0.02)
    body = col_std[col_std <= 0.1]
    assert abs(float(body.mean()) - 0.02) < 0.001


def test_activation_channel_scales_are_lognormal():
    X = synth.make("c1", "cpu").sites["x"].X[0].float()
    log_rms = torch.log(X.pow(2).mean(dim=0).sqrt()).numpy()
    assert abs(log_rms.mean()) < 0.1 and abs(log_rms.std() - 1.0) < 0.1    # c_j ~ LogNormal(0, 1)


def test_moe_and_layer_structure_at_small_scale():
    c2 = synth.make("c2", "cpu", scale=0.05)
    experts, tail = c2.units
    E, O, I = experts.W.shape
    assert c2.sites["x"].X.shape[0] == E and tail.W.shape[-1] == I + 40 and not tail.timed
    rows = experts.W.float().abs().amax(dim=2)                 # rows x15 stand far above the t(4) * 0.015 body
    assert all(int((rows[e] > 15 * 0.015 * 2).sum()) >= 1 for e in range(E))
    c3 = synth.make("c3", "cpu", scale=0.05)
    assert [u.name for u in c3.units] == [n for n, *_ in synth.C3_LINEARS]
    assert {u.site for u in c3.units} == set(c3.sites)
    for u in c3.units:
        assert u.W.shape[-1] == c3.sites[u.site].X.shape[-1]
    c4 = synth.make("c4", "cpu", scale=0.05)
    assert c4.units[0].fmt == "nvfp4_g16" and c4.units[0].W.shape[0] == c4.sites["x"].X.shape[0]


def test_seeded_and_deterministic():
    a = synth.make("c1", "cpu", scale=0.125)
    b = synth.make("c1", "cpu", scale=0.125)
    c = synth.make("c1", "cpu", seed=1, scale=0.125)
    assert torch.equal(a.units[0].W, b.units[0].W) and torch.equal(a.sites["x"].X, b.sites["x"].X)
    assert not torch.equal(a.units[0].W, c.units[0].W)
    assert np.isfinite(a.units[0].W.float().numpy()).all()


def test_layout_matches_the_drawn_shapes():
    """synth.layout (shapes only, used for the bench's configuration and the
    ranks' split) agrees with what synth.make draws, and max_mats draws the
    first experts of the whole stack."""
    for name in ("c0", "c1", "c2", "c3", "c4"):
        lay = synth.layout(name, 0.05)
        wl = synth.make(name, "cpu", scale=0.05)
        assert [(u.name, u.fmt, tuple(u.W.shape), u.site, u.timed) for u in wl.units] == lay["units"]
        assert {k: tuple(s.X.shape) for k, s in wl.sites.items()} == {k: v[:3] for k, v in lay["sites"].items()}
    full = synth.make("c4", "cpu", scale=0.05)
    first = synth.make("c4", "cpu", scale=0.05, max_mats=1)
    assert torch.equal(first.units[0].W[0], full.units[0].W[0]) and first.units[0].W.shape[0] == 1
    assert torch.equal(first.sites["x"].X[0], full.sites["x"].X[0])
    assert synth.layout("c2")["units"][0][2] == (64, 2048, 7168)
