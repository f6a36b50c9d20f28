"""NVFP4 W4A4 product against the oracle: the activation quantizer bit for bit
(global scale, E4M3 block scales, E2M1 records), the scale tiles against
their stated layout, and the block-scaled tensor-core GEMM against the exact
value of the block-scaled representation within the fp32 accumulation bound
(ragged tokens, rows and columns; one and several matrices; the NVFP4 MoE
expert shape; and records written by the search fed straight in)."""
import numpy as np
import pytest
import torch

import synth
from gpu_checks import host32

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("group_scale_search_b200")
import oracle  # noqa: E402

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    oracle.build()
    tq.lib()


def _acts(E, T, I, seed, dtype=torch.bfloat16):
    """Tokens with LogNormal channel scales; rows padded to a 16-byte stride
    (the library's alignment rule) when I alone would not give one."""
    g = torch.Generator(device=DEV).manual_seed(seed)
    ld = -(-I * torch.tensor([], dtype=dtype).element_size() // 16) * 16 // torch.tensor([], dtype=dtype).element_size()
    X = torch.zeros((E, T, ld), dtype=dtype, device=DEV)[:, :, :I]
    for e in range(E):
        c = synth.lognormal_channels(I, g, DEV)
        X[e] = (torch.randn((T, I), generator=g, device=DEV) * c).to(dtype)
    return X


def _oracle_quant(Xh):
    """Per matrix: the oracle's global scale, scale codes, E2M1 codes and records."""
    gs, scs, cs, recs = [], [], [], []
    for x in Xh:
        g, sc, c = oracle.nvfp4_quant_act(x)
        gs.append(g)
        scs.append(sc)
        cs.append(c)
        recs.append(oracle.pack_nibbles(c, 16))
    return np.array(gs, np.float32), np.stack(scs), np.stack(cs), np.stack(recs)


@pytest.mark.parametrize("E,T,I", [(1, 37, 100), (3, 64, 2688), (2, 1, 48), (1, 300, 320), (2, 129, 16)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quant_act_matches_oracle(E, T, I, dtype):
    X = _acts(E, T, I, seed=T + I, dtype=dtype)
    X[0, 0, : min(I, 16)] = 0                       # an all-zero block
    r = tq.tq_quant_nvfp4_act(X)
    tq.tq_sync()
    g, sc, c, rec = _oracle_quant(host32(X))
    assert np.array_equal(r.global_scale.cpu().numpy(), g)
    assert np.array_equal(r.scales.cpu().numpy(), sc)
    assert np.array_equal(r.packed.cpu().numpy().reshape(E, -1), rec.reshape(E, -1))
    assert np.all(sc[0, 0, 0] == 0)


def test_quant_act_strided_and_zero_matrix():
    big = _acts(2, 40, 384, seed=5)
    X = big[:, 3:35, :256]                          # row stride 384, matrix stride 40 x 384
    X[1] = 0                                        # an all-zero matrix: g = 0, every code 0
    r = tq.tq_quant_nvfp4_act(X)
    tq.tq_sync()
    g, sc, c, rec = _oracle_quant(host32(X))
    assert np.array_equal(r.global_scale.cpu().numpy(), g) and g[1] == 0
    assert np.array_equal(r.scales.cpu().numpy(), sc)
    assert np.array_equal(r.packed.cpu().numpy().reshape(2, -1), rec.reshape(2, -1))


@pytest.mark.parametrize("E,rows,cols", [(1, 5, 48), (2, 300, 2688), (1, 129, 16), (3, 256, 4096)])
def test_scale_tiles_follow_the_stated_layout(E, rows, cols):
    G = (cols + 15) // 16
    rng = np.random.default_rng(rows + cols)
    sc = rng.integers(0, 127, size=(E, rows, G)).astype(np.uint8)
    out = tq.tq_nvfp4_scales_to_mma(torch.from_numpy(sc).to(DEV), E, rows, cols)
    tq.tq_sync()
    RT = 2 * -(-rows // 256)
    KC = 4 * -(-G // 16)
    assert out.numel() == E * RT * KC * 512
    ref = np.zeros((E, RT, KC, 512), np.uint8)
    for r in range(rows):
        for k in range(G):
            rr = r % 128
            ref[:, r // 128, k // 4, (rr % 32) * 16 + (rr // 32) * 4 + k % 4] = sc[:, r, k]
    assert np.array_equal(out.cpu().numpy().reshape(E, RT, KC, 512), ref)


def _gemm_bound(Xd, Wd, I):
    """(I/16 + 32) 2^-22 sum |x w| (fp32 accumulation) plus a global-scale rounding."""
    mag = np.einsum("eti,eoi->eto", np.abs(Xd), np.abs(Wd))
    return (I / 16 + 32) * 2.0 ** -22 * mag


def _run_gemm(x_rec, x_sc, gx, w_rec, w_sc, gw, E, T, O, I):
    dv = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)  # noqa: E731
    xs = tq.tq_nvfp4_scales_to_mma(dv(x_sc), E, T, I)
    ws = tq.tq_nvfp4_scales_to_mma(dv(w_sc), E, O, I)
    y = tq.tq_gemm_nvfp4(dv(x_rec), xs, dv(gx), dv(w_rec), ws, dv(gw), E, T, O, I)
    tq.tq_sync()
    return y.cpu().numpy().astype(np.float64)


def _check(y, yref, bound, label):
    bad = np.abs(y - yref) > bound + 2.0 ** -23 * np.abs(yref)
    assert not bad.any(), (label, int(bad.sum()), np.argwhere(bad)[:3], y[bad][:3], yref[bad][:3])


@pytest.mark.parametrize("E,T,O,I", [(1, 1, 1, 32), (1, 100, 37, 96), (2, 129, 300, 320), (1, 300, 256, 256),
                                     (1, 64, 513, 2688), (2, 257, 130, 64)])
def test_gemm_matches_oracle(E, T, O, I):
    rng = np.random.default_rng(T * 7 + O + I)
    Xh = host32(_acts(E, T, I, seed=O + I))
    Wh = (rng.standard_t(4, size=(E, O, I)) * 0.02).astype(np.float32)
    gx, scx, cx, recx = _oracle_quant(Xh)
    gw, scw, cw, recw = _oracle_quant(Wh)
    y = _run_gemm(recx, scx, gx, recw, scw, gw, E, T, O, I)
    Xd = np.stack([oracle.dequant_nvfp4(cx[e][None], scx[e][None], gx[e:e + 1])[0] for e in range(E)])
    Wd = np.stack([oracle.dequant_nvfp4(cw[e][None], scw[e][None], gw[e:e + 1])[0] for e in range(E)])
    for e in range(E):
        yref = oracle.gemm_nvfp4(cw[e], scw[e], gw[e], cx[e], scx[e], gx[e])
        _check(y[e], yref, _gemm_bound(Xd[e:e + 1], Wd[e:e + 1], I)[0], f"E={E} T={T} O={O} I={I} e={e}")


def test_gemm_on_searched_expert_records():
    """The NVFP4 MoE expert shape (1856 x 2688, 512 tokens) on two experts:
    weight records and block scales straight from tq_search_groups, tokens
    from tq_quant_nvfp4_act, the product checked against the oracle on the
    GPU's own codes (sampled token rows, every output row)."""
    E, T, O, I = 2, 512, 1856, 2688
    g = torch.Generator(device=DEV).manual_seed(17)
    W = (synth.student_t((E, O, I), 4, g, DEV) * 0.02).bfloat16()
    X = _acts(E, T, I, seed=18)
    m = tq.tq_imatrix(X)
    res = tq.tq_search_groups(W, m, tq.NVFP4_G16, want_idx=False, want_loss=False)
    act = tq.tq_quant_nvfp4_act(X)
    ws = tq.tq_nvfp4_scales_to_mma(res.scales.reshape(E, O, -1).contiguous(), E, O, I)
    xs = tq.tq_nvfp4_scales_to_mma(act.scales, E, T, I)
    y = tq.tq_gemm_nvfp4(act.packed, xs, act.global_scale, res.packed, ws, res.global_scale, E, T, O, I)
    tq.tq_sync()
    G = I // 16
    rows = [0, 1, 127, 128, 255, 300, 511]
    for e in range(E):
        cw = oracle.unpack_nibbles(res.packed.reshape(E, -1)[e].cpu().numpy(), O, I, 16)
        cx = oracle.unpack_nibbles(act.packed[e].reshape(-1).cpu().numpy(), T, I, 16)[rows]
        scw = res.scales[e].reshape(O, G).cpu().numpy()
        scx = act.scales[e].cpu().numpy()[rows]
        gw = float(res.global_scale[e].item())
        gx = float(act.global_scale[e].item())
        yref = oracle.gemm_nvfp4(cw, scw, gw, cx, scx, gx)
        Wd = oracle.dequant_nvfp4(cw[None], scw[None], np.array([gw], np.float32))
        Xd = oracle.dequant_nvfp4(cx[None], scx[None], np.array([gx], np.float32))
        _check(y[e].cpu().numpy().astype(np.float64)[rows], yref, _gemm_bound(Xd, Wd, I)[0], f"expert {e}")


def test_gemm_deterministic_and_refusals():
    """X X^T of quantized tokens twice: bitwise the same, symmetric within the
    accumulation bound, a non-negative diagonal; I not a multiple of 32 is
    refused before any launch."""
    E, T, I = 1, 130, 256
    X = _acts(E, T, I, seed=3)
    act = tq.tq_quant_nvfp4_act(X)
    xs = tq.tq_nvfp4_scales_to_mma(act.scales, E, T, I)
    y1 = tq.tq_gemm_nvfp4(act.packed, xs, act.global_scale, act.packed, xs, act.global_scale, E, T, T, I)
    y2 = tq.tq_gemm_nvfp4(act.packed, xs, act.global_scale, act.packed, xs, act.global_scale, E, T, T, I)
    tq.tq_sync()
    assert torch.equal(y1, y2)
    yy = y1[0].double().cpu().numpy()
    assert np.all(np.diag(yy) >= 0)
    Xd = oracle.dequant_nvfp4(oracle.unpack_nibbles(act.packed.reshape(-1).cpu().numpy(), T, I, 16)[None],
                              act.scales.cpu().numpy(), act.global_scale.cpu().numpy())
    bound = _gemm_bound(Xd, Xd, I)[0]
    assert np.all(np.abs(yy - yy.T) <= 2 * bound + 2.0 ** -22 * np.abs(yy))
    with pytest.raises(tq.TQError):
        tq.tq_gemm_nvfp4(act.packed, xs, act.global_scale, act.packed, xs, act.global_scale, E, T, T, 48)


@pytest.mark.parametrize("mag", [1e-36, 1e-20, 1e20])
def test_quant_act_extreme_magnitudes(mag):
    """Tiny (a subnormal global scale), small and huge activations: the
    nearest-code estimate switches to the IEEE quotient where the
    approximate reciprocal is not accurate; the result stays bit-exact."""
    X = (_acts(2, 33, 256, seed=9, dtype=torch.float32) * mag).contiguous()
    r = tq.tq_quant_nvfp4_act(X)
    tq.tq_sync()
    g, sc, c, rec = _oracle_quant(host32(X))
    assert np.array_equal(r.global_scale.cpu().numpy(), g)
    assert np.array_equal(r.scales.cpu().numpy(), sc)
    assert np.array_equal(r.packed.cpu().numpy().reshape(2, -1), rec.reshape(2, -1))
