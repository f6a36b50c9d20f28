"""Full-size parity: each workload at its full size, run exactly as bench.py
runs it (one call per unit over all matrices), checked against the oracle on
outputs it can compute one by one -- 2048 whole sampled rows of every unit
(search choice and loss, scales, packed records, dequantized weights),
sampled imatrix columns, and the proxy error of one whole matrix per unit --
and the stand-alone pack against the fused one on whole tensors."""
import numpy as np
import pytest
import torch

import synth
from gpu_checks import LOSS_RTOL, MATCH_MIN, SUM_RTOL, host32, oracle_dequant, oracle_packed, rel_close

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("group_scale_search_b200")
import oracle  # noqa: E402

DEV = "cuda"
RECORD = {tq.INT3_G64_SYM: 24, tq.INT4_G128_ASYM: 64, tq.NVFP4_G16: 8}
GROUP = {tq.INT3_G64_SYM: 64, tq.INT4_G128_ASYM: 128, tq.NVFP4_G16: 16}


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    oracle.build()
    tq.lib()


def _sample_rows(E, O, n, seed):
    rng = np.random.default_rng(seed)
    rows = {(0, 0), (E - 1, O - 1), (E // 2, O // 2)}
    n = min(n, E * O)
    while len(rows) < n:
        rows.add((int(rng.integers(E)), int(rng.integers(O))))
    return sorted(rows)


def _check_unit(u, m_full, res, n_rows, seed, gscale_oracle=None):
    fmt = tq.FORMATS[u.fmt]
    E, O, I = u.W.shape
    g = GROUP[fmt]
    G = (I + g - 1) // g
    rows = _sample_rows(E, O, n_rows, seed)
    idx = torch.tensor([e * O + o for e, o in rows], device=DEV)
    Wh = host32(u.W.reshape(E * O, I)[idx]).reshape(len(rows), 1, I)
    mh = m_full.reshape(-1, I).cpu().numpy()
    mrows = np.stack([mh[e if mh.shape[0] > 1 else 0] for e, _ in rows])     # one imatrix per sampled row
    gi = res.cand_idx.reshape(E * O, G)[idx].cpu().numpy()
    gs = res.scales.reshape(E * O, G)[idx].cpu().numpy()
    gz = res.zeros.reshape(E * O, G)[idx].cpu().numpy() if res.zeros is not None else None
    if fmt == tq.INT3_G64_SYM:
        s, oi, L, v = oracle.search_sym_int3(Wh, mrows)
        Lg = oracle.loss_given_int3(Wh, mrows, gs.reshape(len(rows), 1, G))
    elif fmt == tq.INT4_G128_ASYM:
        s, z, oi, L, q = oracle.search_asym_int4(Wh, mrows)
        Lg = oracle.loss_given_int4(Wh, mrows, gs.reshape(len(rows), 1, G), gz.reshape(len(rows), 1, G))
    else:
        grow = np.array([gscale_oracle[e] for e, _ in rows], np.float32)
        assert np.array_equal(res.global_scale.cpu().numpy(), gscale_oracle), "global scale"
        _, s, oi, L, c = oracle.search_nvfp4(Wh, mrows, gscale=grow)
        Lg = oracle.loss_given_nvfp4(Wh, mrows, gs.reshape(len(rows), 1, G), grow)
    oi = oi.reshape(len(rows), G)
    L = L.reshape(len(rows), G)
    Lg = Lg.reshape(len(rows), G)
    match = float((gi == oi).mean())
    assert match >= MATCH_MIN, f"{u.name}: match {match}"
    assert np.all(Lg <= L * (1 + LOSS_RTOL) + 1e-30), f"{u.name}: loss above the oracle minimum"
    same = gi == oi
    assert np.array_equal(gs[same], s.reshape(len(rows), G)[same])
    lo = res.loss.reshape(E * O, G)[idx].cpu().numpy()
    nz = Lg > 0
    assert np.max(np.abs(lo[nz] - Lg[nz]) / Lg[nz]) <= LOSS_RTOL
    # packed records and dequantized weights of the sampled rows, bit-exact
    rec = RECORD[fmt]
    packed = res.packed.reshape(E * O, G * rec)[idx].cpu().numpy()
    if fmt == tq.NVFP4_G16:
        ref_packed, codes = oracle_packed(fmt, Wh, gs.reshape(len(rows), 1, G), gscale=grow)
    else:
        ref_packed, codes = oracle_packed(fmt, Wh, gs.reshape(len(rows), 1, G),
                                          None if gz is None else gz.reshape(len(rows), 1, G))
    assert np.array_equal(packed.reshape(-1), ref_packed), f"{u.name}: packed records"
    return rows, idx, codes, gs, gz, (grow if fmt == tq.NVFP4_G16 else None), match


def _run_workload(name, n_rows=2048, seed=0):
    wl = synth.make(name, DEV)
    ms = {}
    for sname, site in wl.sites.items():
        m = tq.tq_imatrix(site.X)
        torch.cuda.synchronize()
        # sampled columns of every site's imatrix
        I = site.X.shape[2]
        cols = torch.tensor(sorted(set(np.random.default_rng(seed).integers(0, I, 96).tolist()) | {0, I - 1}),
                            device=DEV)
        for e in {0, site.X.shape[0] - 1}:
            Xs = host32(site.X[e][:, cols])
            ref = oracle.imatrix(Xs)
            assert rel_close(m[e][cols].cpu().numpy(), ref, SUM_RTOL) <= SUM_RTOL, f"{name}/{sname} imatrix"
        ms[sname] = m
    out = []
    for k, u in enumerate(wl.units):
        fmt = tq.FORMATS[u.fmt]
        m = ms[u.site]
        m = m if u.W.shape[0] > 1 else m[0]
        res = tq.tq_search_groups(u.W, m, fmt)
        E, O, I = u.W.shape
        dq = tq.tq_dequant(res.packed, fmt, res.scales, res.zeros, res.global_scale, E, O, I)
        num, den = tq.tq_proxy_error(u.W, res.packed, fmt, res.scales, res.zeros, res.global_scale, m)
        torch.cuda.synchronize()
        gso = None
        if fmt == tq.NVFP4_G16:   # per-tensor global scales, one expert at a time
            gso = np.concatenate([oracle.nvfp4_global(host32(u.W[e:e + 1])) for e in range(E)])
        rows, idx, codes, gs, gz, grow, match = _check_unit(u, m, res, n_rows, seed + k, gso)
        # stand-alone RTN + pack with the searched scales: the whole tensor, bit for bit
        p2 = tq.tq_pack(u.W, fmt, res.scales, res.zeros, res.global_scale)
        torch.cuda.synchronize()
        assert torch.equal(p2, res.packed), f"{name}/{u.name}: tq_pack differs from the fused pack"
        del p2
        # dequantized weights of the sampled rows, bit-exact
        ref = oracle_dequant(fmt, codes, gs.reshape(len(rows), 1, -1),
                             None if gz is None else gz.reshape(len(rows), 1, -1), grow)
        assert np.array_equal(dq.reshape(E * O, I)[idx].cpu().numpy(), ref.reshape(len(rows), I)), \
            f"{name}/{u.name}: dequant"
        # proxy error of one whole matrix against the oracle
        e = E - 1
        We = host32(u.W[e])
        G = res.scales.shape[-1]
        se = res.scales[e].cpu().numpy()
        if fmt == tq.INT3_G64_SYM:
            What = oracle.dequant_int3(oracle.rtn_int3(We, se), se)
        elif fmt == tq.INT4_G128_ASYM:
            ze = res.zeros[e].cpu().numpy()
            What = oracle.dequant_int4(oracle.rtn_int4(We, se, ze), se, ze)
        else:
            ce = oracle.rtn_nvfp4(We[None], se[None], gso[e:e + 1])
            What = oracle.dequant_nvfp4(ce, se[None], gso[e:e + 1])[0]
        me = (m[e] if m.dim() == 2 else m).cpu().numpy()
        rn, rd = oracle.proxy_error(We, What, me)
        assert rel_close(num[e].item(), rn, SUM_RTOL) <= SUM_RTOL, f"{name}/{u.name}: proxy num"
        assert rel_close(den[e].item(), rd, SUM_RTOL) <= SUM_RTOL, f"{name}/{u.name}: proxy den"
        assert 0.0 < num[e].item() < den[e].item()
        out.append((u.name, match, len(rows) * ((I + GROUP[fmt] - 1) // GROUP[fmt])))
        del res, dq
    return out


@pytest.mark.parametrize("name", ["c0", "c1", "c2", "c3", "c4"])
def test_full_size_workload(name):
    """Every unit at full size: 2048 sampled rows (every row where the unit
    has fewer) checked against the oracle group by group."""
    results = _run_workload(name)
    assert results
    for unit, match, groups in results:
        print(f"{name}/{unit}: candidate match {match:.5f} over {groups} sampled groups")


@pytest.mark.parametrize("name", ["c1", "c3"])
def test_full_size_hessian(name):
    """tq_hessian on the first unit's full calibration activations (c1: 2048 x
    4096; c3: 65,536 tokens x 5120), launched as bench.py launches it: sampled
    entries (the diagonal corners, tile edges, random) against the oracle one
    by one within the fp32 accumulation bound, exact symmetry of the whole H,
    and its diagonal against the imatrix of the same activations."""
    wl = synth.make(name, DEV)
    u = [x for x in wl.units if x.timed][0]
    X = wl.sites[u.site].X[0]
    T, I = X.shape
    H = tq.tq_hessian(X)
    tq.tq_sync()
    assert torch.equal(H, H.T)
    Xh = X.float().cpu().numpy()
    Ah = np.abs(Xh)
    rng = np.random.default_rng(7)
    pairs = {(0, 0), (I - 1, I - 1), (0, I - 1), (127, 128), (128, 127), (I // 2, I // 3)}
    while len(pairs) < 300:
        pairs.add((int(rng.integers(I)), int(rng.integers(I))))
    Hh = H.cpu().numpy()
    for i, j in sorted(pairs):
        ref = oracle.hessian_entry(Xh, i, j)
        bound = (T / 16 + 32) * 2.0 ** -22 * oracle.hessian_entry(Ah, i, j)
        assert abs(float(Hh[i, j]) - ref) <= bound, (i, j, float(Hh[i, j]), ref, bound)
    m = tq.tq_imatrix(X)[0]
    tq.tq_sync()
    d = np.diag(Hh).astype(np.float64) / T
    assert np.allclose(d, m.cpu().numpy().astype(np.float64), rtol=(T / 16 + 64) * 2.0 ** -22, atol=0)


def test_full_size_proxy_full():
    """tq_proxy_error_full on the dense int4-g128 4096 x 4096 workload (2048
    calibration tokens), launched as bench.py launches it: the whole-matrix
    call equals the sum of the calls on its 128-token blocks (each output tile
    of X E^T is computed the same way in both) to fp64 rounding, and two
    sampled 128-token x 256-row tiles match the oracle's tr(E H E^T),
    tr(W H W^T) within the fp32 accumulation bound."""
    wl = synth.make("c1", DEV)
    u = [x for x in wl.units if x.timed][0]
    X = wl.sites[u.site].X[0]
    W = u.W
    fmt = tq.FORMATS[u.fmt]
    m = tq.tq_imatrix(X)[0]
    res = tq.tq_search_groups(W, m, fmt)
    num, den = tq.tq_proxy_error_full(X, W, res.packed, fmt, res.scales, res.zeros, res.global_scale)
    tq.tq_sync()
    T, I = X.shape
    O = W.shape[1]
    sn = sd = 0.0
    for t0 in range(0, T, 128):
        a, b = tq.tq_proxy_error_full(X[t0:t0 + 128], W, res.packed, fmt, res.scales, res.zeros, res.global_scale)
        sn += a.item()
        sd += b.item()
    tq.tq_sync()
    assert abs(num.item() - sn) <= 1e-12 * sn and abs(den.item() - sd) <= 1e-12 * sd
    assert 0.0 < num.item() < den.item()
    G = I // 128
    for t0, o0 in [(0, 0), (T - 128, O - 256)]:
        Wt = W[:, o0:o0 + 256]
        sc, z = res.scales.view(1, O, G)[:, o0:o0 + 256], res.zeros.view(1, O, G)[:, o0:o0 + 256]
        pk = res.packed.view(O, -1)[o0:o0 + 256]
        a, b = tq.tq_proxy_error_full(X[t0:t0 + 128], Wt, pk, fmt, sc.contiguous(), z.contiguous(), None)
        tq.tq_sync()
        Wh = host32(Wt)[0]
        codes = oracle.rtn_int4(Wh[None], sc.cpu().numpy(), z.cpu().numpy(), g=128)
        What = oracle_dequant(fmt, codes, sc.cpu().numpy(), z.cpu().numpy())[0]
        Xh = host32(X[t0:t0 + 128])
        rn, rd = oracle.proxy_error_full(Wh, What, oracle.hessian(Xh))
        X64, E64, W64 = Xh.astype(np.float64), Wh.astype(np.float64) - What, Wh.astype(np.float64)
        for got, ref, M, K, extra in [(a.item(), rn, E64, 2 * I, 2.0 ** -15), (b.item(), rd, W64, I, 0.0)]:
            D = ((K / 16 + 32) * 2.0 ** -22 + extra) * (np.abs(X64) @ np.abs(M).T)
            bound = float(np.sum((2 * np.abs(X64 @ M.T) + D) * D))
            assert abs(got - ref) <= bound + 1e-12 * ref, (t0, o0, got, ref, bound)


def test_full_size_gptq_sweep():
    """tq_gptq_sweep on the dense int4-g128 4096 x 4096 workload with the
    search's scales and the factor of its calibration Hessian (damped by 1 %
    of the mean diagonal; fp64 Cholesky and inverse by the library, outside
    the method), launched as bench.py launches it: sampled whole rows (the
    first, the last, a CTA's 16th and random ones) bit for bit against the
    oracle's sweep of the same rows, and a lower proxy error tr(E H E^T) than
    round-to-nearest with the same scales."""
    wl = synth.make("c1", DEV)
    u = [x for x in wl.units if x.timed][0]
    X = wl.sites[u.site].X[0]
    W = u.W
    fmt = tq.FORMATS[u.fmt]
    m = tq.tq_imatrix(X)[0]
    res = tq.tq_search_groups(W, m, fmt)
    H = X.double().T @ X.double()
    H += 0.01 * H.diagonal().mean() * torch.eye(H.shape[0], device=DEV, dtype=torch.float64)
    U = torch.linalg.cholesky(torch.cholesky_inverse(torch.linalg.cholesky(H)), upper=True).float().contiguous()
    codes, loss = tq.tq_gptq_sweep(W, fmt, res.scales, res.zeros, U)
    tq.tq_sync()
    O, I = W.shape[1], W.shape[2]
    rng = np.random.default_rng(5)
    rows = sorted({0, 15, 16, O - 1, *rng.integers(0, O, 5).tolist()})
    Uh, Wh = U.cpu().numpy(), host32(W[0])
    sc = res.scales.reshape(O, -1).cpu().numpy()
    zz = res.zeros.reshape(O, -1).cpu().numpy()
    c_ref, l_ref = oracle.gptq_sweep(Wh[rows], 4, sc[rows], zz[rows], Uh, g=128)
    assert np.array_equal(codes[0, rows].cpu().numpy(), c_ref)
    assert np.array_equal(loss[0, rows].cpu().numpy(), l_ref)
    # the sweep's purpose, on the whole matrix: a lower tr(E H E^T) than RTN with the same scales
    Hf = H - 0.01 * H.diagonal().mean() * torch.eye(I, device=DEV, dtype=torch.float64)
    wq = tq.tq_dequant(tq.tq_pack_codes(codes.view(torch.uint8), fmt, res.zeros.reshape(O, -1)), fmt, res.scales,
                       res.zeros, None, 1, O, I)
    wr = tq.tq_dequant(res.packed, fmt, res.scales, res.zeros, None, 1, O, I)
    tq.tq_sync()
    pe = lambda Wq: float(torch.einsum("oi,ij,oj->", W[0].double() - Wq[0].double(), Hf,  # noqa: E731
                                       W[0].double() - Wq[0].double()))
    assert pe(wq) < pe(wr)
