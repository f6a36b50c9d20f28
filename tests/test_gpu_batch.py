"""GPU parity of the grouped launches (tq_pack_batch, tq_dequant_batch,
tq_proxy_error_batch): several units of different shapes -- ragged column
counts, per-matrix and shared imatrix, strided weights, matrix batches -- in
one launch, each unit against the fp64 oracle exactly as the one-unit calls
are checked."""
import numpy as np
import pytest
import torch

import synth
from gpu_checks import SUM_RTOL, host32, oracle_dequant, oracle_packed, rel_close

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("group_scale_search_b200")
import oracle  # noqa: E402

DEV = "cuda"
FMTS = [tq.INT3_G64_SYM, tq.INT4_G128_ASYM, tq.INT4_G64_ASYM, tq.INT4_G32_ASYM, tq.NVFP4_G16]


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    oracle.build()
    tq.lib()


def _units(dtype, seed):
    """Weights of several shapes, one imatrix each ([n_mat, I] or shared [I])."""
    g = torch.Generator(device=DEV).manual_seed(seed)
    shapes = [(1, 37, 200), (3, 24, 1802), (1, 5, 7), (2, 64, 512), (1, 130, 4160), (4, 9, 48)]
    Ws, ms = [], []
    for k, (E, O, I) in enumerate(shapes):
        ld = (I + 7) // 8 * 8 + (8 if k % 2 else 0)   # 16-byte rows, some with padding
        W = (synth.student_t((E, O, ld), 4, g, DEV) * 0.02).to(dtype)[:, :, :I]
        Ws.append(W)
        if E > 1 and k % 2:   # per-matrix imatrix rows at a stride that is a multiple of 4
            mp = torch.zeros((E, (I + 3) // 4 * 4), dtype=torch.float32, device=DEV)
            for e in range(E):
                mp[e, :I] = synth.random_imatrix(I, 30 + 7 * k + e, DEV)
            ms.append(mp[:, :I])
        else:
            ms.append(synth.random_imatrix(I, 30 + 7 * k, DEV))
    return Ws, ms


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_batched_pack_dequant_proxy_match_oracle(fmt, dtype):
    Ws, ms = _units(dtype, 101 + fmt)
    res = [tq.tq_search_groups(W, m, fmt, want_idx=False, want_loss=False) for W, m in zip(Ws, ms)]
    zeros = [r.zeros for r in res] if res[0].zeros is not None else None
    gsc = [r.global_scale for r in res] if res[0].global_scale is not None else None
    scales = [r.scales for r in res]
    packed = tq.tq_pack_batch(Ws, fmt, scales, zeros, gsc)
    shapes = [tuple(W.shape) for W in Ws]
    dq = tq.tq_dequant_batch(packed, fmt, scales, zeros, gsc, shapes)
    dqb = tq.tq_dequant_batch(packed, fmt, scales, zeros, gsc, shapes, out_dtype=torch.bfloat16)
    px = tq.tq_proxy_error_batch(Ws, packed, fmt, scales, zeros, gsc, ms)
    torch.cuda.synchronize()
    for i, (W, m, r) in enumerate(zip(Ws, ms, res)):
        label = f"unit {i} {tuple(W.shape)} {dtype}"
        Wh = host32(W)
        gs = r.scales.cpu().numpy()
        z = r.zeros.cpu().numpy() if r.zeros is not None else None
        g = r.global_scale.cpu().numpy() if r.global_scale is not None else None
        packed_ref, codes_ref = oracle_packed(fmt, Wh, gs, z, g)
        assert np.array_equal(packed[i].cpu().numpy(), packed_ref), f"{label}: batched pack differs"
        assert np.array_equal(r.packed.cpu().numpy(), packed_ref), f"{label}: fused pack differs"
        ref = oracle_dequant(fmt, codes_ref, gs, z, g)
        assert np.array_equal(dq[i].cpu().numpy(), ref), f"{label}: batched dequant differs"
        assert torch.equal(dqb[i].cpu(), torch.from_numpy(ref).to(torch.bfloat16)), f"{label}: bf16 dequant"
        E = W.shape[0]
        mh = (m if m.dim() == 2 else m.unsqueeze(0).expand(E, -1)).cpu().numpy()
        num, den = px[i]
        for e in range(E):
            rn, rd = oracle.proxy_error(Wh[e], ref[e], mh[e])
            assert rel_close(num[e].item(), rn, SUM_RTOL) <= SUM_RTOL, f"{label}: num[{e}]"
            assert rel_close(den[e].item(), rd, SUM_RTOL) <= SUM_RTOL, f"{label}: den[{e}]"


def test_batch_of_one_equals_the_single_call():
    """A batch of one unit is the one-unit call: same records, same values,
    the same proxy sums bit for bit (same geometry, same order)."""
    Ws, ms = _units(torch.bfloat16, 7)
    W, m = Ws[1], ms[1]
    fmt = tq.INT3_G64_SYM
    r = tq.tq_search_groups(W, m, fmt, want_idx=False, want_loss=False)
    p1 = tq.tq_pack(W, fmt, r.scales)
    (pb,) = tq.tq_pack_batch([W], fmt, [r.scales])
    n1, d1 = tq.tq_proxy_error(W, r.packed, fmt, r.scales, None, None, m)
    ((nb, db),) = tq.tq_proxy_error_batch([W], [r.packed], fmt, [r.scales], None, None, [m])
    torch.cuda.synchronize()
    assert torch.equal(p1, pb)
    assert torch.equal(n1, nb) and torch.equal(d1, db)


def test_batch_argument_errors():
    W = torch.zeros((1, 8, 64), dtype=torch.bfloat16, device=DEV)
    s = torch.zeros((1, 8, 1), dtype=torch.float32, device=DEV)
    with pytest.raises(tq.TQError):
        tq.tq_pack_batch([W] * (tq.MAX_BATCH + 1), tq.INT3_G64_SYM, [s] * (tq.MAX_BATCH + 1))
    with pytest.raises(tq.TQError):   # mixed weight dtypes in one launch
        tq.tq_pack_batch([W, W.float()], tq.INT3_G64_SYM, [s, s])
    with pytest.raises(tq.TQError):   # int4 without zero-points
        tq.tq_pack_batch([W], tq.INT4_G128_ASYM, [s])


def _strided_units(seed):
    """bf16 units with padded row and matrix strides: a ragged last column
    tile, a last group shorter than the group, and a matrix batch with many
    rows per block whose row ranges cross matrices."""
    g = torch.Generator(device=DEV).manual_seed(seed)
    shapes = [(8, 1000, 512), (1, 37, 200), (2, 300, 4160), (1, 64, 2688), (3, 5, 1032)]
    Ws, ms = [], []
    for k, (E, O, I) in enumerate(shapes):
        ld = I + (8 if k % 2 == 0 else 0)
        mstride = O * ld + (64 if k % 2 == 0 else 0)
        buf = (synth.student_t((E * mstride,), 4, g, DEV) * 0.02).to(torch.bfloat16)
        Ws.append(buf.as_strided((E, O, I), (mstride, ld, 1)))
        ms.append(synth.random_imatrix(I, 50 + k, DEV))
    return Ws, ms


@pytest.mark.parametrize("fmt", FMTS)
def test_strided_pack_matches_oracle(fmt):
    """tq_pack and tq_pack_batch on strided units, bit-exact against the
    oracle's RTN and record layout, and equal to the search's fused pack."""
    Ws, ms = _strided_units(211 + fmt)
    res = [tq.tq_search_groups(W, m, fmt, want_idx=False, want_loss=False) for W, m in zip(Ws, ms)]
    zeros = [r.zeros for r in res] if res[0].zeros is not None else None
    gsc = [r.global_scale for r in res] if res[0].global_scale is not None else None
    packed = tq.tq_pack_batch(Ws, fmt, [r.scales for r in res], zeros, gsc)
    single = [tq.tq_pack(W, fmt, r.scales, r.zeros, r.global_scale) for W, r in zip(Ws, res)]
    torch.cuda.synchronize()
    for i, (W, r) in enumerate(zip(Ws, res)):
        z = r.zeros.cpu().numpy() if r.zeros is not None else None
        gl = r.global_scale.cpu().numpy() if r.global_scale is not None else None
        packed_ref, _ = oracle_packed(fmt, host32(W), r.scales.cpu().numpy(), z, gl)
        label = f"unit {i} {tuple(W.shape)} strides {W.stride()}"
        assert np.array_equal(packed[i].cpu().numpy(), packed_ref), f"{label}: batched pack differs"
        assert np.array_equal(single[i].cpu().numpy(), packed_ref), f"{label}: pack differs"
        assert torch.equal(r.packed, single[i]), f"{label}: fused pack differs from tq_pack"
