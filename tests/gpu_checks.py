"""Shared comparison helpers for the GPU parity tests (CUDA path vs oracle).

Criteria (stated by the workload definition):
  * packing and dequantization: bit-exact given the same codes and scales;
  * search: the chosen candidate equals the oracle's on >= 99.9 % of groups,
    and every group's chosen parameters have an fp64 loss within a relative
    1e-5 of the oracle's minimum (fp32 ranking against fp64 near ties);
  * imatrix and proxy error: relative 1e-5 (fp32 accumulation into fp64).
"""
import numpy as np
import torch

import group_scale_search_b200 as tq
import oracle

MATCH_MIN = 0.999
LOSS_RTOL = 1e-5
SUM_RTOL = 1e-5

ORC_FMT = {tq.INT3_G64_SYM: "int3", tq.INT4_G128_ASYM: "int4", tq.INT4_G64_ASYM: "int4", tq.INT4_G32_ASYM: "int4",
           tq.NVFP4_G16: "nvfp4"}
INT4 = {tq.INT4_G128_ASYM: 128, tq.INT4_G64_ASYM: 64, tq.INT4_G32_ASYM: 32}   # int4 formats -> group size


def host32(t: torch.Tensor) -> np.ndarray:
    """Exact fp32 host copy (bf16 widens exactly)."""
    return t.detach().float().cpu().numpy()


def oracle_search(fmt, Wh, mh):
    if fmt == tq.INT3_G64_SYM:
        s, i, L, v = oracle.search_sym_int3(Wh, mh)
        return dict(scales=s, idx=i, loss=L, codes=v)
    if fmt in INT4:
        s, z, i, L, q = oracle.search_asym_int4(Wh, mh, g=INT4[fmt])
        return dict(scales=s, zeros=z, idx=i, loss=L, codes=q)
    g, sc, i, L, c = oracle.search_nvfp4(Wh, mh)
    return dict(gscale=g, scales=sc, idx=i, loss=L, codes=c)


def loss_of_gpu_choice(fmt, Wh, mh, res):
    s = res.scales.cpu().numpy()
    if fmt == tq.INT3_G64_SYM:
        return oracle.loss_given_int3(Wh, mh, s)
    if fmt in INT4:
        return oracle.loss_given_int4(Wh, mh, s, res.zeros.cpu().numpy(), g=INT4[fmt])
    return oracle.loss_given_nvfp4(Wh, mh, s, res.global_scale.cpu().numpy())


def check_search(fmt, W: torch.Tensor, m: torch.Tensor, res, label=""):
    """Compares a GPU search result with the oracle on the same inputs."""
    Wh = host32(W if W.dim() == 3 else W.unsqueeze(0))
    mh = m.cpu().numpy()
    o = oracle_search(fmt, Wh, mh)
    gi = res.cand_idx.cpu().numpy()
    match = float((gi == o["idx"]).mean())
    assert match >= MATCH_MIN, f"{label}: candidate match {match:.5f} < {MATCH_MIN}"
    Lg = loss_of_gpu_choice(fmt, Wh, mh, res)
    Lo = o["loss"]
    over = Lg - Lo * (1 + LOSS_RTOL)
    bad = over > 1e-30
    assert not bad.any(), f"{label}: {int(bad.sum())} groups lose more than 1e-5 to the oracle minimum"
    # the GPU's reported loss is its choice's loss
    lo = res.loss.cpu().numpy().astype(np.float64)
    nz = Lg > 0
    rel = np.abs(lo[nz] - Lg[nz]) / Lg[nz]
    assert rel.size == 0 or rel.max() <= LOSS_RTOL, f"{label}: reported loss off by {rel.max():.2e}"
    assert np.all(lo[~nz] == 0)
    # same candidate => bit-identical parameters
    same = gi == o["idx"]
    gs = res.scales.cpu().numpy()
    assert np.array_equal(gs[same], o["scales"][same]), f"{label}: scale bits differ on matching groups"
    if fmt in INT4:
        assert np.array_equal(res.zeros.cpu().numpy()[same], o["zeros"][same])
    if fmt == tq.NVFP4_G16:
        assert np.array_equal(res.global_scale.cpu().numpy(), o["gscale"]), f"{label}: global scale"
    return dict(match=match, n_groups=gi.size, Wh=Wh, mh=mh, oracle=o)


def oracle_packed(fmt, Wh, scales, zeros=None, gscale=None):
    """Oracle RTN with the given parameters, then the oracle's packing."""
    E, O, I = Wh.shape
    if fmt == tq.INT3_G64_SYM:
        v = oracle.rtn_int3(Wh, scales)
        return oracle.pack_int3(v.reshape(E * O, I)), v
    if fmt in INT4:
        q = oracle.rtn_int4(Wh, scales, zeros, g=INT4[fmt])
        return oracle.pack_nibbles(q.reshape(E * O, I), INT4[fmt], zeros.reshape(E * O, -1)), q
    c = oracle.rtn_nvfp4(Wh, scales, gscale)
    return oracle.pack_nibbles(c.reshape(E * O, I), 16), c


def oracle_dequant(fmt, codes, scales, zeros=None, gscale=None):
    E, O, I = codes.shape
    if fmt == tq.INT3_G64_SYM:
        return oracle.dequant_int3(codes.reshape(E * O, I), scales.reshape(E * O, -1)).reshape(E, O, I)
    if fmt in INT4:
        return oracle.dequant_int4(codes.reshape(E * O, I), scales.reshape(E * O, -1),
                                   zeros.reshape(E * O, -1), g=INT4[fmt]).reshape(E, O, I)
    return oracle.dequant_nvfp4(codes, scales, gscale)


def rel_close(a, b, rtol):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.maximum(np.abs(b), 1e-300)
    return float(np.max(np.abs(a - b) / den)) if a.size else 0.0
