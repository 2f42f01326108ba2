"""GPU parity of the group-wise row-scale format (one row scale per group of
G input columns; the "g128" reading of the FluxBin page's "2b-s16-g128"
setting) against the fp64 group-wise oracle, through the C ABI's
fb_gemv_group_scales.  Bars as for the ordinary format: bit-exact in
integer mode, else |y - y_ref| <= 1e-3 * sum_j |W_ij x_j| per row, plus the
fp32 accumulation bound (V + 96) * 2^-24 * e_i."""

import numpy as np
import pytest
import torch

import lut_binary_gemv_b200 as fb
import workloads as wl
from oracle import groupwise as GW

pytestmark = pytest.mark.gpu
DEV = "cuda"
U = 2.0 ** -24


def x_tensor(p):
    if p.x_dtype == "bf16":
        return torch.from_numpy(p.x.view(np.int16)).to(DEV).view(torch.bfloat16)
    return torch.from_numpy(p.x).to(DEV)


def reference(p, ar, G):
    """fp64 y, d = sum_j |W_ij x_j| and e = sum over bases of sum_j |a_r a_c x_j|."""
    x = p.x_f32()[0].astype(np.float64)
    sal = {}
    if p.nS:
        sal = dict(s_idx=p.s_idx, s_signs=p.s_signs(), s_alpha_r=p.s_alpha_r, s_alpha_c=p.s_alpha_c)
    y = GW.gemv(p.signs(), ar, p.alpha_c, G, x, **sal)
    W = GW.dequant(p.signs(), ar, p.alpha_c, G)
    ac = np.ones((p.K, p.N)) if p.alpha_c is None else p.alpha_c.astype(np.float64)
    grp = GW.group_of(p.N, G)
    e = np.einsum("kmn,kn->m", np.abs(ar.astype(np.float64)[:, :, grp]), np.abs(ac * x[None, :]))
    if p.nS:
        S = np.asarray(p.s_idx, np.int64)
        Ws = np.einsum("km,kt,kmt->mt", p.s_alpha_r.astype(np.float64),
                       p.s_alpha_c.astype(np.float64)[:, :p.nS], p.s_signs().astype(np.float64))
        W[:, S] += Ws
        e = e + np.einsum("km,kt->m", np.abs(p.s_alpha_r.astype(np.float64)),
                          np.abs(p.s_alpha_c.astype(np.float64)[:, :p.nS] * x[S][None, :]))
    d = np.abs(W * x[None, :]).sum(1)
    return y, d, e


def run(p, ar, G, flags=0):
    W = fb.Weights.from_problem(p)
    arg = torch.from_numpy(np.ascontiguousarray(np.transpose(ar, (0, 2, 1)))).to(DEV)   # [K][N/G][M]
    y = fb.fb_gemv_group_scales(W, G, x_tensor(p)[0], arg, flags=flags)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


def check(p, ar, G, y):
    y_ref, d, e = reference(p, ar, G)
    if p.integer_mode:
        assert np.array_equal(y, y_ref.astype(np.float32).astype(np.float64)), \
            f"integer mode not bit-exact: max diff {np.abs(y - y_ref).max()}"
        return
    err = np.abs(y - y_ref)
    assert np.all(err <= 1e-3 * d), f"tolerance: worst {np.max(err / np.maximum(d, 1e-300)):.3e}"
    V = 2 * p.K * p.N // 256 + 4 * p.Ks
    assert np.all(err <= (V + 96) * U * e + 1e-30), f"fp32 bound: worst {np.max(err / np.maximum(e, 1e-300)):.3e}"


CASES = [
    # M, N, K, nS, Ks, x dtype, G
    (4096, 4096, 2, 128, 2, "f16", 128),     # the 4096-layer workload with g128 row scales
    (70, 800, 2, 45, 2, "f16", 160 * 5),     # one group (G = N): the ordinary format
    (96, 1152, 3, 0, 2, "bf16", 128),        # N % 256 = 128: the last panel is a single half
    (100, 2048, 1, 300, 3, "f32", 512),      # groups of two panels
    (33, 512, 4, 512, 1, "f16", 128),        # every column salient
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}x{c[1]}k{c[2]}s{c[3]}G{c[6]}" for c in CASES])
@pytest.mark.parametrize("integer_mode", [False, True])
@pytest.mark.parametrize("flags", [0, 3], ids=["dependent", "independent"])
def test_group_scales_match_oracle(case, integer_mode, flags):
    M, N, K, nS, Ks, xd, G = case
    if G > N:
        G = N
    p = wl.make_problem(M, N, K, g=4, nS=nS, Ks=Ks, x_dtype=xd, alpha_dist="small", seed=(40, M, N),
                        integer_mode=integer_mode)
    ar = wl.group_row_scales(K, M, N // G, seed=(41, M, N), integer_mode=integer_mode)
    check(p, ar, G, run(p, ar, G, flags))


def test_one_group_equals_fb_gemv_bits():
    """G = N is the ordinary format: the same bits as fb_gemv."""
    p = wl.layer4096()
    W = fb.Weights.from_problem(p)
    x = x_tensor(p)[0]
    for flags in (0, 3):
        y0 = fb.fb_gemv(W, x, flags=flags)
        y1 = fb.fb_gemv_group_scales(W, p.N, x, W.alpha_r.reshape(p.K, 1, p.M).contiguous(), flags=flags)
        torch.cuda.synchronize()
        assert torch.equal(y0, y1)


def test_group_scales_rejects_bad_groups():
    p = wl.make_problem(64, 512, 2, seed=42)
    W = fb.Weights.from_problem(p)
    x = x_tensor(p)[0]
    for G in (64, 192, 384, 0, -128):   # not 128, N or a multiple of 256 dividing N
        ar = torch.ones(max(1, 2 * (512 // G if G > 0 and 512 % G == 0 else 1) * 64), device=DEV)
        with pytest.raises((fb.FbError, ValueError)):
            fb.fb_gemv_group_scales(W, G, x, ar)
