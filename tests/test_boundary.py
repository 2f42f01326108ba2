"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/fluxbin.h declares, and rejects bad arguments with
the documented status before touching the GPU."""

import ctypes as C
import os
import re

import numpy as np
import pytest

import lut_binary_gemv_b200 as fb
from lut_binary_gemv_b200 import build as fb_build
from tests.layout_spec import pack_reference

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fluxbin.h")

OK, INVALID, UNSUPPORTED, MISALIGNED, WORKSPACE, CUDA = range(6)


@pytest.fixture(scope="module")
def L():
    fb_build.build()
    return fb.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"FB_API[^;{]*?\b(fb_\w+)\s*\(", text)))


def test_header_declares_the_five_hot_path_calls():
    names = declared_functions()
    for n in ("fb_pack", "fb_lut_build", "fb_vcm_gather", "fb_gemv", "fb_gemv_batched"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 12
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing


def test_binding_constants_match_header():
    text = open(HEADER).read()
    defines = dict((n, int(v, 0)) for n, v in re.findall(r"#define\s+(FB_GEMV_\w+)\s+(0x[0-9a-fA-F]+|\d+)u", text))
    assert len(defines) == 3, f"launch flags found in the header: {sorted(defines)}"
    for name, value in defines.items():
        assert getattr(fb, name) == value, name
    enums = dict((n, int(v)) for n, v in re.findall(r"\b(FB_(?:OK|ERR_\w+))\s*=\s*(\d+)", text))
    assert enums["FB_OK"] == fb.FB_OK
    for name, value in enums.items():
        assert fb.fb_status_string(value) == name


def test_status_strings_and_version(L):
    for code, name in enumerate(["FB_OK", "FB_ERR_INVALID_VALUE", "FB_ERR_UNSUPPORTED",
                                 "FB_ERR_MISALIGNED", "FB_ERR_WORKSPACE", "FB_ERR_CUDA"]):
        assert fb.fb_status_string(code) == name
    assert L.fb_abi_version() == 1


def test_packed_words(L):
    assert fb.fb_packed_words(2, 4096, 4096) == 2 * 4096 * 4096 // 32
    assert fb.fb_packed_words(3, 33, 800) == 3 * 64 * 800 // 32
    assert fb.fb_packed_words(1, 1, 32) == 32
    for bad in [(0, 8, 32), (5, 8, 32), (1, 0, 32), (1, 8, 48), (1, 8, 0), (1, 8, 16)]:
        assert fb.fb_packed_words(*bad) == 0


FAKE = 0x10000   # an aligned non-null address; host-only calls never dereference it


def fake_weights(M=256, N=512, K=2, g=4, nS=0, Ks=2, **over):
    s = fb.FbWeightsStruct(M=M, N=N, K=K, g=g, planes=FAKE, alpha_r=FAKE, alpha_c=FAKE, nS=nS,
                           Ks=Ks if nS else 0, s_idx=FAKE if nS else None,
                           s_planes=FAKE if nS else None, s_alpha_r=FAKE if nS else None,
                           s_alpha_c=FAKE if nS else None)
    for k, v in over.items():
        setattr(s, k, v)
    return s


def ws_bytes(L, s, batch=1):
    return L.fb_gemv_workspace_bytes(C.byref(s), batch)


def test_workspace_bytes_is_zero(L):
    # partial sums live in the cluster's shared memory: no workspace needed
    assert ws_bytes(L, fake_weights(M=4096, N=4096, K=2, nS=128, Ks=2)) == 0
    assert ws_bytes(L, fake_weights(M=100, N=800, K=3), 4) == 0


@pytest.mark.parametrize("over,status", [
    (dict(g=3), INVALID), (dict(g=16), INVALID), (dict(N=48), INVALID), (dict(K=0), INVALID),
    (dict(K=5), INVALID), (dict(M=0), INVALID), (dict(planes=None), INVALID),
    (dict(alpha_r=None), INVALID), (dict(planes=FAKE + 4), MISALIGNED),
    (dict(alpha_r=FAKE + 2), MISALIGNED), (dict(alpha_c=FAKE + 1), MISALIGNED),
    (dict(nS=600), INVALID), (dict(nS=-1), INVALID),
])
def test_gemv_rejects_bad_weights(L, over, status):
    s = fake_weights(**over)
    assert L.fb_gemv(C.byref(s), FAKE, 1, FAKE, None, 0, 0, None) == status


def test_gemv_rejects_bad_salient(L):
    s = fake_weights(nS=10, Ks=0)
    assert L.fb_gemv(C.byref(s), FAKE, 1, FAKE, None, 0, 0, None) == INVALID
    s = fake_weights(nS=10, Ks=5)
    assert L.fb_gemv(C.byref(s), FAKE, 1, FAKE, None, 0, 0, None) == INVALID
    s = fake_weights(nS=10, Ks=2)
    s.s_idx = None
    assert L.fb_gemv(C.byref(s), FAKE, 1, FAKE, None, 0, 0, None) == INVALID
    s = fake_weights(nS=10, Ks=2)
    s.s_planes = FAKE + 8
    assert L.fb_gemv(C.byref(s), FAKE, 1, FAKE, None, 0, 0, None) == MISALIGNED


def test_gemv_rejects_bad_call_arguments(L):
    s = fake_weights()
    W = C.byref(s)
    assert L.fb_gemv(None, FAKE, 1, FAKE, None, 0, 0, None) == INVALID
    assert L.fb_gemv(W, None, 1, FAKE, None, 0, 0, None) == INVALID
    assert L.fb_gemv(W, FAKE, 1, None, None, 0, 0, None) == INVALID
    assert L.fb_gemv(W, FAKE, 7, FAKE, None, 0, 0, None) == INVALID      # dtype
    assert L.fb_gemv(W, FAKE, 1, FAKE, None, 0, 4, None) == INVALID      # unknown flag
    assert L.fb_gemv(W, FAKE, 1, FAKE, None, 0, 2, None) == INVALID      # INDEPENDENT needs PDL
    assert L.fb_gemv(W, FAKE + 1, 1, FAKE, None, 0, 0, None) == MISALIGNED
    assert L.fb_gemv(W, FAKE, 0, FAKE + 2, None, 0, 0, None) == MISALIGNED
    b = L.fb_gemv_batched
    assert b(W, FAKE, 1, 0, 512, FAKE, 256, None, 0, 0, None) == INVALID   # batch 0
    assert b(W, FAKE, 1, 65, 512, FAKE, 256, None, 0, 0, None) == INVALID
    assert b(W, FAKE, 1, 2, 500, FAKE, 256, None, 0, 0, None) == INVALID  # ldx < N
    assert b(W, FAKE, 1, 2, 512, FAKE, 200, None, 0, 0, None) == INVALID  # ldy < M


def test_other_entry_points_reject_bad_arguments(L):
    assert L.fb_pack(None, 1, 8, 32, FAKE, None) == INVALID
    assert L.fb_pack(FAKE, 1, 8, 40, FAKE, None) == INVALID
    assert L.fb_pack(FAKE, 1, 8, 32, FAKE + 4, None) == MISALIGNED
    assert L.fb_pack(FAKE + 1, 1, 8, 32, FAKE, None) == MISALIGNED
    assert L.fb_pack_bits(FAKE, 5, 8, 32, FAKE, None) == INVALID
    assert L.fb_unpack(FAKE, 1, 8, 32, None, None) == INVALID
    assert L.fb_lut_build(FAKE, 1, None, 2, 64, 3, FAKE, None) == INVALID
    assert L.fb_lut_build(FAKE, 9, None, 2, 64, 4, FAKE, None) == INVALID
    assert L.fb_lut_build(FAKE + 1, 1, None, 2, 64, 4, FAKE, None) == MISALIGNED
    assert L.fb_vcm_gather(FAKE, 1, 1, 64, 64, FAKE, 10, 8, FAKE, 32, None) == INVALID   # nS_pad < nS
    assert L.fb_vcm_gather(FAKE, 1, 1, 64, 32, FAKE, 10, 32, FAKE, 32, None) == INVALID  # ld_src < n_src
    assert L.fb_vcm_gather(FAKE, 1, 1, 64, 64, None, 10, 32, FAKE, 32, None) == INVALID
    assert L.fb_validate_weights(C.byref(fake_weights(g=5))) == INVALID
    assert L.fb_validate_weights(None) == INVALID
    s = fake_weights(M=64, N=512)
    for G in (64, 192, 384, 1024, 0, -128):     # not 128, N or a multiple of 256 dividing N
        assert L.fb_gemv_group_scales(C.byref(s), G, FAKE, 0, FAKE, 0, None) == INVALID
    assert L.fb_gemv_group_scales(C.byref(fake_weights(K=5)), 128, FAKE, 0, FAKE, 0, None) == INVALID


@pytest.mark.parametrize("shape", [
    (256, 256, 2, 4, 0, 0), (4096, 4096, 2, 4, 128, 2), (11008, 4096, 2, 4, 123, 2),
    (4096, 11008, 2, 4, 330, 2), (8192, 8192, 3, 8, 410, 2), (28672, 8192, 3, 8, 410, 2),
    (8192, 28672, 3, 8, 1434, 2), (131077, 64, 1, 2, 0, 0), (100, 800, 4, 1, 800, 4),
])
@pytest.mark.parametrize("batch", [1, 16, 64])
@pytest.mark.parametrize("flags", [0, 1, 3])
def test_launch_plan_covers_the_matrix(L, shape, batch, flags):
    M, N, K, g, nS, Ks = shape
    s = fake_weights(M=M, N=N, K=K, g=g, nS=nS, Ks=Ks)
    plan = fb.fb_gemv_launch_plan(s, batch, flags, 148)
    nchunks = -(-M // 32)
    P = lambda n: -(-n // 256)
    V = P(N) * K + (P(-(-nS // 32) * 32) * Ks if nS else 0)
    assert plan["V"] == V
    assert 1 <= plan["C"] <= min(16, V)
    assert plan["RB"] * plan["cpb"] >= nchunks > (plan["RB"] - 1) * plan["cpb"]
    assert plan["cpb"] <= (64 if batch == 1 and flags == 3 else 32)   # 64: large independent calls
    assert plan["warps"] == 8
    assert 0 < plan["smem"] <= 225 * 1024
    if batch > 1:                       # the row partials of a pass fit in the 64 KB table bytes
        tp = min(batch + batch % 2, 8)
        assert tp * (plan["cpb"] * 32 + 16) * 4 <= 65536


@pytest.mark.parametrize("M", [1, 32, 4096, 1 << 24])
@pytest.mark.parametrize("N", [32, 4096, 1 << 20])
@pytest.mark.parametrize("K,nS,Ks", [(1, 0, 1), (4, 0, 1), (4, -1, 4)])
@pytest.mark.parametrize("batch", [1, 2, 64])
@pytest.mark.parametrize("flags", [0, 1, 3])
def test_launch_plan_fits_at_the_abi_corners(L, M, N, K, nS, Ks, batch, flags):
    """Every plan the ABI's extreme sizes can ask for fits one CTA's shared
    memory, stays within the grid's row-block limit and covers the matrix
    (nS = -1: every column salient)."""
    nS = N if nS < 0 else nS
    s = fake_weights(M=M, N=N, K=K, g=4, nS=nS, Ks=Ks)
    plan = fb.fb_gemv_launch_plan(s, batch, flags, 148)
    nchunks = -(-M // 32)
    assert 0 < plan["smem"] <= 225 * 1024
    assert 1 <= plan["C"] <= min(16, plan["V"])
    assert plan["RB"] <= 65535
    assert plan["RB"] * plan["cpb"] >= nchunks > (plan["RB"] - 1) * plan["cpb"]


def test_launch_plan_fits_on_random_valid_arguments(L):
    """Seeded sweep over valid sizes, salient counts, batches, flags and SM
    counts (1 to 296): every plan fits one CTA's shared memory and covers the
    matrix."""
    import random
    rng = random.Random(7)
    seen = 0
    while seen < 3000:
        M = rng.choice([1, 31, 33, 4096, 11008, 131077, 1 << 24, rng.randint(1, 300000)])
        N = rng.choice([32, 96, 288, 4096, 11008, 28672, 1 << 20, 32 * rng.randint(1, 20000)])
        g = rng.choice([1, 2, 4, 8])
        nS = min(N, rng.choice([0, 0, 1, 31, 33, N // 20, N]))
        s = fake_weights(M=M, N=N, K=rng.randint(1, 4), g=g, nS=nS, Ks=rng.randint(1, 4))
        batch, flags = rng.choice([1, 2, 3, 16, 17, 64]), rng.choice([0, 1, 2, 3])
        plan = fb.fb_gemv_launch_plan(s, batch, flags, rng.choice([1, 2, 16, 132, 148, 296]))
        nchunks = -(-M // 32)
        assert 0 < plan["smem"] <= 225 * 1024, (M, N, nS, batch, flags, plan)
        assert 1 <= plan["C"] <= min(16, plan["V"]) and plan["RB"] <= 65535, (M, N, nS, batch, flags, plan)
        assert plan["RB"] * plan["cpb"] >= nchunks > (plan["RB"] - 1) * plan["cpb"]
        seen += 1


def test_launch_plan_shapes_by_call_kind(L):
    """Batch-1 calls get the 8-warp streaming CTA with rows in whole chunks
    per warp; calls flagged independent take row blocks of up to 32 chunks
    (64 from 64 MiB of packed planes); dependent calls one wave of clusters
    at two CTAs per SM, in clusters of 1, 2, 3, 4, 6, 8, 10, 12 or 16.
    Batched calls (8-warp CTAs, two tokens per pass on matrices of at most 32
    MiB of packed planes, else eight) fill the SMs' CTA slots once at most."""
    for M, N, K, g, nS, Ks in ((4096, 4096, 2, 4, 128, 2), (11008, 4096, 2, 4, 123, 2), (8192, 8192, 3, 8, 410, 2)):
        s = fake_weights(M=M, N=N, K=K, g=g, nS=nS, Ks=Ks)
        ind = fb.fb_gemv_launch_plan(s, 1, 3, 148)
        dep = fb.fb_gemv_launch_plan(s, 1, 1, 148)
        bat = fb.fb_gemv_launch_plan(s, 16, 1, 148)
        assert ind["warps"] == 8 and ind["cpb"] <= (64 if M * N * K >= 64 * 8 * 2**20 else 32)
        assert dep["warps"] == 8 and dep["cpb"] <= 32 and dep["cpb"] % 8 == 0
        assert dep["C"] * dep["RB"] <= 2 * 148 and dep["C"] in (1, 2, 3, 4, 6, 8, 10, 12, 16)
        small = M * N * K <= 32 * 8 * 2**20             # at most 32 MiB of packed planes
        passes = 8 if small else 2                       # 16 tokens: passes of 2 (three CTAs per SM) or 8
        assert bat["warps"] == 8 and bat["C"] * bat["RB"] * passes <= (3 if small else 2) * 148
        per_sm = 3 if small else 2                       # CTAs that must fit in an SM's 228 KB
        assert per_sm * (bat["smem"] + 1024) <= 228 * 1024
        assert 3 * (ind["smem"] + 1024) <= 228 * 1024 or ind["cpb"] > 32   # independent: three per SM


def test_independent_plans_keep_a_ctas_panel_list_short(L):
    """Calls flagged independent on matrices of at most 4 row blocks split
    the virtual panels so that a CTA works through at most 40 of them (one
    CTA per row block up to 40 panels, about 24 per CTA beyond); larger
    matrices keep row blocks of 32 or 64 chunks in clusters of 1 or 2."""
    for M, N, K, g, nS, Ks in ((4096, 4096, 2, 4, 128, 2), (4096, 11008, 2, 4, 330, 2), (1024, 28672, 3, 8, 1434, 2),
                               (4096, 65536, 1, 2, 0, 2), (11008, 4096, 2, 4, 123, 2), (8192, 8192, 3, 8, 410, 2)):
        s = fake_weights(M=M, N=N, K=K, g=g, nS=nS, Ks=Ks)
        plan = fb.fb_gemv_launch_plan(s, 1, 3, 148)
        if plan["RB"] <= 4 and plan["cpb"] <= 32:
            assert -(-plan["V"] // plan["C"]) <= 40 or plan["C"] == 16
            assert plan["C"] == 1 or plan["V"] > 40
        else:
            assert plan["C"] <= 2


def test_launch_plan_rejects_bad_arguments(L):
    s = fake_weights()
    out = (C.c_int * 6)()
    assert L.fb_gemv_launch_plan(C.byref(s), 1, 4, 148, C.cast(out, C.c_void_p)) == INVALID   # unknown flag
    assert L.fb_gemv_launch_plan(C.byref(s), 0, 0, 148, C.cast(out, C.c_void_p)) == INVALID   # batch 0
    assert L.fb_gemv_launch_plan(C.byref(s), 1, 0, 0, C.cast(out, C.c_void_p)) == INVALID     # sms 0
    assert L.fb_gemv_launch_plan(C.byref(s), 1, 0, 148, None) == INVALID
    assert L.fb_device_errors(None, 0) == INVALID


def test_grouped_rejects_bad_arguments(L):
    def call(structs, n, x=FAKE, ys=None, flags=0):
        arr = (C.POINTER(fb.FbWeightsStruct) * max(1, len(structs)))(*[C.pointer(s) for s in structs])
        yp = (C.c_void_p * max(1, len(structs)))(*([FAKE] * len(structs) if ys is None else ys))
        return L.fb_gemv_grouped(C.cast(arr, C.c_void_p), n, x, 1, C.cast(yp, C.c_void_p), flags, None)
    a = fake_weights()
    assert call([a, fake_weights(N=1024)], 2) == INVALID              # another N
    assert call([a, fake_weights(K=3)], 2) == INVALID                 # another K
    assert call([a, fake_weights(g=8)], 2) == INVALID                 # another g
    assert call([a, fake_weights(nS=10, Ks=2)], 2) == INVALID         # another salient format
    assert call([a] * 5, 5) == INVALID                                 # at most 4
    assert call([a], 0) == INVALID
    assert call([a, fake_weights(M=300)], 2, ys=[FAKE, None]) == INVALID
    assert call([a, fake_weights(M=300)], 2, ys=[FAKE, FAKE + 2]) == MISALIGNED
    assert call([a, fake_weights(M=300)], 2, flags=2) == INVALID       # INDEPENDENT needs PDL
    assert call([a, fake_weights(planes=FAKE + 4)], 2) == MISALIGNED
    assert L.fb_gemv_grouped(None, 1, FAKE, 1, None, 0, None) == INVALID


def test_layout_spec_is_a_bijection():
    """Every (base, row, column) lands on its own bit of the packed buffer."""
    rng = np.random.default_rng(0)
    for K, M, N in [(1, 32, 32), (2, 40, 288), (1, 64, 800), (3, 7, 416)]:
        n = K * ((M + 31) // 32 * 32) * N // 8
        seen = np.zeros(n * 8, dtype=np.int64)
        for k in range(K):
            for r in rng.choice(M, min(M, 5), replace=False):
                for c in range(N):
                    s = -np.ones((K, M, N), np.int8)
                    s[k, r, c] = 1
                    bits = np.unpackbits(pack_reference(s), bitorder="little")
                    pos = np.flatnonzero(bits)
                    assert len(pos) == 1
                    seen[pos[0]] += 1
        assert seen.max() == 1


def test_fit_calls_reject_bad_arguments(L):
    """The fitter's entry points check every argument on the host and return
    before any launch (nothing here touches a GPU)."""
    F, P = FAKE, FAKE + 4
    sal = L.fb_fit_saliency
    assert sal(None, 8, 64, 64, F, 4, 64, 3, F, F, None) == INVALID            # no W
    assert sal(F, 0, 64, 64, F, 4, 64, 3, F, F, None) == INVALID               # M = 0
    big = (1 << 20) + 1
    assert sal(F, 8, big, big, F, 4, big, 3, F, F, None) == INVALID            # N past 2^20
    assert sal(F, 8, 64, 63, F, 4, 64, 3, F, F, None) == INVALID               # ldw < N
    assert sal(F, 8, 64, 64, F, 4, 64, 65, F, F, None) == INVALID              # nS > N
    assert sal(F, 8, 64, 64, F, 4, 64, 3, F, None, None) == INVALID            # nS > 0 without s_idx
    assert sal(F + 1, 8, 64, 64, F, 4, 64, 3, F, F, None) == MISALIGNED
    base = L.fb_fit_base
    assert base(F, 8, 64, 64, 0, F, 64, F, F, None) == INVALID                 # no sweep
    assert base(F, 8, 64, 64, 1001, F, 64, F, F, None) == INVALID
    assert base(F, 8, 64, 32, 2, F, 64, F, F, None) == INVALID                 # ldr < N
    assert base(F, 8, 64, 64, 2, F, 63, F, F, None) == INVALID                 # lds < N
    assert base(None, 8, 64, 64, 2, F, 64, F, F, None) == INVALID
    assert base(F, 8, 64, 64, 2, F, 64, P + 1, F, None) == MISALIGNED


def test_fit_binding_checks_shapes_before_calling():
    """The Python fitter calls refuse wrong dtypes and shapes before reaching
    the library (CPU tensors suffice: nothing is launched)."""
    import torch
    with pytest.raises(ValueError):
        fb.fb_fit_base(torch.zeros((3, 4), dtype=torch.float64), 2)
    with pytest.raises(ValueError):
        fb.fb_fit_base(torch.zeros((3, 4)).t(), 2)                      # columns not contiguous
    with pytest.raises(ValueError):
        fb.fb_fit_saliency(torch.zeros((3, 4)), torch.zeros((2, 5)), 1)   # X has other columns
    with pytest.raises(ValueError):
        fb.fb_fit_base(torch.zeros((3, 4)), 2, signs=torch.zeros((3, 4), dtype=torch.int32))
