"""Canary checks (the stand-in for a memory sanitizer): every output is
written into a larger buffer filled with a sentinel, with row pitches wider
than the rows where the call allows it, and nothing outside the documented
output region may change.  Ragged sizes (M, N, nS not multiples of the tile)
are used so every kernel's edge guards are exercised."""

import numpy as np
import pytest
import torch

import lut_binary_gemv_b200 as fb
import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda"
SENT_F = -12345.5
SENT_I8 = 77
SENT_I32 = 0x5A5A5A5A


def _stream():
    return torch.cuda.current_stream().cuda_stream


def test_gemv_writes_only_its_rows():
    p = wl.make_problem(1000, 512, 2, nS=45, Ks=2, seed=51, x_dtype="f32")
    W = fb.Weights.from_problem(p)
    x = torch.from_numpy(p.x[0]).to(DEV)
    for flags in (0, fb.FB_GEMV_PDL | fb.FB_GEMV_INDEPENDENT):
        ref = fb.fb_gemv(W, x, flags=flags)
        buf = torch.full((p.M + 96,), SENT_F, device=DEV)
        fb.fb_gemv(W, x, y=buf[: p.M], flags=flags)
        torch.cuda.synchronize()
        assert bool((buf[p.M:] == SENT_F).all())
        assert torch.equal(buf[: p.M], ref)                               # the same plan: the same bits
        assert bool(torch.isfinite(buf[: p.M]).all())


def test_gemv_batched_respects_the_row_pitch():
    p = wl.make_problem(777, 256, 2, nS=0, seed=52, x_dtype="f32", batch=3)
    W = fb.Weights.from_problem(p)
    X = torch.from_numpy(p.x).to(DEV)
    ref = fb.fb_gemv_batched(W, X)
    buf = torch.full((3, p.M + 41), SENT_F, device=DEV)
    fb.fb_gemv_batched(W, X, Y=buf[:, : p.M])
    torch.cuda.synchronize()
    assert bool((buf[:, p.M:] == SENT_F).all())
    assert torch.equal(buf[:, : p.M], ref)


def test_pack_writes_only_its_words():
    K, M, N = 2, 45, 96
    signs = torch.from_numpy(np.where(np.random.default_rng(53).random((K, M, N)) < 0.5, 1, -1).astype(np.int8)).to(DEV)
    n = fb.fb_packed_words(K, M, N)
    buf = torch.full((n + 64,), SENT_I32, dtype=torch.int32, device=DEV)
    fb.fb_pack(signs, planes=buf[:n])
    torch.cuda.synchronize()
    assert bool((buf[n:] == SENT_I32).all())
    assert torch.equal(buf[:n], fb.fb_pack(signs))


def test_vcm_gather_respects_the_destination_pitch():
    nvec, n_src, nS, nS_pad, ld_dst = 5, 300, 45, 64, 80
    src = torch.randn((nvec, n_src), device=DEV)
    s_idx = torch.from_numpy(np.sort(np.random.default_rng(54).choice(n_src, nS, replace=False)).astype(np.int32)).to(DEV)
    buf = torch.full((nvec * ld_dst + 32,), SENT_F, device=DEV)
    rc = fb.lib().fb_vcm_gather(src.data_ptr(), 0, nvec, n_src, n_src, s_idx.data_ptr(), nS, nS_pad,
                                buf.data_ptr(), ld_dst, _stream())
    assert rc == 0
    torch.cuda.synchronize()
    rows = buf[: nvec * ld_dst].view(nvec, ld_dst)
    assert bool((rows[:, nS_pad:] == SENT_F).all()) and bool((buf[nvec * ld_dst:] == SENT_F).all())
    assert torch.equal(rows[:, :nS], src[:, s_idx.long()])
    assert bool((rows[:, nS:nS_pad] == 0).all())


def test_fit_base_writes_only_its_outputs():
    M, N, ldr, lds = 70, 45, 64, 50
    W = torch.from_numpy(wl.fit_inputs(M, N, T=2, seed=55).W).to(DEV)
    Rbuf = torch.full((M, ldr), SENT_F, device=DEV)
    Rbuf[:, :N] = W
    sbuf = torch.full((M, lds), SENT_I8, dtype=torch.int8, device=DEV)
    abuf = torch.full((M + 16,), SENT_F, device=DEV)
    cbuf = torch.full((N + 16,), SENT_F, device=DEV)
    fb.fb_fit_base(Rbuf[:, :N], 3, signs=sbuf[:, :N], alpha_r=abuf[:M], alpha_c=cbuf[:N])
    torch.cuda.synchronize()
    assert bool((Rbuf[:, N:] == SENT_F).all()) and bool((sbuf[:, N:] == SENT_I8).all())
    assert bool((abuf[M:] == SENT_F).all()) and bool((cbuf[N:] == SENT_F).all())
    R2 = W.clone()
    s2, a2, c2 = fb.fb_fit_base(R2, 3)
    assert torch.equal(sbuf[:, :N], s2) and torch.equal(abuf[:M], a2) and torch.equal(cbuf[:N], c2)
    assert torch.equal(Rbuf[:, :N], R2)


def test_fit_saliency_writes_only_its_outputs():
    M, N, T, nS = 33, 333, 5, 17
    fi = wl.fit_inputs(M, N, T=T, seed=56)
    Wt, Xt = torch.from_numpy(fi.W).to(DEV), torch.from_numpy(fi.X).to(DEV)
    score = torch.full((N + 16,), SENT_F, device=DEV)
    s_idx = torch.full((nS + 16,), SENT_I32, dtype=torch.int32, device=DEV)
    rc = fb.lib().fb_fit_saliency(Wt.data_ptr(), M, N, N, Xt.data_ptr(), T, N, nS, score.data_ptr(),
                                  s_idx.data_ptr(), _stream())
    assert rc == 0
    torch.cuda.synchronize()
    assert bool((score[N:] == SENT_F).all()) and bool((s_idx[nS:] == SENT_I32).all())
    sc, si = fb.fb_fit_saliency(Wt, Xt, nS)
    assert torch.equal(score[:N], sc) and torch.equal(s_idx[:nS], si)


def test_lut_build_and_unpack_write_only_their_outputs():
    K, M, N, g = 2, 45, 96, 4
    rng = np.random.default_rng(57)
    x = torch.from_numpy(rng.normal(size=N).astype(np.float32)).to(DEV)
    ac = torch.from_numpy(rng.uniform(0.5, 2.0, size=(K, N)).astype(np.float32)).to(DEV)
    n = K * (N // g) * (1 << g)
    lut = torch.full((n + 32,), SENT_F, device=DEV)
    assert fb.lib().fb_lut_build(x.data_ptr(), 0, ac.data_ptr(), K, N, g, lut.data_ptr(), _stream()) == 0
    torch.cuda.synchronize()
    assert bool((lut[n:] == SENT_F).all())
    assert torch.equal(lut[:n], fb.fb_lut_build(x, ac, K, g).reshape(-1))
    signs = torch.from_numpy(np.where(rng.random((K, M, N)) < 0.5, 1, -1).astype(np.int8)).to(DEV)
    planes = fb.fb_pack(signs)
    out = torch.full((K * M * N + 64,), SENT_I8, dtype=torch.int8, device=DEV)
    assert fb.lib().fb_unpack(planes.data_ptr(), K, M, N, out.data_ptr(), _stream()) == 0
    torch.cuda.synchronize()
    assert bool((out[K * M * N:] == SENT_I8).all())
    assert torch.equal(out[: K * M * N].view(K, M, N), signs)
