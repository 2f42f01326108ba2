"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Bars: bit-exact for the packers, the gather and every integer-valued-input
case; otherwise |y - y_ref| <= 1e-3 * sum_j |W_ij x_j| per row (the stated
tolerance), plus a tighter fp32 accumulation bound (V + 96) * 2^-24 * e_i
(e_i = the per-base magnitude before bases cancel, V = panels summed) that
would catch a single dropped or doubled column.
"""

import numpy as np
import pytest
import torch

import lut_binary_gemv_b200 as fb
import oracle
import workloads as wl
from tests.layout_spec import pack_reference

pytestmark = pytest.mark.gpu
DEV = "cuda"
U = 2.0 ** -24


def x_tensor(p):
    if p.x_dtype == "bf16":
        return torch.from_numpy(p.x.view(np.int16)).to(DEV).view(torch.bfloat16)
    return torch.from_numpy(p.x).to(DEV)


def panels(p):
    V = (p.N + 255) // 256 * p.K
    if p.nS:
        V += ((p.nS + 31) // 32 * 32 + 255) // 256 * p.Ks
    return V


def run_gpu(p, g=None, flags=0, W=None):
    W = fb.Weights.from_problem(p, g=g) if W is None else W
    X = x_tensor(p)
    if p.batch == 1:
        y = fb.fb_gemv(W, X[0], flags=flags)[None]
    else:
        y = fb.fb_gemv_batched(W, X, flags=flags)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


def check(p, y_gpu, rows=None):
    y_ref, d, e = oracle.problem_reference(p, rows)
    yg = y_gpu if rows is None else y_gpu[:, rows]
    if p.integer_mode:
        assert np.array_equal(yg, y_ref.astype(np.float32).astype(np.float64)), \
            f"integer mode not bit-exact: max diff {np.abs(yg - y_ref).max()}"
        return
    err = np.abs(yg - y_ref)
    assert np.all(err <= 1e-3 * d), f"tolerance: worst {np.max(err / np.maximum(d, 1e-300)):.3e}"
    tight = (panels(p) + 96) * U * e
    assert np.all(err <= tight + 1e-30), f"fp32 bound: worst {np.max(err / np.maximum(e, 1e-300)):.3e}"


def sample_rows(M, n=96, seed=0):
    rng = np.random.default_rng(seed)
    r = set(rng.choice(M, min(n, M), replace=False).tolist()) | {0, M - 1, min(31, M - 1), min(32, M - 1)}
    return np.array(sorted(r))


# --- packers, gather, tables ---------------------------------------------------

@pytest.mark.parametrize("K,M,N", [(1, 32, 32), (2, 70, 800), (3, 33, 416), (4, 1, 128), (1, 65, 4096)])
def test_pack_matches_documented_layout(K, M, N):
    rng = np.random.default_rng(K * M + N)
    signs = np.where(rng.integers(0, 2, (K, M, N)) > 0, 1, -1).astype(np.int8)
    planes = fb.fb_pack(torch.from_numpy(signs).to(DEV))
    got = planes.cpu().numpy().view(np.uint8)
    assert np.array_equal(got, pack_reference(signs))
    bits = torch.from_numpy(wl.pack_signs(signs)[..., : N // 8]).to(DEV)
    assert torch.equal(fb.fb_pack_bits(bits, N), planes)
    back = fb.fb_unpack(planes, K, M, N).cpu().numpy()
    assert np.array_equal(back, signs)


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
def test_vcm_gather_matches_oracle(dtype):
    rng = np.random.default_rng(1)
    src = torch.randn(3, 1000, device=DEV).to(dtype)
    s = np.sort(rng.choice(1000, 77, replace=False)).astype(np.int32)
    got = fb.fb_vcm_gather(src, torch.from_numpy(s).to(DEV), 96).float().cpu().numpy()
    for v in range(3):
        want = oracle.vcm_gather(src[v].float().cpu().numpy().astype(np.float64), s.astype(np.uint32), 96)
        assert np.array_equal(got[v].astype(np.float64), want)


def test_vcm_gather_out_of_range_index_gives_zero():
    src = torch.arange(64, dtype=torch.float32, device=DEV)
    s = torch.tensor([3, 64, 70, 5], dtype=torch.int32, device=DEV)
    got = fb.fb_vcm_gather(src, s, 8).cpu().numpy()
    assert got.tolist() == [3, 0, 0, 5, 0, 0, 0, 0]


@pytest.mark.parametrize("g", [1, 2, 4, 8])
@pytest.mark.parametrize("integer_mode", [False, True])
def test_lut_build_matches_oracle(g, integer_mode):
    p = wl.make_problem(8, 512, 3, x_dtype="f16", alpha_dist="unit", seed=g, integer_mode=integer_mode)
    x = x_tensor(p)[0]
    ac = torch.from_numpy(p.alpha_c).to(DEV)
    got = fb.fb_lut_build(x, ac, p.K, g).cpu().numpy().astype(np.float64)
    x64 = oracle.x_to_f64(p.x, p.x_dtype)[0]
    want = oracle.lut_tables(x64, p.alpha_c, p.K, g)
    if integer_mode:
        assert np.array_equal(got, want)
    else:
        mag = (np.abs(p.alpha_c.astype(np.float64) * x64[None, :])).reshape(p.K, -1, g).sum(-1)
        assert np.all(np.abs(got - want) <= (g + 1) * U * mag[..., None])
    none = fb.fb_lut_build(x, None, p.K, g).cpu().numpy().astype(np.float64)
    want1 = oracle.lut_tables(x64, None, p.K, g)
    assert np.all(np.abs(none - want1) <= (g + 1) * U * np.abs(x64).reshape(-1, g).sum(-1)[None, :, None])


# --- the GEMV ------------------------------------------------------------------

SMALL = [
    # M, N, K, nS, Ks, x dtype
    (70, 800, 2, 45, 2, "f16"),     # ragged rows, 32-column tail panel, ragged salient panel
    (33, 288, 3, 0, 2, "f32"),
    (1, 32, 1, 0, 2, "bf16"),
    (257, 512, 4, 512, 1, "f16"),   # every column salient
    (100, 2080, 1, 300, 3, "bf16"),  # salient panels 256 + 64
    (64, 256, 2, 1, 4, "f32"),
]


@pytest.mark.parametrize("g", [1, 2, 4, 8])
@pytest.mark.parametrize("shape", SMALL, ids=[f"{s[0]}x{s[1]}k{s[2]}s{s[3]}{s[5]}" for s in SMALL])
@pytest.mark.parametrize("integer_mode", [False, True])
@pytest.mark.parametrize("flags", [0, 3], ids=["dependent", "independent"])   # both CTA shapes
def test_gemv_small(g, shape, integer_mode, flags):
    M, N, K, nS, Ks, dt = shape
    p = wl.make_problem(M, N, K, g=g, nS=nS, Ks=Ks, x_dtype=dt, alpha_dist="unit",
                        seed=(M * 31 + N * 7 + K * 3 + nS) % 997 + g, integer_mode=integer_mode)
    check(p, run_gpu(p, flags=flags))


@pytest.mark.parametrize("flags", [0, 3], ids=["dependent", "independent"])
def test_gemv_maximum_rows(flags):
    """M = 2^24 rows (the largest M the ABI takes), one 32-column panel."""
    p = wl.make_problem(1 << 24, 32, 1, g=4, x_dtype="f16", seed=80)
    check(p, run_gpu(p, flags=flags), sample_rows(p.M, 128, 80))


@pytest.mark.parametrize("flags", [0, 3], ids=["dependent", "independent"])
def test_gemv_maximum_columns(flags):
    """N = 2^20 columns (the largest N the ABI takes): 4096 panels, 1000
    salient columns."""
    p = wl.make_problem(64, 1 << 20, 1, g=8, nS=1000, Ks=1, x_dtype="bf16", seed=81)
    check(p, run_gpu(p, flags=flags))


@pytest.mark.parametrize("fill", [0x00, 0xFF], ids=["all_minus", "all_plus"])
def test_gemv_constant_signs(fill):
    """Every weight -1 (or +1): each row is -(or +) alpha_r times the
    alpha_c-weighted sum of x; integer mode makes it exact."""
    p = wl.make_problem(300, 1056, 2, g=4, nS=70, Ks=2, x_dtype="f16", seed=82, integer_mode=True)
    p.sign_bits[...] = fill
    p.s_sign_bits[...] = fill
    check(p, run_gpu(p))
    check(p, run_gpu(p, flags=3))


def test_gemv_alpha_c_none():
    p = wl.make_problem(96, 544, 2, nS=20, Ks=2, x_dtype="f16", seed=3, alpha_c_ones=True)
    check(p, run_gpu(p))


@pytest.mark.parametrize("g", [4, 8])
def test_gemv_batched_small(g):
    p = wl.make_problem(130, 1056, 3, g=g, nS=70, Ks=2, x_dtype="f16", batch=5, seed=4)
    check(p, run_gpu(p))
    pi = wl.make_problem(130, 1056, 3, g=g, nS=70, Ks=2, x_dtype="bf16", batch=7, seed=5, integer_mode=True)
    check(pi, run_gpu(pi))


@pytest.mark.parametrize("batch", [2, 3, 16])
@pytest.mark.parametrize("flags", [0, 3])
def test_gemv_batched_tokens(batch, flags):
    """Batched calls at full panels, narrow salient tails and both plans
    (dependent and independent), odd and even batches."""
    p = wl.make_problem(1000, 2304, 2, g=4, nS=300, Ks=2, x_dtype="f16", batch=batch, seed=50 + batch)
    check(p, run_gpu(p, flags=flags))
    pi = wl.make_problem(700, 1312, 3, g=8, nS=45, Ks=2, x_dtype="bf16", batch=batch, seed=60 + batch,
                         integer_mode=True)
    check(pi, run_gpu(pi, flags=flags))


def test_gemv_batched_max_batch():
    p = wl.make_problem(40, 256, 1, g=4, x_dtype="f32", batch=64, seed=6)
    check(p, run_gpu(p))


def test_gemv_many_rows():
    p = wl.make_problem(131077, 64, 1, g=8, x_dtype="f16", seed=7)
    y = run_gpu(p)
    check(p, y, sample_rows(p.M, 200))


def test_gemv_zero_x_gives_zero():
    p = wl.make_problem(64, 512, 2, nS=10, Ks=2, x_dtype="f32", seed=8)
    p.x[:] = 0
    assert np.all(run_gpu(p) == 0)


def test_gemv_deterministic_and_pdl():
    p = wl.layer4096()
    W = fb.Weights.from_problem(p)
    a = run_gpu(p, W=W)
    b = run_gpu(p, W=W)
    c = run_gpu(p, W=W, flags=fb.FB_GEMV_PDL)
    assert np.array_equal(a, b) and np.array_equal(a, c)


def test_interleaved_weights_and_flags():
    """Different weight sets back to back, with every flag combination."""
    p1 = wl.make_problem(300, 1024, 2, nS=40, Ks=2, x_dtype="f16", seed=9)
    p2 = wl.make_problem(500, 512, 3, g=8, x_dtype="f32", seed=10)
    W1, W2 = fb.Weights.from_problem(p1), fb.Weights.from_problem(p2)
    for flags in (0, fb.FB_GEMV_PDL, fb.FB_GEMV_PDL | fb.FB_GEMV_INDEPENDENT):
        for _ in range(3):
            y1 = fb.fb_gemv(W1, x_tensor(p1)[0], flags=flags)
            y2 = fb.fb_gemv(W2, x_tensor(p2)[0], flags=flags)
        torch.cuda.synchronize()
        check(p1, y1.cpu().numpy()[None].astype(np.float64))
        check(p2, y2.cpu().numpy()[None].astype(np.float64))


def test_independent_chain_in_graph_matches():
    """Independent calls overlap each other; results must not change."""
    ps = [wl.make_problem(700, 1280, 2, nS=33, Ks=2, x_dtype="f16", seed=20 + i) for i in range(6)]
    Ws = [fb.Weights.from_problem(p) for p in ps]
    xs = [x_tensor(p)[0] for p in ps]
    ys = [torch.full((p.M,), float("nan"), device=DEV) for p in ps]
    s = torch.cuda.Stream()
    flags = fb.FB_GEMV_PDL | fb.FB_GEMV_INDEPENDENT
    with torch.cuda.stream(s):
        for W, x, y in zip(Ws, xs, ys):
            fb.fb_gemv(W, x, y=y, flags=flags)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for _ in range(2):
                for W, x, y in zip(Ws, xs, ys):
                    fb.fb_gemv(W, x, y=y, flags=flags)
    for y in ys:
        y.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    for p, y in zip(ps, ys):
        check(p, y.cpu().numpy()[None].astype(np.float64))


def test_plain_and_pdl_graphs_give_the_same_bits():
    """A graph of ordinary launches (flags 0) and one with programmatic
    dependent launch compute the same bits for a chain of mixed shapes."""
    ps = [wl.make_problem(M, N, 2, nS=nS, Ks=2, x_dtype="f16", seed=40 + i)
          for i, (M, N, nS) in enumerate(((512, 1024, 31), (1100, 512, 16), (256, 2304, 70)))]
    Ws = [fb.Weights.from_problem(p) for p in ps]
    xs = [x_tensor(p)[0] for p in ps]
    s = torch.cuda.Stream()
    outs = []
    for flags in (0, fb.FB_GEMV_PDL):
        ys = [torch.full((p.M,), float("nan"), device=DEV) for p in ps]
        with torch.cuda.stream(s):
            for W, x, y in zip(Ws, xs, ys):
                fb.fb_gemv(W, x, y=y, flags=flags)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                for _ in range(2):
                    for W, x, y in zip(Ws, xs, ys):
                        fb.fb_gemv(W, x, y=y, flags=flags)
        for y in ys:
            y.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        outs.append([y.cpu().numpy() for y in ys])
    for p, a, b in zip(ps, *outs):
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
        check(p, a[None].astype(np.float64))


def test_gemv_in_cuda_graph():
    p = wl.make_problem(1000, 2048, 2, nS=60, Ks=2, x_dtype="f16", seed=11)
    W = fb.Weights.from_problem(p)
    x = x_tensor(p)[0]
    y = torch.empty(p.M, device=DEV)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        fb.fb_gemv(W, x, y=y, flags=fb.FB_GEMV_PDL)     # warm-up outside capture
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for _ in range(3):
                fb.fb_gemv(W, x, y=y, flags=fb.FB_GEMV_PDL)
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    check(p, y.cpu().numpy()[None].astype(np.float64))


def test_invalid_salient_index_reads_nothing():
    p = wl.make_problem(64, 256, 2, nS=8, Ks=2, x_dtype="f32", seed=12)
    W = fb.Weights.from_problem(p)
    assert fb.fb_validate_weights(W) == 0
    bad = W.s_idx.clone()
    bad[3] = 100000
    Wb = fb.Weights(p.M, p.N, p.K, p.g, W.planes, W.alpha_r, W.alpha_c, p.nS, p.Ks, bad, W.s_planes,
                    W.s_alpha_r, W.s_alpha_c)
    assert fb.fb_validate_weights(Wb) == 1
    y = fb.fb_gemv(Wb, x_tensor(p)[0])
    torch.cuda.synchronize()
    p.s_alpha_c[:, 3] = 0          # the column with the bad index contributes nothing
    check(p, y.cpu().numpy()[None].astype(np.float64))
    unsorted = W.s_idx.flip(0).contiguous()
    Wu = fb.Weights(p.M, p.N, p.K, p.g, W.planes, W.alpha_r, W.alpha_c, p.nS, p.Ks, unsorted, W.s_planes,
                    W.s_alpha_r, W.s_alpha_c)
    assert fb.fb_validate_weights(Wu) == 1


# --- grouped calls (several matrices of one format reading one x) ------------

@pytest.mark.parametrize("flags", [0, 1, 3])
def test_grouped_qkv_and_gate_up(flags):
    """q, k, v of a 7B layer in one launch, and gate, up (another M) in one
    launch; each result against the oracle with the shared x."""
    for ms in ((0, 1, 2), (4, 5)):
        ps = [wl.step7b_matrix(2, m) for m in ms]
        for p in ps[1:]:
            p.x = ps[0].x            # one x for the group
        Ws = [fb.Weights.from_problem(p) for p in ps]
        x = x_tensor(ps[0])[0]
        ys = fb.fb_gemv_grouped(Ws, x, flags=flags)
        torch.cuda.synchronize()
        for p, y in zip(ps, ys):
            check(p, y.cpu().numpy()[None].astype(np.float64), sample_rows(p.M, 96, 3))


def test_grouped_equals_single_calls_and_ragged_rows():
    """Matrices of different M (ragged last row blocks) in one launch give the
    bits of separate calls with the same plan."""
    ps = [wl.make_problem(M, 1280, 2, nS=45, Ks=2, x_dtype="f16", seed=40 + i) for i, M in enumerate((700, 33, 1000, 64))]
    for p in ps[1:]:
        p.x = ps[0].x
    Ws = [fb.Weights.from_problem(p) for p in ps]
    x = x_tensor(ps[0])[0]
    ys = fb.fb_gemv_grouped(Ws, x)
    torch.cuda.synchronize()
    for p, y in zip(ps, ys):
        check(p, y.cpu().numpy()[None].astype(np.float64))
    one = fb.fb_gemv_grouped(Ws[:1], x)[0]
    torch.cuda.synchronize()
    assert torch.equal(one, ys[0])


def test_grouped_in_graph_with_pdl():
    ps = [wl.step7b_matrix(7, m) for m in (4, 5)]
    ps[1].x = ps[0].x
    Ws = [fb.Weights.from_problem(p) for p in ps]
    x = x_tensor(ps[0])[0]
    ys = [torch.full((p.M,), float("nan"), device=DEV) for p in ps]
    s = torch.cuda.Stream()
    flags = fb.FB_GEMV_PDL | fb.FB_GEMV_INDEPENDENT
    with torch.cuda.stream(s):
        fb.fb_gemv_grouped(Ws, x, ys, flags=flags)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for _ in range(3):
                fb.fb_gemv_grouped(Ws, x, ys, flags=flags)
    for y in ys:
        y.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    for p, y in zip(ps, ys):
        check(p, y.cpu().numpy()[None].astype(np.float64), sample_rows(p.M, 64, 9))


# --- the five workloads ----------------------------------------------------------

@pytest.mark.parametrize("integer_mode", [False, True])
def test_workload_tiny(integer_mode):
    p = wl.tiny(integer_mode)
    check(p, run_gpu(p))


@pytest.mark.parametrize("integer_mode", [False, True])
def test_workload_layer4096(integer_mode):
    p = wl.layer4096(integer_mode)
    y = run_gpu(p)
    check(p, y)
    check(p, run_gpu(p, g=8))
    # the launch the bench times: PDL + independent (its own plan)
    check(p, run_gpu(p, flags=fb.FB_GEMV_PDL | fb.FB_GEMV_INDEPENDENT))


@pytest.mark.parametrize("integer_mode", [False, True])
def test_workload_ternary(integer_mode):
    p = wl.ternary11008(integer_mode)
    y = run_gpu(p)
    check(p, y)
    check(p, run_gpu(p, flags=fb.FB_GEMV_PDL | fb.FB_GEMV_INDEPENDENT))
    if integer_mode:    # against the dense ternary matvec itself
        xi = p.x_f32()[0].astype(np.int64)
        want = 2.0 * p.alpha_r[0].astype(np.float64) * (p.ternary.astype(np.int64) @ xi)
        assert np.array_equal(y[0], want)


def test_workload_7b_step():
    indep = fb.FB_GEMV_PDL | fb.FB_GEMV_INDEPENDENT
    for m in range(len(wl.STEP7B_MATRICES)):
        p = wl.step7b_matrix(0, m)
        check(p, run_gpu(p))
        check(p, run_gpu(p, flags=indep))
    for layer in (13, 31):
        for m in range(len(wl.STEP7B_MATRICES)):
            p = wl.step7b_matrix(layer, m)
            check(p, run_gpu(p), sample_rows(p.M, 64, layer * 7 + m))
    pi = wl.step7b_matrix(5, 6, integer_mode=True)
    check(pi, run_gpu(pi))


@pytest.mark.parametrize("shape_index", [0, 1, 2])
@pytest.mark.parametrize("batch", wl.BATCHES70B)
def test_workload_70b(shape_index, batch):
    p = wl.layer70b(shape_index, batch)
    check(p, run_gpu(p), sample_rows(p.M, 64, shape_index))
    if batch == 4:
        pi = wl.layer70b(shape_index, batch, integer_mode=True)
        check(pi, run_gpu(pi), sample_rows(pi.M, 64, 10 + shape_index))


@pytest.mark.parametrize("batch", [1, 16])
def test_workload_70b_every_row(batch):
    """The 28672 x 8192 layer (K = 3, g = 8, 5% salient) checked on every
    row of every token, in both launch plans of batch-1 calls."""
    p = wl.layer70b(1, batch)
    check(p, run_gpu(p))
    if batch == 1:
        check(p, run_gpu(p, flags=fb.FB_GEMV_PDL | fb.FB_GEMV_INDEPENDENT))


@pytest.mark.gpu
def test_device_error_flags_stay_clear():
    # every bounded wait for a weight copy in the runs above ended in time
    p = wl.layer4096()
    W = fb.Weights.from_problem(p)
    fb.fb_gemv(W, torch.from_numpy(p.x[0]).cuda(), flags=fb.FB_GEMV_PDL | fb.FB_GEMV_INDEPENDENT)
    assert fb.fb_device_errors(clear=True) == 0


def test_bounded_wait_runs_out_and_reports():
    """The failure path of the weight-copy waits: with no copy issued, each
    wait gives up after its bound, the rows come back NaN, the device error
    flag is raised, and the next call on the same context is correct."""
    p = wl.make_problem(96, 512, 1, g=4, x_dtype="f32", seed=70)
    W = fb.Weights.from_problem(p)
    x = x_tensor(p)[0]
    assert fb.fb_device_errors(clear=True) == 0
    y = fb.fb_gemv(W, x, flags=fb.FB_GEMV_TEST_WAIT_TIMEOUT)
    torch.cuda.synchronize()
    assert torch.isnan(y).all()
    assert fb.fb_device_errors(clear=True) == 1
    assert fb.fb_device_errors(clear=True) == 0
    check(p, run_gpu(p, W=W))
    assert fb.fb_device_errors(clear=True) == 0

