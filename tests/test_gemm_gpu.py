"""GPU parity of the CUDA path (through the C ABI) against the fp64 oracle.

Bar (stated with the target): every output within
    |y - y_ref| <= 1e-2 + 2e-3 |y_ref|
for fp16 outputs with fp32 accumulation.  Inputs are the seeded synthetic
recipe of bit_gemv_bcq_b200/synth.py.  Sizes: the five workload shapes (some
at full size, the 70B-like ones on sampled output rows), plus small and
ragged shapes spanning several row-blocks, K-blocks and split-K CTAs.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_gemv_bcq_b200 import api, synth

pytestmark = pytest.mark.gpu

ATOL, RTOL = 1e-2, 2e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    api.lib()
    yield
    assert api.device_error() == api.BCQ_OK


def _weights(prob):
    return api.BcqWeights.from_canonical(prob.planes, prob.alphas, prob.z)


def _x(prob):
    return torch.from_numpy(prob.x.view(np.int16)).view(torch.float16).cuda()


def _check(y_gpu, y_ref, what=""):
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    err = np.abs(y - y_ref)
    bound = ATOL + RTOL * np.abs(y_ref)
    bad = err > bound
    assert not bad.any(), (
        f"{what}: {bad.sum()} of {bad.size} outside tolerance; worst "
        f"err {err.max():.3e} at {np.unravel_index(err.argmax(), err.shape)}")
    return float(err.max())


def _run(prob, w=None, p=None, p_row=None):
    w = _weights(prob) if w is None else w
    y = w.gemm(_x(prob), p=p, p_row=p_row)
    torch.cuda.synchronize()
    return y


# --------------------------------------------------------------- small / ragged

@pytest.fixture(params=["lut", "sync", "tcgen05"])
def path(request, monkeypatch):
    """Run a test through one of the kernels for every batch size: the
    lookup-table kernel, the mma.sync tensor-core kernel or the tcgen05 one."""
    monkeypatch.setenv("BCQ_MMA_MIN_ROWS", "1000" if request.param == "lut" else "1")
    if request.param != "lut":
        monkeypatch.setenv("BCQ_MMA_KIND", request.param)
    return request.param


@pytest.mark.parametrize("N,K", [(1, 128), (31, 384), (33, 640), (100, 1024),
                                 (256, 512), (1000, 2048), (64, 128 * 33)])
@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 9, 16, 17])
def test_parity_small_and_ragged(N, K, M, path):
    prob = synth.make_problem(N, K, M, seed=N + K + M, precisions=(1, 2, 3, 4))
    w = _weights(prob)
    for p in (1, 2, 3, 4):
        y = _run(prob, w, p=p)
        _check(y, oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p=p),
               f"N={N} K={K} M={M} p={p}")


def test_parity_tiny_config_all_precisions():
    """256 x 512, M = 1, p = 2, 3, 4, seed 0 (the tiny workload)."""
    prob = synth.make_problem(256, 512, 1, seed=0)
    w = _weights(prob)
    for p in (2, 3, 4):
        _check(_run(prob, w, p=p), oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p=p))


def test_parity_attention_projection_full():
    """4096 x 4096, M = 1, p = 2, 3, 4 (every output)."""
    prob = synth.make_problem(4096, 4096, 1, seed=1)
    w = _weights(prob)
    for p in (2, 3, 4):
        _check(_run(prob, w, p=p), oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p=p),
               f"p={p}")


@pytest.mark.parametrize("N,K", [(14336, 4096), (4096, 14336)])
def test_parity_mlp_decode_with_outliers_full(N, K):
    """Llama-3.1-8B MLP shapes, M = 1, 0.1 % outlier channels x 20."""
    prob = synth.make_problem(N, K, 1, seed=2, outliers=True)
    w = _weights(prob)
    for p in (2, 3, 4):
        _check(_run(prob, w, p=p), oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p=p),
               f"{N}x{K} p={p}")


@pytest.mark.parametrize("N,K", [(4096, 4096), (14336, 4096)])
def test_parity_batch_sweep(N, K, path):
    """M in {1, 2, 4, 8, 16}, p = 2, 3, 4, all outputs."""
    prob = synth.make_problem(N, K, 16, seed=3)
    w = _weights(prob)
    for M in (1, 2, 4, 8, 16):
        sub = synth.Problem(x=prob.x[:M], planes=prob.planes, alphas=prob.alphas, z=prob.z)
        for p in (2, 3, 4):
            y = _run(sub, w, p=p)
            _check(y, oracle.gemm(sub.x, prob.planes, prob.alphas, prob.z, p=p), f"M={M} p={p}")


@pytest.mark.parametrize("N,K", [(4096, 4096), (1000, 2048), (14336, 4096)])
def test_parity_wide_batches(N, K, path):
    """17 to 64 rows of one precision: one tcgen05 launch of up to 64 rows (the
    lookup kernel in pairs; 32 rows at two bits are two 16-row launches), and
    mixed precisions that split into groups of more and of fewer than 16 rows."""
    prob = synth.make_problem(N, K, 64, seed=4)
    w = _weights(prob)
    for M in (17, 32, 33, 64):
        sub = synth.Problem(x=prob.x[:M], planes=prob.planes, alphas=prob.alphas, z=prob.z)
        for p in (2, 4):
            y = _run(sub, w, p=p)
            _check(y, oracle.gemm(sub.x, prob.planes, prob.alphas, prob.z, p=p), f"M={M} p={p}")
    p_row = np.array([2] * 40 + [3] * 5 + [4] * 19, dtype=np.int32)
    y = _run(prob, w, p_row=p_row)
    _check(y, oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p_row=p_row), "mixed 64")


@pytest.mark.parametrize("N,K", [(28672, 8192), (8192, 28672)])
def test_parity_mixed_precision_70b_every_output(N, K):
    """M = 8 rows with p drawn from {2,3,4}: one launch that streams the
    planes once up to the largest precision; every output checked."""
    prob = synth.make_problem(N, K, 8, seed=4, mixed=True)
    assert set(prob.p_row.tolist()) <= {2, 3, 4} and len(set(prob.p_row.tolist())) > 1
    assert api.route_query(8, N, K, p_row=prob.p_row) == [("mma_mixed", 8, int(prob.p_row.max()))]
    y = _run(prob, p_row=prob.p_row)
    ref = oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p_row=prob.p_row)
    _check(y, ref, f"{N}x{K} mixed")


@pytest.mark.parametrize("N,K", [(1000, 2048), (14336, 4096), (300, 128 * 33)])
@pytest.mark.parametrize("M", [3, 5, 8, 9, 16])
def test_parity_mixed_batches_in_one_launch(N, K, M):
    """Per-request precision inside one tensor-core launch (rows of 1 to 4
    bits), including precision-1 rows and rows past a multiple of 8."""
    prob = synth.make_problem(N, K, M, seed=30 + M + N, precisions=(1, 2, 3, 4), mixed=True)
    rng = np.random.default_rng(M * 7 + N)
    prob.p_row[:] = rng.integers(1, 5, size=M)
    prob.p_row[0], prob.p_row[-1] = 1, 4   # at least two precisions, 4 the largest
    assert api.route_query(M, N, K, p_row=prob.p_row) == [("mma_mixed", M, 4)]
    y = _run(prob, p_row=prob.p_row)
    _check(y, oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p_row=prob.p_row),
           f"N={N} K={K} M={M}")


def test_parity_large_mixed_batch_with_leftovers():
    """22 rows: a group of one precision on the tensor cores, the rows left
    over in every group sharing one mixed launch."""
    prob = synth.make_problem(4096, 4096, 22, seed=33, mixed=True)
    prob.p_row[:] = [2] * 18 + [3] * 2 + [4] * 2
    rng = np.random.default_rng(34)
    rng.shuffle(prob.p_row)
    r = api.route_query(22, 4096, 4096, p_row=prob.p_row)
    assert ("mma_mixed", 6, 4) in r
    y = _run(prob, p_row=prob.p_row)
    _check(y, oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p_row=prob.p_row))


def test_four_row_launch_with_a_row_map_in_one_k_block():
    """K = 256 (one K-block: results stored directly, no split-K) and a
    four-row lookup launch that takes rows 1, 3, 5 of the batch."""
    prob = synth.make_problem(300, 256, 20, seed=35, mixed=True)
    prob.p_row[:] = [2, 4, 2, 4, 2, 4] + [2] * 14
    r = api.route_query(20, 300, 256, p_row=prob.p_row)
    assert ("lut_four", 3, 4) in r
    y = _run(prob, p_row=prob.p_row)
    _check(y, oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p_row=prob.p_row))


# ------------------------------------------------------------------ invariants

def test_p_prefix_poisoned_planes_are_never_read(path):
    """Planes p..p_H-1 replaced by random bits: bitwise identical output."""
    prob = synth.make_problem(1000, 2048, 3, seed=5, precisions=(1, 2, 3, 4))
    w = _weights(prob)
    rng = np.random.default_rng(50)
    for p in (1, 2, 3):
        y1 = _run(prob, w, p=p)
        poisoned = prob.planes.copy()
        poisoned[p:] = rng.integers(0, 2**32, size=poisoned[p:].shape, dtype=np.uint32)
        w2 = api.BcqWeights.from_canonical(poisoned, prob.alphas, prob.z)
        y2 = _run(prob, w2, p=p)
        assert torch.equal(y1, y2), f"p={p}"


def test_results_are_reproducible(path):
    prob = synth.make_problem(14336, 4096, 2, seed=6)
    w = _weights(prob)
    ys = [_run(prob, w, p=3) for _ in range(3)]
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2])


def test_mixed_rows_match_uniform_calls(path):
    prob = synth.make_problem(4096, 4096, 8, seed=7, mixed=True)
    prob.p_row[:] = [4, 2, 3, 3, 2, 4, 2, 3]
    w = _weights(prob)
    y = _run(prob, w, p_row=prob.p_row)
    for m, q in enumerate(prob.p_row):
        one = synth.Problem(x=prob.x[m:m + 1], planes=prob.planes, alphas=prob.alphas, z=prob.z)
        ym = _run(one, w, p=int(q))
        assert (y[m].float() - ym[0].float()).abs().max().item() <= 2 * ATOL
    _check(y, oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p_row=prob.p_row))


def test_sign_symmetry():
    prob = synth.make_problem(512, 1024, 1, seed=8)
    y = _run(prob, p=4)
    flipped = prob.planes.copy()
    flipped[1] = ~flipped[1]
    al = {q: a.copy() for q, a in prob.alphas.items()}
    al[4][:, :, 1] = -al[4][:, :, 1]
    y2 = _run(synth.Problem(x=prob.x, planes=flipped, alphas=al, z=prob.z), p=4)
    assert (y.float() - y2.float()).abs().max().item() <= 2 * ATOL


def test_fewer_stored_planes_and_no_offset():
    prob = synth.make_problem(300, 768, 2, seed=9, p_H=2, precisions=(1, 2))
    w = api.BcqWeights.from_canonical(prob.planes, prob.alphas, None)
    for p in (1, 2):
        y = _run(prob, w, p=p)
        _check(y, oracle.gemm(prob.x, prob.planes, prob.alphas, None, p=p), f"p={p}")


def test_hand_example_through_the_gpu():
    """The BiLoCo hand example: x = [0.5, -1.2, 2.0, 0.3], v = [+1,-1,+1,-1],
    v.x = 3.4 (K = 128, p = 1, alpha = 1, z = 0)."""
    x = np.zeros((1, 128), dtype=np.float16)
    x[0, :4] = [0.5, -1.2, 2.0, 0.3]
    planes = np.zeros((1, 1, 4), dtype=np.uint32)
    planes[0, 0, 0] = 0b0101
    alphas = {1: np.ones((1, 1, 1), dtype=np.float16)}
    prob = synth.Problem(x=x, planes=planes, alphas=alphas, z=np.zeros((1, 1), np.float16))
    y = _run(prob, p=1)
    assert abs(float(y[0, 0]) - 3.4) < 2e-3


def test_empty_batch():
    prob = synth.make_problem(64, 256, 1, seed=10)
    w = _weights(prob)
    y = w.gemm(torch.empty((0, 256), dtype=torch.float16, device="cuda"), p=2)
    assert y.shape == (0, 64)


# -------------------------------------------------- steps of the path (a1, a2)

@pytest.mark.parametrize("M,K", [(1, 128), (1, 4096), (2, 640), (3, 384), (4, 1024)])
def test_lut_and_group_sums_match_oracle(M, K):
    x = synth.make_x(M, K, seed=K + M)
    lut, gs = api.build_lut(torch.from_numpy(x.view(np.int16)).view(torch.float16).cuda())
    torch.cuda.synchronize()
    ref = oracle.lut(x)
    # each entry is a sum of 8 fp16 values in fp32: a few ulps of |sum|
    err = np.abs(lut.cpu().numpy().astype(np.float64) - ref)
    assert err.max() <= 1e-5 * (1 + np.abs(ref).max())
    gref = oracle.group_sums(x)
    assert np.abs(gs.cpu().numpy() - gref).max() <= 1e-4 * (1 + np.abs(gref).max())


# ---------------------------------------------------------------- host path

def test_host_buffers_path_matches_device_path():
    prob = synth.make_problem(4096, 4096, 4, seed=11)
    w = _weights(prob)
    y_dev_ref = _run(prob, w, p=3)
    x_host = torch.from_numpy(prob.x.view(np.int16)).view(torch.float16).pin_memory()
    y_host = torch.empty((4, 4096), dtype=torch.float16).pin_memory()
    x_dev = torch.empty((4, 4096), dtype=torch.float16, device="cuda")
    y_dev = torch.empty((4, 4096), dtype=torch.float16, device="cuda")
    api.gemm_host(x_host, w, y_host, x_dev, y_dev, p=3)
    torch.cuda.synchronize()
    assert torch.equal(y_host, y_dev_ref.cpu())


def test_binding_rejects_buffers_of_the_wrong_size_before_any_launch():
    """The kernels write through raw pointers: the binding checks every
    caller-given buffer's shape before it calls the library."""
    prob = synth.make_problem(256, 512, 2, seed=12)
    w = _weights(prob)
    x = _x(prob)
    dev = x.device
    bad_out = [torch.empty((2, 255), dtype=torch.float16, device=dev),
               torch.empty((1, 256), dtype=torch.float16, device=dev),
               torch.empty((2, 256), dtype=torch.float32, device=dev)]
    for out in bad_out:
        with pytest.raises(ValueError):
            api.gemm(x, w, p=2, out=out)
        with pytest.raises(ValueError):
            api.gemm_noalloc(x, w, p=2, out=out)
    with pytest.raises(ValueError):
        api.gemm(x[:, :384].contiguous(), w, p=2)
    x_host = x.cpu().pin_memory()
    y_host = torch.empty((2, 256), dtype=torch.float16).pin_memory()
    x_dev = torch.empty((2, 512), dtype=torch.float16, device=dev)
    y_dev = torch.empty((2, 256), dtype=torch.float16, device=dev)
    for args in [(x_host, torch.empty((2, 255), dtype=torch.float16), x_dev, y_dev),
                 (x_host, y_host, x_dev[:1], y_dev),
                 (x_host, y_host, x_dev, y_dev[:1]),
                 (x_host[:, :256].contiguous(), y_host, x_dev, y_dev)]:
        with pytest.raises(ValueError):
            api.gemm_host(args[0], w, args[1], args[2], args[3], p=2)
    torch.cuda.synchronize()
    assert api.device_error() == api.BCQ_OK
    # the right buffers still work
    api.gemm_host(x_host, w, y_host, x_dev, y_dev, p=2)
    torch.cuda.synchronize()
    assert torch.equal(y_host, api.gemm(x, w, p=2).cpu())


# ------------------------------------------------------------- bounded waits

def test_bounded_wait_reports_timeout_and_context_survives():
    assert api.device_error() == api.BCQ_OK
    api.debug_wait_timeout(20000)          # 20 ms on a barrier nothing completes
    assert api.device_error() == api.BCQ_ERR_TIMEOUT
    assert api.device_error() == api.BCQ_OK   # read clears it
    prob = synth.make_problem(256, 512, 1, seed=12)
    _check(_run(prob, p=2), oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p=2))


# ------------------------------------------------- launch shapes and workspace

@pytest.mark.parametrize("C,D,NP", [(1, 2, 1), (3, 4, 2), (7, 6, 2), (13, 2, 2), (148, 8, 2)])
def test_forced_launch_shapes(monkeypatch, C, D, NP, path):
    """Few CTAs (each spanning several K-blocks, groups cut at K-block
    boundaries), shallow and deep rings, one or two producer warps."""
    monkeypatch.setenv("BCQ_FORCE_C", str(C))
    monkeypatch.setenv("BCQ_FORCE_D", str(D))
    monkeypatch.setenv("BCQ_FORCE_NP", str(NP))
    prob = synth.make_problem(1000, 2048, 3, seed=20 + C, mixed=True)
    prob.p_row[:] = [4, 2, 3]
    w = _weights(prob)
    _check(_run(prob, w, p_row=prob.p_row),
           oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p_row=prob.p_row), f"C={C}")
    for p in (2, 4):
        _check(_run(prob, w, p=p), oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p=p),
               f"C={C} p={p}")


def test_workspace_is_left_zero_filled(path):
    prob = synth.make_problem(4096, 4096, 2, seed=21)
    w = _weights(prob)
    for p in (2, 3):
        _run(prob, w, p=p)
    ws = api.workspace(2, 4096, 4096, "cuda")
    torch.cuda.synchronize()
    assert ws is not None and int(ws.count_nonzero()) == 0


def test_concurrent_calls_on_two_streams(path):
    """Two calls at the same time on two streams, each with its own
    workspace, a few rounds without synchronising in between: both results
    match the oracle and no wait ran out.  (Each GEMV grid is launched
    cooperatively: its CTAs are resident together, so the split-K polling of
    one grid never waits for a CTA that the other grid keeps off the SMs.)"""
    a = synth.make_problem(14336, 4096, 1, seed=26)
    b = synth.make_problem(4096, 14336, 5, seed=27, mixed=True)
    wa, wb = _weights(a), _weights(b)
    xa, xb = _x(a), _x(b)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    outs = []
    for _ in range(4):
        ya = torch.empty((1, 14336), dtype=torch.float16, device="cuda")
        yb = torch.empty((5, 4096), dtype=torch.float16, device="cuda")
        with torch.cuda.stream(s1):
            wa.gemm(xa, p=3, out=ya, stream=s1)
        with torch.cuda.stream(s2):
            wb.gemm(xb, p_row=b.p_row, out=yb, stream=s2)
        outs.append((ya, yb))
    torch.cuda.synchronize()
    assert api.device_error(s1) == api.BCQ_OK and api.device_error(s2) == api.BCQ_OK
    ra = oracle.gemm(a.x, a.planes, a.alphas, a.z, p=3)
    rb = oracle.gemm(b.x, b.planes, b.alphas, b.z, p_row=b.p_row)
    for ya, yb in outs:
        _check(ya, ra, "stream 1")
        _check(yb, rb, "stream 2")


@pytest.mark.parametrize("mode", [1, 2])
def test_programmatic_dependent_launch_gives_the_same_bits(mode, path):
    """Back-to-back calls with PDL (and early plane streaming) equal the plain
    stream-ordered results bit for bit."""
    prob = synth.make_problem(14336, 4096, 2, seed=22)
    w = _weights(prob)
    x = _x(prob)
    ref = [w.gemm(x[:1], p=2), w.gemm(x, p=3), w.gemm(x[1:], p=4)]
    torch.cuda.synchronize()
    try:
        api.set_pdl(mode)
        for _ in range(3):
            got = [w.gemm(x[:1], p=2), w.gemm(x, p=3), w.gemm(x[1:], p=4)]
        torch.cuda.synchronize()
    finally:
        api.set_pdl(0)
    for a, b in zip(ref, got):
        assert torch.equal(a, b)


def test_workspace_shared_across_shapes(path):
    """One workspace serves calls of different shapes in turn."""
    a = synth.make_problem(4096, 4096, 2, seed=23)
    b = synth.make_problem(14336, 4096, 1, seed=24)
    wa, wb = _weights(a), _weights(b)
    for _ in range(2):
        _check(_run(a, wa, p=3), oracle.gemm(a.x, a.planes, a.alphas, a.z, p=3), "4096")
        _check(_run(b, wb, p=2), oracle.gemm(b.x, b.planes, b.alphas, b.z, p=2), "14336")


def test_both_paths_agree_with_each_other(monkeypatch):
    """The lookup-table and tensor-core kernels compute the same sums (fp32,
    different order): within the parity bound of each other on a full-size
    batch of 16 rows of mixed precision."""
    prob = synth.make_problem(14336, 4096, 16, seed=25, mixed=True)
    w = _weights(prob)
    monkeypatch.setenv("BCQ_MMA_MIN_ROWS", "1000")
    y_lut = _run(prob, w, p_row=prob.p_row)
    monkeypatch.setenv("BCQ_MMA_MIN_ROWS", "1")
    for kind in ("sync", "tcgen05"):
        monkeypatch.setenv("BCQ_MMA_KIND", kind)
        y_mma = _run(prob, w, p_row=prob.p_row)
        d = (y_lut.float() - y_mma.float()).abs()
        assert (d <= ATOL + RTOL * y_lut.float().abs()).all(), kind
