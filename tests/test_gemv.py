"""GPU bandwidth kernel (M = 1..8) against the fp64 oracle, element by element.

Tolerance: |y - y_ref| <= 2e-3 * sum_k |x_k w_k| + 1e-5 (helpers.check_close).
"""
import os

import numpy as np
import pytest
import torch

from helpers import check_close, np_inputs

pytestmark = pytest.mark.gpu
NCPU = os.cpu_count() or 1


@pytest.fixture(scope="module")
def T():
    from ternary_weight_only_b200 import build
    build.build()
    from ternary_weight_only_b200 import tern
    yield tern
    for o in (1, 2, 3, 4, 5, 6, 7):
        tern.tern_set_option(o, 0)


def run_case(T, orc, x, codes, scales, what="", threads=None, workspace=None):
    """Pack with the oracle (host), run the GPU product on those slots, compare."""
    xn, cn, sn = np_inputs(x, codes, scales)
    slots, sc, bad, _ = orc.pack(cn, sn)
    assert bad == 0
    yd = T.tern_gemm(x.cuda(), torch.from_numpy(slots).cuda(), scales.cuda(), workspace=workspace)
    torch.cuda.synchronize()
    y_ref, bound = orc.matmul(xn, slots, sc, threads=threads or NCPU)
    return check_close(yd, y_ref, bound, what)


def test_tiny_gemv(T, orc):
    from ternary_weight_only_b200 import synth
    x, codes, scales = synth.tiny_gemv()
    xn, cn, sn = np_inputs(x, codes, scales)
    slots, sc, _, _ = orc.pack(cn, sn)
    y = T.tern_gemv(x[0].cuda(), torch.from_numpy(slots).cuda(), scales.cuda())
    torch.cuda.synchronize()
    y_ref, bound = orc.matmul(xn, slots, sc)
    check_close(y.view(1, -1), y_ref, bound, "tiny")


@pytest.mark.parametrize("i", range(7))
def test_decode_layer_projection(T, orc, i):
    from ternary_weight_only_b200 import synth
    x, codes, scales = synth.decode_proj(i)
    run_case(T, orc, x, codes, scales, synth.LAYER_PROJ[i][0])


@pytest.mark.parametrize("M", [2, 4, 8])
@pytest.mark.parametrize("i", range(7))
def test_verify_batch(T, orc, i, M):
    from ternary_weight_only_b200 import synth
    x, codes, scales = synth.decode_proj(i, M=M)
    run_case(T, orc, x, codes, scales, f"{synth.LAYER_PROJ[i][0]} M={M}")


@pytest.mark.parametrize("M,K,N", [
    (1, 128, 1), (1, 128, 17), (3, 256, 5), (8, 384, 33), (5, 640, 100), (1, 1152, 129),
    (2, 2048, 250), (7, 128, 16), (1, 4096, 1000), (6, 17408, 40), (8, 17408, 300),
    (4, 25600, 64),
])
def test_ragged(T, orc, M, K, N):
    from ternary_weight_only_b200 import synth
    x, codes, scales = synth.case(M, K, N, seed=M * 1000 + K + N, codes="sparse", outlier_p=0.01)
    run_case(T, orc, x, codes, scales, f"M={M} K={K} N={N}")


@pytest.mark.parametrize("variant", [2])
@pytest.mark.parametrize("ks", [1, 2, 4, 8])
@pytest.mark.parametrize("cl", [1, 2, 4])
def test_split_options(T, orc, ks, cl, variant):
    """Every forced k split inside the CTA and across a cluster, TMA-staged kernel."""
    from ternary_weight_only_b200 import synth
    x, codes, scales = synth.case(3, 17408, 200, seed=ks * 10 + cl, codes="sparse")
    T.tern_set_option(T.TERN_OPT_GEMV_VARIANT, variant)
    T.tern_set_option(T.TERN_OPT_GEMV_KSPLIT, ks)
    T.tern_set_option(T.TERN_OPT_GEMV_CLUSTER, cl)
    try:
        run_case(T, orc, x, codes, scales, f"v{variant} ks={ks} cl={cl}")
        x1, c1, s1 = synth.case(1, 17408, 1040, seed=ks * 10 + cl + 1, codes="sparse")
        run_case(T, orc, x1, c1, s1, f"M=1 v{variant} ks={ks} cl={cl}")
    finally:
        T.tern_set_option(T.TERN_OPT_GEMV_KSPLIT, 0)
        T.tern_set_option(T.TERN_OPT_GEMV_CLUSTER, 0)
        T.tern_set_option(T.TERN_OPT_GEMV_VARIANT, 0)


@pytest.fixture
def tc(T):
    """Select the tcgen05 bandwidth kernel for the duration of a test."""
    T.tern_set_option(T.TERN_OPT_GEMV_VARIANT, 3)
    yield T
    T.tern_set_option(T.TERN_OPT_GEMV_VARIANT, 0)


@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("K,N", [(128, 1), (384, 130), (5120, 1024), (6144, 5120), (17408, 640), (1152, 4000)])
def test_tensor_core_split_and_whole(tc, orc, M, K, N):
    """The tcgen05 kernel with its K split (cached workspace) and without (no workspace)."""
    from ternary_weight_only_b200 import synth
    x, codes, scales = synth.case(M, K, N, seed=M * 7 + K + N, codes="sparse", outlier_p=0.01)
    run_case(tc, orc, x, codes, scales, f"tc split M={M} K={K} N={N}")
    run_case(tc, orc, x, codes, scales, f"tc whole M={M} K={K} N={N}", workspace=False)


@pytest.mark.parametrize("M", [1, 2, 4])
@pytest.mark.parametrize("i", range(7))
def test_tensor_core_decode_layer(tc, orc, i, M):
    from ternary_weight_only_b200 import synth
    x, codes, scales = synth.decode_proj(i, M=M)
    run_case(tc, orc, x, codes, scales, f"tc {synth.LAYER_PROJ[i][0]} M={M}")


def test_workspace_shared_by_shapes(tc, orc):
    """One workspace serves calls of different shapes in turn (the counters of a
    larger call never land on a smaller call's leftover partial sums)."""
    from ternary_weight_only_b200 import synth
    shapes = [(2, 6144, 5120), (2, 5120, 17408), (1, 17408, 5120), (4, 5120, 1024), (2, 5120, 17408)]
    need = max(tc.tern_workspace_bytes(M, N, K) for M, K, N in shapes)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for i, (M, K, N) in enumerate(shapes):
        x, codes, scales = synth.case(M, K, N, seed=500 + i, codes="sparse")
        run_case(tc, orc, x, codes, scales, f"shared ws M={M} K={K} N={N}", workspace=ws)


def test_split_is_deterministic_and_workspace_reusable(tc, orc):
    T = tc
    """Repeated calls sharing one workspace give bit-identical results (fixed
    reduction order, counters reset by every call)."""
    from ternary_weight_only_b200 import synth
    x, codes, scales = synth.case(1, 17408, 5120, seed=99, codes="sparse")
    xd, cd, sd = x.cuda(), codes.cuda(), scales.cuda()
    slots, sc = T.tern_pack_g128(cd, sd)
    need = T.tern_workspace_bytes(1, 5120, 17408)
    assert need > 0
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    ys = [T.tern_gemv(xd[0], slots, sc, workspace=ws).clone() for _ in range(4)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(y.view(torch.int16), ys[0].view(torch.int16))
    assert int(ws[: 128 * 1024].view(torch.int32).abs().sum().item()) == 0  # counters back to zero
    xn, cn, sn = np_inputs(x, codes, scales)
    ref_slots, ref_sc, _, _ = orc.pack(cn, sn)
    y_ref, bound = orc.matmul(xn, ref_slots, ref_sc, threads=NCPU)
    check_close(ys[0].view(1, -1), y_ref, bound, "deterministic split")


@pytest.mark.parametrize("variant", [3, 2])
def test_variant_grouped_layer(T, orc, variant):
    from ternary_weight_only_b200 import synth
    T.tern_set_option(T.TERN_OPT_GEMV_VARIANT, variant)
    try:
        mats, refs = [], []
        for i in range(7):
            x, codes, scales = synth.decode_proj(i, M=2)
            xn, cn, sn = np_inputs(x, codes, scales)
            slots, sc, _, _ = orc.pack(cn, sn)
            y = torch.full((2, codes.shape[0]), float("nan"), dtype=torch.float16, device="cuda")
            mats.append((x.cuda(), torch.from_numpy(slots).cuda(), scales.cuda(), y))
            refs.append((xn, slots, sc))
        T.tern_gemv_grouped(mats, 2)
        torch.cuda.synchronize()
        for i, ((xn, slots, sc), m) in enumerate(zip(refs, mats)):
            y_ref, bound = orc.matmul(xn, slots, sc, threads=NCPU)
            check_close(m[3], y_ref, bound, f"v{variant} grouped {synth.LAYER_PROJ[i][0]}")
    finally:
        T.tern_set_option(T.TERN_OPT_GEMV_VARIANT, 0)


def test_timeout_path_reports_and_recovers(T, orc):
    """A TMA wait that can never complete (nothing is loaded) gives up after its
    limit; the status reaches the host and the context stays usable."""
    from ternary_weight_only_b200 import synth
    x, codes, scales = synth.case(2, 2048, 700, seed=78, codes="sparse")
    xn, cn, sn = np_inputs(x, codes, scales)
    slots, sc, _, _ = orc.pack(cn, sn)
    xd, sd, scd = x.cuda(), torch.from_numpy(slots).cuda(), scales.cuda()
    for variant in (3, 2):
        T.tern_set_option(T.TERN_OPT_GEMV_VARIANT, variant)
        T.tern_set_option(T.TERN_OPT_TEST_STALL_US, 2000)
        try:
            T.tern_gemm(xd, sd, scd)
            with pytest.raises(T.TernError) as ei:
                T.tern_sync_status()
            assert ei.value.status == T.TERN_ERR_TIMEOUT
        finally:
            T.tern_set_option(T.TERN_OPT_TEST_STALL_US, 0)
            T.tern_set_option(T.TERN_OPT_GEMV_VARIANT, 0)
        T.tern_reset_workspaces()
        T.tern_sync_status()
        run_case(T, orc, x, codes, scales, f"after timeout v{variant}")


def test_grid_cap(T, orc):
    """TMA-staged kernel with few resident CTAs: every CTA walks many tiles."""
    from ternary_weight_only_b200 import synth
    x, codes, scales = synth.case(1, 1024, 4000, seed=3, codes="sparse")
    T.tern_set_option(T.TERN_OPT_GEMV_VARIANT, 2)
    T.tern_set_option(T.TERN_OPT_GEMV_CTAS, 1)
    try:
        run_case(T, orc, x, codes, scales, "one CTA per SM")
    finally:
        T.tern_set_option(T.TERN_OPT_GEMV_CTAS, 0)
        T.tern_set_option(T.TERN_OPT_GEMV_VARIANT, 0)


def test_exact_special_cases(T, orc):
    """Zero codes give exactly 0; a single non-zero per row gives s*t*x within
    fp16 output rounding; all +1 codes with unit scales give row sums."""
    from ternary_weight_only_b200 import synth
    M, K, N = 4, 1024, 48
    x, codes, scales = synth.case(M, K, N, seed=41)
    z = torch.zeros_like(codes)
    slots, _ = T.tern_pack_g128(z.cuda(), scales.cuda())
    y = T.tern_gemm(x.cuda(), slots, scales.cuda())
    torch.cuda.synchronize()
    assert torch.all(y == 0)
    one = torch.zeros_like(codes)
    for n in range(N):
        one[n, (n * 37 + 5) % K] = 1 if n % 2 else -1
    run_case(T, orc, x, one, scales, "single non-zero")
    ones = torch.ones_like(codes)
    unit = torch.ones_like(scales)
    xs = (torch.randn(M, K) * 0.05).half()  # keep row sums inside fp16 range
    run_case(T, orc, xs, ones, unit, "row sums")


def test_adversarial_accumulation(T, orc):
    """Same-sign terms: x all +1 or with x20 outliers, codes all +1 in a group."""
    M, K, N = 8, 2048, 64
    codes = torch.ones((N, K), dtype=torch.int8)
    codes[N // 2:, 128:] = -1
    scales = torch.full((N, K // 128), 0.0499).half()
    x = torch.ones((M, K)).half()
    x[1::2, ::3] = 20.0
    run_case(T, orc, x, codes, scales, "same sign")


def test_negative_and_zero_scales(T, orc):
    from ternary_weight_only_b200 import synth
    x, codes, scales = synth.case(2, 768, 90, seed=43)
    scales = scales.clone()
    scales[::3] = -scales[::3]
    scales[1::5] = 0
    run_case(T, orc, x, codes, scales, "signed scales")


def test_invalid_slot_value_is_finite(T):
    slots = torch.full((32, 64), 0xFF, dtype=torch.uint8, device="cuda")  # every code 3
    scales = torch.full((32, 2), 0.01).half().cuda()
    x = torch.randn(1, 256).half().cuda()
    y = T.tern_gemm(x, slots, scales)
    torch.cuda.synchronize()
    assert torch.isfinite(y.float()).all()


def test_grouped_layer(T, orc):
    """All seven projections of one decode layer in one launch."""
    from ternary_weight_only_b200 import synth
    for M in (1, 4):
        mats, refs = [], []
        for i in range(7):
            x, codes, scales = synth.decode_proj(i, M=M)
            xn, cn, sn = np_inputs(x, codes, scales)
            slots, sc, _, _ = orc.pack(cn, sn)
            N = codes.shape[0]
            y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
            mats.append((x.cuda(), torch.from_numpy(slots).cuda(), scales.cuda(), y))
            refs.append((xn, slots, sc))
        T.tern_gemv_grouped(mats, M)
        torch.cuda.synchronize()
        for i, ((xn, slots, sc), m) in enumerate(zip(refs, mats)):
            y_ref, bound = orc.matmul(xn, slots, sc, threads=NCPU)
            check_close(m[3], y_ref, bound, f"grouped {synth.LAYER_PROJ[i][0]} M={M}")


def test_head_full(T, orc):
    """The 5120 -> 151936 output head at full size, every output checked."""
    from ternary_weight_only_b200 import synth
    N, K = 151936, 5120
    g = synth.gen(4999, "cuda")
    codes = synth.codes_sparse(N, K, g, device="cuda")
    scales = synth.scales_uniform(N, K, g, device="cuda")
    x = synth.activations(1, K, g, device="cuda")
    slots, sc = T.tern_pack_g128(codes, scales)
    y = T.tern_gemm(x, slots, sc)
    torch.cuda.synchronize()
    xn, cn, sn = np_inputs(x.cpu(), codes.cpu(), scales.cpu())
    ref_slots, ref_sc, _, _ = orc.pack(cn, sn)
    assert np.array_equal(ref_slots, slots.cpu().numpy())
    y_ref, bound = orc.matmul(xn, ref_slots, ref_sc, threads=NCPU)
    check_close(y, y_ref, bound, "head")


def test_stream_argument(T, orc):
    from ternary_weight_only_b200 import synth
    x, codes, scales = synth.case(1, 512, 256, seed=8)
    xn, cn, sn = np_inputs(x, codes, scales)
    slots, sc, _, _ = orc.pack(cn, sn)
    s = torch.cuda.Stream()
    xd, sd, scd = x.cuda(), torch.from_numpy(slots).cuda(), scales.cuda()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        y = T.tern_gemm(xd, sd, scd)
    s.synchronize()
    y_ref, bound = orc.matmul(xn, slots, sc)
    check_close(y, y_ref, bound, "side stream")


@pytest.fixture(params=[(4, 0), (6, 0)], ids=["pc", "pc_token_columns"])
def pc(T, request):
    """Select the producer/consumer mma.sync kernel for K a multiple of 1024,
    with the scale groups (4) or the token rows (6) in the mma columns at M = 1."""
    variant, ctas = request.param
    T.tern_set_option(T.TERN_OPT_GEMV_VARIANT, variant)
    T.tern_set_option(T.TERN_OPT_GEMV_CTAS, ctas)
    yield T
    T.tern_set_option(T.TERN_OPT_GEMV_VARIANT, 0)
    T.tern_set_option(T.TERN_OPT_GEMV_CTAS, 0)


@pytest.mark.parametrize("M", [1, 2, 4, 8])
@pytest.mark.parametrize("i", range(7))
def test_producer_consumer_layer(pc, orc, i, M):
    from ternary_weight_only_b200 import synth
    x, codes, scales = synth.decode_proj(i, M=M)
    run_case(pc, orc, x, codes, scales, f"pc {synth.LAYER_PROJ[i][0]} M={M}")


@pytest.mark.parametrize("grid", [0, 1, 5, 37])
@pytest.mark.parametrize("M,K,N", [(1, 1024, 17), (1, 17408, 1000), (2, 5120, 4000), (3, 2048, 250),
                                   (1, 20480, 33), (8, 2048, 129), (1, 12288, 5000), (4, 3072, 7)])
def test_producer_consumer_grids(pc, orc, grid, M, K, N):
    """Capped grids give each CTA many tiles, whose (tile, slice) units its
    twelve warps split evenly: tiles shared by neighbouring warps are summed
    at the end of the CTA."""
    from ternary_weight_only_b200 import synth
    x, codes, scales = synth.case(M, K, N, seed=grid * 31 + M + K + N, codes="sparse", outlier_p=0.01)
    pc.tern_set_option(pc.TERN_OPT_GEMV_GRID, grid)
    try:
        run_case(pc, orc, x, codes, scales, f"pc grid={grid} M={M} K={K} N={N}")
    finally:
        pc.tern_set_option(pc.TERN_OPT_GEMV_GRID, 0)


@pytest.mark.parametrize("grid", [0, 7, 30])
def test_producer_consumer_layer_grids(pc, orc, grid):
    """A grouped decode layer (K = 5120, 6144 and 17408: 5, 6 and 17 slices
    of 1024 per row) on full and capped grids, twice in a row."""
    from ternary_weight_only_b200 import synth
    mats, refs = [], []
    for i in range(7):
        x, codes, scales = synth.decode_proj(i, M=2)
        xn, cn, sn = np_inputs(x, codes, scales)
        slots, sc, _, _ = orc.pack(cn, sn)
        y = torch.full((2, codes.shape[0]), float("nan"), dtype=torch.float16, device="cuda")
        mats.append((x.cuda(), torch.from_numpy(slots).cuda(), scales.cuda(), y))
        refs.append((xn, slots, sc))
    pc.tern_set_option(pc.TERN_OPT_GEMV_GRID, grid)
    try:
        for _ in range(2):
            pc.tern_gemv_grouped(mats, 2)
        pc.tern_sync_status()
    finally:
        pc.tern_set_option(pc.TERN_OPT_GEMV_GRID, 0)
    for i, ((xn, slots, sc), m) in enumerate(zip(refs, mats)):
        y_ref, bound = orc.matmul(xn, slots, sc, threads=NCPU)
        check_close(m[3], y_ref, bound, f"pc grid={grid} {synth.LAYER_PROJ[i][0]}")


def test_producer_consumer_exact_cases(pc, orc):
    """All-zero weights give exactly zero; one-hot x gives s * t exactly; large
    activations (|x| > 256, where the staged x is scaled down) stay in bound."""
    from ternary_weight_only_b200 import synth
    N, K = 64, 2048
    g = synth.gen(99, "cuda")
    scales = synth.scales_uniform(N, K, g, device="cuda")
    x = synth.activations(1, K, g, device="cuda")
    codes = torch.zeros((N, K), dtype=torch.int8, device="cuda")  # t = 0 everywhere
    slots, sc = pc.tern_pack_g128(codes, scales)
    y = pc.tern_gemv(x[0], slots, sc)
    pc.tern_sync_status()
    assert bool(torch.all(y == 0)), y.abs().max()
    codes = synth.codes_uniform(N, K, g, device="cuda")
    slots, sc = pc.tern_pack_g128(codes, scales)
    for k in (0, 1, 7, 8, 15, 127, 128, 1000, 2047):
        xe = torch.zeros(K, dtype=torch.float16, device="cuda")
        xe[k] = 3.0
        y = pc.tern_gemv(xe, slots, sc)
        want = (3.0 * scales[:, k // 128].float() * codes[:, k].float()).half()
        assert torch.equal(y, want), (k, (y.float() - want.float()).abs().max())
    for amp in (300.0, 20000.0):
        xb = (x.float() * amp / x.float().abs().max()).half()
        y = pc.tern_gemv(xb[0], slots, sc)
        xn, cn, sn = np_inputs(xb.cpu(), codes.cpu(), scales.cpu())
        ref_slots, ref_sc, _, _ = orc.pack(cn, sn)
        y_ref, bound = orc.matmul(xn, ref_slots, ref_sc, threads=NCPU)
        check_close(y.view(1, -1), y_ref, bound, f"pc |x| up to {amp}")
    pc.tern_sync_status()


def test_producer_consumer_grouped_and_timeout(pc, orc):
    from ternary_weight_only_b200 import synth
    mats, refs = [], []
    for i in range(7):
        x, codes, scales = synth.decode_proj(i, M=1)
        xn, cn, sn = np_inputs(x, codes, scales)
        slots, sc, _, _ = orc.pack(cn, sn)
        y = torch.full((1, codes.shape[0]), float("nan"), dtype=torch.float16, device="cuda")
        mats.append((x.cuda(), torch.from_numpy(slots).cuda(), scales.cuda(), y))
        refs.append((xn, slots, sc))
    pc.tern_gemv_grouped(mats, 1)
    pc.tern_sync_status()
    for i, ((xn, slots, sc), m) in enumerate(zip(refs, mats)):
        y_ref, bound = orc.matmul(xn, slots, sc, threads=NCPU)
        check_close(m[3], y_ref, bound, f"pc grouped {synth.LAYER_PROJ[i][0]}")
    # a wait that can never complete gives up, is reported, and the context survives
    pc.tern_set_option(pc.TERN_OPT_TEST_STALL_US, 2000)
    try:
        pc.tern_gemv_grouped(mats, 1)
        with pytest.raises(pc.TernError) as ei:
            pc.tern_sync_status()
        assert ei.value.status == pc.TERN_ERR_TIMEOUT
    finally:
        pc.tern_set_option(pc.TERN_OPT_TEST_STALL_US, 0)
    pc.tern_gemv_grouped(mats, 1)
    pc.tern_sync_status()
    xn, slots, sc = refs[4]
    y_ref, bound = orc.matmul(xn, slots, sc, threads=NCPU)
    check_close(mats[4][3], y_ref, bound, "pc after timeout")
