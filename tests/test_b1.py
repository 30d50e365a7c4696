"""The 1-bit variant (weights in {-1, +1}, fp16 scale per 128 weights) on the
GPU against the fp64 oracle: tern_b1_pack / tern_b1_unpack bit-exact, and
tern_b1_gemv_step element by element within the tolerance of
helpers.check_close.  Shapes cover ragged N (partial tiles), mixed K, capped
grids (split tiles in every CTA), M = 1..4, a whole synthetic decode layer
plus the output head at full size, exact cases and the timeout path.
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
    tern.tern_set_option(tern.TERN_OPT_GEMV_GRID, 0)
    tern.tern_set_option(tern.TERN_OPT_TEST_STALL_US, 0)


@pytest.mark.parametrize("N,K", [(1, 128), (33, 384), (257, 1024), (1000, 5120)])
def test_pack_matches_oracle(T, orc, N, K):
    from ternary_weight_only_b200 import synth
    g = synth.gen(N * 7 + K, "cpu")
    codes = synth.codes_sign(N, K, g)
    scales = synth.scales_uniform(N, K, g)
    _, cn, sn = np_inputs(torch.zeros(1, K, dtype=torch.float16), codes, scales)
    want_bits, want_sc, bad, _ = orc.b1_pack(cn, sn)
    assert bad == 0
    ic = torch.zeros(1, dtype=torch.int32, device="cuda")
    bits, sc = T.tern_b1_pack(codes.cuda(), scales.cuda(), invalid_count=ic)
    torch.cuda.synchronize()
    assert np.array_equal(bits.cpu().numpy(), want_bits)
    assert np.array_equal(sc.cpu().view(torch.int16).numpy().view(np.uint16), want_sc)
    assert int(ic.item()) == 0
    back = T.tern_b1_unpack(bits, K)
    assert torch.equal(back.cpu(), codes)


def test_pack_counts_invalid(T, orc):
    N, K = 8, 256
    codes = torch.ones((N, K), dtype=torch.int8)
    codes[1, 3] = 0
    codes[5, 200] = 2
    codes[7, 255] = -128
    scales = torch.full((N, K // 128), 0.01, dtype=torch.float16)
    _, cn, sn = np_inputs(torch.zeros(1, K, dtype=torch.float16), codes, scales)
    want_bits, _, bad, _ = orc.b1_pack(cn, sn)
    ic = torch.zeros(1, dtype=torch.int32, device="cuda")
    bits, _ = T.tern_b1_pack(codes.cuda(), scales.cuda(), invalid_count=ic)
    torch.cuda.synchronize()
    assert int(ic.item()) == bad == 3
    assert np.array_equal(bits.cpu().numpy(), want_bits)


@pytest.fixture(params=[0, 1], ids=["digit", "fp16"])
def form(T, request):
    """The two arithmetic forms of the 1-bit step at M <= 2: 0 = the digit
    form (8-bit integer mma, the default), 1 = the fp16 group-per-column form."""
    T.tern_set_option(T.TERN_OPT_STEP_FORM, request.param)
    yield request.param
    T.tern_set_option(T.TERN_OPT_STEP_FORM, 0)


def make_mats(orc, shapes, seed, M=1):
    """Host inputs packed by the oracle; device copies; outputs pre-filled with NaN."""
    from ternary_weight_only_b200 import synth
    mats, refs = [], []
    for j, (K, N) in enumerate(shapes):
        x, codes, scales = synth.case(M, K, N, seed=seed + 17 * j, codes="sign", outlier_p=0.01)
        xn, cn, sn = np_inputs(x, codes, scales)
        bits, sc, bad, _ = orc.b1_pack(cn, sn)
        assert bad == 0
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        xd = x.cuda()
        mats.append((xd[0] if M == 1 else xd, torch.from_numpy(bits).cuda(), scales.cuda(), y[0] if M == 1 else y))
        refs.append((xn, bits, sc))
    return mats, refs


def check_all(orc, mats, refs, what):
    for j, ((xn, bits, sc), m) in enumerate(zip(refs, mats)):
        y_ref, bound = orc.b1_matmul(xn, bits, sc, threads=NCPU)
        check_close(m[3].reshape(y_ref.shape), y_ref, bound,
                    f"{what} matrix {j} (K={m[0].shape[-1]}, N={m[1].shape[0]})")


SHAPES = [(1024, 1), (2048, 17), (5120, 100), (1024, 16), (3072, 333), (6144, 64), (1024, 250),
          (17408, 40), (4096, 129), (2048, 7)]


@pytest.mark.parametrize("grid", [0, 1, 3, 40])
def test_mixed_shapes(T, orc, grid, form):
    mats, refs = make_mats(orc, SHAPES, seed=8000 + grid)
    T.tern_set_option(T.TERN_OPT_GEMV_GRID, grid)
    try:
        T.tern_b1_gemv_step(mats)
        T.tern_sync_status()
    finally:
        T.tern_set_option(T.TERN_OPT_GEMV_GRID, 0)
    check_all(orc, mats, refs, f"b1 step grid={grid}")


def test_many_small_matrices(T, orc):
    rng = np.random.default_rng(6)
    shapes = [(int(1024 * rng.integers(1, 5)), int(rng.integers(1, 90))) for _ in range(200)]
    mats, refs = make_mats(orc, shapes, seed=8100)
    T.tern_b1_gemv_step(mats)
    T.tern_sync_status()
    check_all(orc, mats, refs, "b1 step x200")


def test_decode_layer_and_head(T, orc, form):
    """The seven projections of a synthetic decode layer plus the 5120x151936
    head as 1-bit matrices, one launch, every output."""
    from ternary_weight_only_b200 import synth
    shapes = [(K, N) for _, K, N in synth.LAYER_PROJ] + [(synth.HEAD[1], synth.HEAD[2])]
    mats, refs = make_mats(orc, shapes, seed=8200)
    T.tern_b1_gemv_step(mats)
    T.tern_sync_status()
    check_all(orc, mats, refs, "b1 step layer+head")


@pytest.mark.parametrize("M", [2, 3, 4])
@pytest.mark.parametrize("grid", [0, 5])
def test_verify_batch_mixed(T, orc, M, grid, form):
    shapes = [(1024, 1), (2048, 17), (5120, 100), (3072, 333), (6144, 64), (17408, 40), (4096, 129)]
    mats, refs = make_mats(orc, shapes, seed=8500 + 10 * M + grid, M=M)
    T.tern_set_option(T.TERN_OPT_GEMV_GRID, grid)
    try:
        T.tern_b1_gemv_step(mats, M)
        T.tern_sync_status()
    finally:
        T.tern_set_option(T.TERN_OPT_GEMV_GRID, 0)
    check_all(orc, mats, refs, f"b1 step M={M} grid={grid}")


def test_exact_cases(T, form):
    """One-hot x gives s * t exactly, for bit positions in both halves of a
    word, both byte halves and the last group; all-(+1) weights with unit
    scales and x = 1 give exactly K."""
    from ternary_weight_only_b200 import synth
    N, K = 80, 3072
    g = synth.gen(99, "cuda")
    scales = synth.scales_uniform(N, K, g, device="cuda")
    codes = synth.codes_sign(N, K, g, device="cuda")
    bits, sc = T.tern_b1_pack(codes, scales)
    ks = (0, 1, 7, 8, 15, 16, 23, 24, 31, 127, 128, 1000, 3071)
    xes, ys = [], []
    for k in ks:
        xe = torch.zeros(K, dtype=torch.float16, device="cuda")
        xe[k] = 3.0
        xes.append(xe)
        ys.append(torch.empty(N, dtype=torch.float16, device="cuda"))
    ones = torch.ones((N, K), dtype=torch.int8, device="cuda")
    obits, osc = T.tern_b1_pack(ones, torch.ones((N, K // 128), dtype=torch.float16, device="cuda"))
    x1 = torch.ones(K, dtype=torch.float16, device="cuda")
    y1 = torch.empty(N, dtype=torch.float16, device="cuda")
    T.tern_b1_gemv_step([(xe, bits, sc, y) for xe, y in zip(xes, ys)] + [(x1, obits, osc, y1)])
    T.tern_sync_status()
    for k, y in zip(ks, ys):
        want = (3.0 * scales[:, k // 128].float() * codes[:, k].float()).half()
        assert torch.equal(y, want), (k, (y.float() - want.float()).abs().max())
    assert bool(torch.all(y1 == float(K))), y1


def test_timeout_reported_and_context_survives(T, orc):
    mats, refs = make_mats(orc, [(2048, 300), (1024, 64)], seed=8400)
    T.tern_set_option(T.TERN_OPT_TEST_STALL_US, 2000)
    try:
        T.tern_b1_gemv_step(mats)
        with pytest.raises(T.TernError) as ei:
            T.tern_sync_status()
        assert ei.value.status == T.TERN_ERR_TIMEOUT
    finally:
        T.tern_set_option(T.TERN_OPT_TEST_STALL_US, 0)
    T.tern_b1_gemv_step(mats)
    T.tern_sync_status()
    check_all(orc, mats, refs, "b1 step after timeout")


@pytest.mark.parametrize("M", [1, 2, 4])
def test_long_rows_run_as_k_segments(T, orc, M, form):
    """Rows longer than the staged x allows run as K segments whose sums are
    added to y; mixed with a short product in one call; every output."""
    shapes = [(65536, 40), (2048, 33)]
    mats, refs = make_mats(orc, shapes, seed=8700 + M, M=M)
    T.tern_b1_gemv_step(mats, M)
    T.tern_sync_status()
    check_all(orc, mats, refs, f"b1 step K segments M={M}")


@pytest.mark.parametrize("M", [3, 4])
def test_digit_form_at_three_and_four_rows(T, orc, M):
    """The digit form at three and four token rows (TERN_OPT_STEP_FORM = 2);
    mixed shapes and a row run as K segments; every output."""
    shapes = [(1024, 40), (5120, 100), (17408, 48), (2048, 17), (32768, 20)]
    mats, refs = make_mats(orc, shapes, seed=8400 + M, M=M)
    T.tern_set_option(T.TERN_OPT_STEP_FORM, 2)
    try:
        T.tern_b1_gemv_step(mats, M)
        T.tern_sync_status()
    finally:
        T.tern_set_option(T.TERN_OPT_STEP_FORM, 0)
    check_all(orc, mats, refs, f"b1 digit form M={M}")
