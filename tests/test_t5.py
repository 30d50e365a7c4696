"""Five trits per byte (base-3 digits, 26 bytes per 128-weight group) on the
GPU against the fp64 oracle: tern_t5_pack / tern_t5_unpack bit-exact, and
tern_t5_gemv_step element by element within the tolerance of
helpers.check_close.  Shapes cover ragged N, mixed K, capped grids, M = 1..4,
a synthetic decode layer plus the output head at full size, exact cases,
invalid bytes and the timeout path.
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


@pytest.mark.parametrize("N,K", [(1, 128), (33, 384), (257, 1024), (1000, 5120), (64, 17408)])
def test_pack_matches_oracle(T, orc, N, K):
    from ternary_weight_only_b200 import synth
    g = synth.gen(N * 11 + K, "cpu")
    codes = synth.codes_uniform(N, K, g)
    scales = synth.scales_uniform(N, K, g)
    _, cn, sn = np_inputs(torch.zeros(1, K, dtype=torch.float16), codes, scales)
    want, want_sc, bad, _ = orc.t5_pack(cn, sn)
    assert bad == 0
    ic = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full(want.shape, 0xAB, dtype=torch.uint8, device="cuda")  # padding must be written
    packed, sc = T.tern_t5_pack(codes.cuda(), scales.cuda(), bytes_out=out, invalid_count=ic)
    torch.cuda.synchronize()
    assert np.array_equal(packed.cpu().numpy(), want)
    assert np.array_equal(sc.cpu().view(torch.int16).numpy().view(np.uint16), want_sc)
    assert int(ic.item()) == 0
    assert torch.equal(T.tern_t5_unpack(packed, K).cpu(), codes)


def test_pack_counts_invalid_and_unpack_marks_bad_bytes(T, orc):
    N, K = 8, 256
    codes = torch.zeros((N, K), dtype=torch.int8)
    codes[1, 3] = 2
    codes[5, 200] = -5
    codes[7, 255] = 100
    scales = torch.full((N, K // 128), 0.01, dtype=torch.float16)
    _, cn, sn = np_inputs(torch.zeros(1, K, dtype=torch.float16), codes, scales)
    want, _, bad, _ = orc.t5_pack(cn, sn)
    ic = torch.zeros(1, dtype=torch.int32, device="cuda")
    packed, _ = T.tern_t5_pack(codes.cuda(), scales.cuda(), invalid_count=ic)
    torch.cuda.synchronize()
    assert int(ic.item()) == bad == 3
    assert np.array_equal(packed.cpu().numpy(), want)
    # every byte value, invalid ones included, unpacks as the oracle does
    allb = np.zeros((8, 64), dtype=np.uint8)
    allb[:, :52] = np.resize(np.arange(256, dtype=np.uint8), (8, 52))
    got = T.tern_t5_unpack(torch.from_numpy(allb).cuda(), 256).cpu().numpy()
    assert np.array_equal(got, orc.t5_unpack(allb, 256))


@pytest.fixture(params=[0, 1], ids=["digit", "fp16"])
def form(T, request):
    """The two arithmetic forms after the base-3 decode at M <= 2: 0 = the
    digit form (8-bit integer mma, the default), 1 = the fp16
    group-per-column form."""
    T.tern_set_option(T.TERN_OPT_STEP_FORM, request.param)
    yield request.param
    T.tern_set_option(T.TERN_OPT_STEP_FORM, 0)


def make_mats(orc, shapes, seed, M=1):
    from ternary_weight_only_b200 import synth
    mats, refs = [], []
    for j, (K, N) in enumerate(shapes):
        x, codes, scales = synth.case(M, K, N, seed=seed + 17 * j, codes="sparse", outlier_p=0.01)
        xn, cn, sn = np_inputs(x, codes, scales)
        packed, sc, bad, _ = orc.t5_pack(cn, sn)
        assert bad == 0
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        xd = x.cuda()
        mats.append((xd[0] if M == 1 else xd, torch.from_numpy(packed).cuda(), scales.cuda(), y[0] if M == 1 else y))
        refs.append((xn, packed, sc))
    return mats, refs


def check_all(orc, mats, refs, what):
    for j, ((xn, packed, sc), m) in enumerate(zip(refs, mats)):
        y_ref, bound = orc.t5_matmul(xn, packed, sc, threads=NCPU)
        check_close(m[3].reshape(y_ref.shape), y_ref, bound,
                    f"{what} matrix {j} (K={m[0].shape[-1]}, N={m[1].shape[0]})")


SHAPES = [(1024, 1), (2048, 17), (5120, 100), (1024, 16), (3072, 333), (6144, 64), (1024, 250),
          (17408, 40), (4096, 129), (2048, 7)]


@pytest.mark.parametrize("grid", [0, 1, 3, 40])
def test_mixed_shapes(T, orc, grid, form):
    mats, refs = make_mats(orc, SHAPES, seed=9000 + grid)
    T.tern_set_option(T.TERN_OPT_GEMV_GRID, grid)
    try:
        T.tern_t5_gemv_step(mats)
        T.tern_sync_status()
    finally:
        T.tern_set_option(T.TERN_OPT_GEMV_GRID, 0)
    check_all(orc, mats, refs, f"t5 step grid={grid}")


def test_many_small_matrices(T, orc):
    rng = np.random.default_rng(7)
    shapes = [(int(1024 * rng.integers(1, 5)), int(rng.integers(1, 90))) for _ in range(200)]
    mats, refs = make_mats(orc, shapes, seed=9100)
    T.tern_t5_gemv_step(mats)
    T.tern_sync_status()
    check_all(orc, mats, refs, "t5 step x200")


def test_decode_layer_and_head(T, orc, form):
    from ternary_weight_only_b200 import synth
    shapes = [(K, N) for _, K, N in synth.LAYER_PROJ] + [(synth.HEAD[1], synth.HEAD[2])]
    mats, refs = make_mats(orc, shapes, seed=9200)
    T.tern_t5_gemv_step(mats)
    T.tern_sync_status()
    check_all(orc, mats, refs, "t5 step layer+head")


@pytest.mark.parametrize("M", [2, 3, 4, 8])
@pytest.mark.parametrize("grid", [0, 5])
def test_verify_batch_mixed(T, orc, M, grid):
    shapes = [(1024, 1), (2048, 17), (5120, 100), (3072, 333), (6144, 64), (4096, 129), (17408, 40)]
    mats, refs = make_mats(orc, shapes, seed=9500 + 10 * M + grid, M=M)
    T.tern_set_option(T.TERN_OPT_GEMV_GRID, grid)
    try:
        T.tern_t5_gemv_step(mats, M)
        T.tern_sync_status()
    finally:
        T.tern_set_option(T.TERN_OPT_GEMV_GRID, 0)
    check_all(orc, mats, refs, f"t5 step M={M} grid={grid}")


def test_shared_memory_limit_is_a_shape_error(T):
    """A row so long that even four K segments leave x too large for the
    room beside the decode table is refused before any launch."""
    K, N = 204800, 16
    x = torch.zeros(8, K, dtype=torch.float16, device="cuda")
    packed = torch.zeros(N, 208 * K // 1024, dtype=torch.uint8, device="cuda")
    sc = torch.zeros(N, K // 128, dtype=torch.float16, device="cuda")
    y = torch.zeros(8, N, dtype=torch.float16, device="cuda")
    with pytest.raises(T.TernError) as ei:
        T.tern_t5_gemv_step([(x, packed, sc, y)], 8)
    assert ei.value.status == T.TERN_ERR_SHAPE


def test_exact_cases(T, form):
    """All-zero codes give exactly zero; one-hot x gives s * t exactly, for
    positions at every lane's window start and digit offset and in the last
    byte of a group."""
    from ternary_weight_only_b200 import synth
    N, K = 80, 3072
    g = synth.gen(97, "cuda")
    scales = synth.scales_uniform(N, K, g, device="cuda")
    zpacked, zsc = T.tern_t5_pack(torch.zeros((N, K), dtype=torch.int8, device="cuda"), scales)
    codes = synth.codes_uniform(N, K, g, device="cuda")
    packed, sc = T.tern_t5_pack(codes, scales)
    x = synth.activations(1, K, g, device="cuda")[0]
    ks = (0, 1, 4, 5, 31, 32, 33, 63, 64, 68, 95, 96, 124, 125, 127, 128, 1000, 3071)
    xes, ys = [], []
    for k in ks:
        xe = torch.zeros(K, dtype=torch.float16, device="cuda")
        xe[k] = 3.0
        xes.append(xe)
        ys.append(torch.empty(N, dtype=torch.float16, device="cuda"))
    y0 = torch.empty(N, dtype=torch.float16, device="cuda")
    T.tern_t5_gemv_step([(x, zpacked, zsc, y0)] + [(xe, packed, sc, y) for xe, y in zip(xes, ys)])
    T.tern_sync_status()
    assert bool(torch.all(y0 == 0)), y0.abs().max()
    for k, y in zip(ks, ys):
        want = (3.0 * scales[:, k // 128].float() * codes[:, k].float()).half()
        assert torch.equal(y, want), (k, (y.float() - want.float()).abs().max())


def test_timeout_reported_and_context_survives(T, orc):
    mats, refs = make_mats(orc, [(2048, 300), (1024, 64)], seed=9400)
    T.tern_set_option(T.TERN_OPT_TEST_STALL_US, 2000)
    try:
        T.tern_t5_gemv_step(mats)
        with pytest.raises(T.TernError) as ei:
            T.tern_sync_status()
        assert ei.value.status == T.TERN_ERR_TIMEOUT
    finally:
        T.tern_set_option(T.TERN_OPT_TEST_STALL_US, 0)
    T.tern_t5_gemv_step(mats)
    T.tern_sync_status()
    check_all(orc, mats, refs, "t5 step after timeout")


@pytest.mark.parametrize("M", [1, 2, 8])
def test_long_rows_run_as_k_segments(T, orc, M, form):
    """Rows longer than the staged x and the decode table allow run as K
    segments whose sums are added to y; every output."""
    K = 65536 if M == 1 else 24576
    shapes = [(K, 40), (2048, 33)]
    mats, refs = make_mats(orc, shapes, seed=9700 + M, M=M)
    T.tern_t5_gemv_step(mats, M)
    T.tern_sync_status()
    check_all(orc, mats, refs, f"t5 step K segments M={M}")


def test_invalid_bytes_give_finite_values_and_spare_other_rows(T, orc, form):
    """Bytes 243..255 are invalid: the rows holding them get some finite
    value, every other row is computed as the oracle computes it."""
    from ternary_weight_only_b200 import synth
    K, N = 2048, 64
    x, codes, scales = synth.case(1, K, N, seed=9800, codes="sparse")
    xn, cn, sn = np_inputs(x, codes, scales)
    packed, sc, _, _ = orc.t5_pack(cn, sn)
    bad_rows = [3, 17, 40]
    for r, b in zip(bad_rows, (243, 250, 255)):
        packed[r, 7] = b
        packed[r, 26 * 9 + 25] = b
    y = torch.full((N,), float("nan"), dtype=torch.float16, device="cuda")
    T.tern_t5_gemv_step([(x[0].cuda(), torch.from_numpy(packed).cuda(), scales.cuda(), y)])
    T.tern_sync_status()
    got = y.float().cpu().double().numpy()
    assert np.all(np.isfinite(got))
    good = [n for n in range(N) if n not in bad_rows]
    y_ref, bound = orc.t5_matmul(xn, packed[good], sc[good], threads=NCPU)
    check_close(y[good].view(1, -1), y_ref, bound, "t5 rows without invalid bytes")


@pytest.mark.parametrize("M", [3, 4])
def test_digit_form_at_three_and_four_rows(T, orc, M):
    """The digit form at three and four token rows (TERN_OPT_STEP_FORM = 2);
    mixed shapes and a row run as K segments; every output."""
    shapes = [(1024, 40), (5120, 100), (17408, 48), (2048, 17), (24576, 20)]
    mats, refs = make_mats(orc, shapes, seed=8400 + M, M=M)
    T.tern_set_option(T.TERN_OPT_STEP_FORM, 2)
    try:
        T.tern_t5_gemv_step(mats, M)
        T.tern_sync_status()
    finally:
        T.tern_set_option(T.TERN_OPT_STEP_FORM, 0)
    check_all(orc, mats, refs, f"t5 digit form M={M}")
