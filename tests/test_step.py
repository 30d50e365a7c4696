"""The persistent decode-step launch (tern_gemv_step) against the fp64 oracle.

Every output of every matrix of a call is compared, element by element, with
the tolerance of helpers.check_close.  The cases cover: ragged N (partial last
tiles), mixed K, many small matrices (several pieces per CTA), capped grids
(pieces and split tiles in every CTA), a whole synthetic decode layer plus
the output head at full size, exact cases, and the timeout path.
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


@pytest.fixture(params=[0, 1], ids=["digit", "fp16"])
def form(T, request):
    """The two arithmetic forms of the 2-bit step at M <= 2: 0 = the digit
    form (8-bit integer mma, the default), 1 = the fp16 group-per-column form."""
    T.tern_set_option(T.TERN_OPT_STEP_FORM, request.param)
    yield request.param
    T.tern_set_option(T.TERN_OPT_STEP_FORM, 0)


def make_mats(orc, shapes, seed, M=1):
    """Host inputs packed by the oracle; device copies; outputs pre-filled with NaN.
    M = 1 passes x [K] and y [N]; M > 1 passes x [M, K] and y [M, N]."""
    from ternary_weight_only_b200 import synth
    mats, refs = [], []
    for j, (K, N) in enumerate(shapes):
        x, codes, scales = synth.case(M, K, N, seed=seed + 17 * j, codes="sparse", outlier_p=0.01)
        xn, cn, sn = np_inputs(x, codes, scales)
        slots, sc, bad, _ = orc.pack(cn, sn)
        assert bad == 0
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        xd = x.cuda()
        mats.append((xd[0] if M == 1 else xd, torch.from_numpy(slots).cuda(), scales.cuda(), y[0] if M == 1 else y))
        refs.append((xn, slots, sc))
    return mats, refs


def check_all(orc, mats, refs, what):
    for j, ((xn, slots, sc), m) in enumerate(zip(refs, mats)):
        y_ref, bound = orc.matmul(xn, slots, sc, threads=NCPU)
        check_close(m[3].reshape(y_ref.shape), y_ref, bound,
                    f"{what} matrix {j} (K={m[0].shape[-1]}, N={m[1].shape[0]})")


@pytest.mark.parametrize("grid", [0, 1, 3, 7, 40])
def test_mixed_shapes(T, orc, grid, form):
    shapes = [(1024, 1), (2048, 17), (5120, 100), (1024, 16), (3072, 333), (6144, 64), (1024, 250),
              (17408, 40), (4096, 129), (2048, 7)]
    mats, refs = make_mats(orc, shapes, seed=7000 + grid)
    T.tern_set_option(T.TERN_OPT_GEMV_GRID, grid)
    try:
        T.tern_gemv_step(mats)
        T.tern_sync_status()
    finally:
        T.tern_set_option(T.TERN_OPT_GEMV_GRID, 0)
    check_all(orc, mats, refs, f"step grid={grid}")


def test_many_small_matrices(T, orc):
    """More matrices than CTAs; every CTA crosses several pieces."""
    rng = np.random.default_rng(5)
    shapes = [(int(1024 * rng.integers(1, 5)), int(rng.integers(1, 90))) for _ in range(300)]
    mats, refs = make_mats(orc, shapes, seed=7100)
    T.tern_gemv_step(mats)
    T.tern_sync_status()
    check_all(orc, mats, refs, "step x300")


def test_decode_layer_and_head(T, orc, form):
    """The seven projections of a synthetic decode layer plus the 5120x151936
    head, one launch, every output."""
    from ternary_weight_only_b200 import synth
    shapes = [(K, N) for _, K, N in synth.LAYER_PROJ] + [(synth.HEAD[1], synth.HEAD[2])]
    mats, refs = make_mats(orc, shapes, seed=7200)
    T.tern_gemv_step(mats)
    T.tern_sync_status()
    check_all(orc, mats, refs, "step layer+head")


def test_matches_single_launches(T, orc):
    """Each matrix of a step call meets the tolerance and agrees with tern_gemv
    on the same inputs within it (the two differ only in summation order)."""
    shapes = [(5120, 6144), (6144, 5120), (17408, 512)]
    mats, refs = make_mats(orc, shapes, seed=7300)
    T.tern_gemv_step(mats)
    T.tern_sync_status()
    for j, (x, slots, sc, y) in enumerate(mats):
        y1 = T.tern_gemv(x, slots, sc)
        T.tern_sync_status()
        xn, sl, scn = refs[j]
        y_ref, bound = orc.matmul(xn, sl, scn, threads=NCPU)
        check_close(y.view(1, -1), y_ref, bound, f"step {j}")
        check_close(y1.view(1, -1), y_ref, bound, f"single {j}")


def test_exact_cases(T, form):
    """All-zero codes give exactly zero; one-hot x gives s * t exactly."""
    from ternary_weight_only_b200 import synth
    N, K = 80, 3072
    g = synth.gen(98, "cuda")
    scales = synth.scales_uniform(N, K, g, device="cuda")
    zero = torch.zeros((N, K), dtype=torch.int8, device="cuda")
    zslots, zsc = T.tern_pack_g128(zero, scales)
    codes = synth.codes_uniform(N, K, g, device="cuda")
    slots, sc = T.tern_pack_g128(codes, scales)
    x = synth.activations(1, K, g, device="cuda")[0]
    ks = (0, 1, 7, 8, 15, 127, 128, 1000, 3071)
    xes = []
    for k in ks:
        xe = torch.zeros(K, dtype=torch.float16, device="cuda")
        xe[k] = 3.0
        xes.append(xe)
    y0 = torch.empty(N, dtype=torch.float16, device="cuda")
    ys = [torch.empty(N, dtype=torch.float16, device="cuda") for _ in ks]
    T.tern_gemv_step([(x, zslots, zsc, y0)] + [(xe, slots, sc, y) for xe, y in zip(xes, ys)])
    T.tern_sync_status()
    assert bool(torch.all(y0 == 0)), y0.abs().max()
    for k, y in zip(ks, ys):
        want = (3.0 * scales[:, k // 128].float() * codes[:, k].float()).half()
        assert torch.equal(y, want), (k, (y.float() - want.float()).abs().max())


def test_timeout_reported_and_context_survives(T, orc):
    shapes = [(2048, 300), (1024, 64)]
    mats, refs = make_mats(orc, shapes, seed=7400)
    T.tern_set_option(T.TERN_OPT_TEST_STALL_US, 2000)
    try:
        T.tern_gemv_step(mats)
        with pytest.raises(T.TernError) as ei:
            T.tern_sync_status()
        assert ei.value.status == T.TERN_ERR_TIMEOUT
    finally:
        T.tern_set_option(T.TERN_OPT_TEST_STALL_US, 0)
    T.tern_gemv_step(mats)
    T.tern_sync_status()
    check_all(orc, mats, refs, "step after timeout")


@pytest.mark.parametrize("M", [2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("grid", [0, 5])
def test_verify_batch_mixed(T, orc, M, grid):
    """M token rows (M = 3 runs padded to 4, 5..8 padded to 8; at M > 4 the
    K = 17408 product does not fit eight rows of x and runs as K segments
    whose sums are added to y): every output of every token."""
    shapes = [(1024, 1), (2048, 17), (5120, 100), (3072, 333), (6144, 64), (17408, 40), (4096, 129)]
    mats, refs = make_mats(orc, shapes, seed=7500 + 10 * M + grid, M=M)
    T.tern_set_option(T.TERN_OPT_GEMV_GRID, grid)
    try:
        T.tern_gemv_step(mats, M)
        T.tern_sync_status()
    finally:
        T.tern_set_option(T.TERN_OPT_GEMV_GRID, 0)
    check_all(orc, mats, refs, f"step M={M} grid={grid}")


@pytest.mark.parametrize("M", [1, 2, 4, 8])
def test_verify_layer(T, orc, M, form):
    """The seven projections of a synthetic decode layer at M token rows."""
    from ternary_weight_only_b200 import synth
    shapes = [(K, N) for _, K, N in synth.LAYER_PROJ]
    mats, refs = make_mats(orc, shapes, seed=7600 + M, M=M)
    T.tern_gemv_step(mats, M)
    T.tern_sync_status()
    check_all(orc, mats, refs, f"step layer M={M}")


def test_chained_calls_see_complete_inputs(T):
    """Calls of more than 96 products run as several launches that may
    overlap; a call whose inputs are the outputs of the previous call must
    still read them complete.  Three chained calls of 200 products (three
    launches each; large matrices first, so the later launches of a call
    finish early): every output equals the same call repeated after a full
    synchronisation (the kernel is deterministic)."""
    from ternary_weight_only_b200 import synth
    g = synth.gen(7700, "cuda")
    count = 200

    def layer(N_of):
        mats = []
        for j in range(count):
            N = N_of(j)
            codes = synth.codes_sparse(N, 1024, g, device="cuda")
            slots, sc = T.tern_pack_g128(codes, synth.scales_uniform(N, 1024, g, device="cuda"))
            mats.append((slots, sc))
        return mats

    # A: x0 -> ya, B: ya -> yb, C: yb -> yc; C's first 20 products have four
    # times the rows, so its first launch runs longest
    A = layer(lambda j: 1024)
    B = layer(lambda j: 1024)
    C = layer(lambda j: 4096 if j < 20 else 1024)
    x0 = [synth.activations(1, 1024, g, device="cuda")[0] for _ in range(count)]
    ya = [torch.empty(1024, dtype=torch.float16, device="cuda") for _ in range(count)]
    yb = [torch.empty(1024, dtype=torch.float16, device="cuda") for _ in range(count)]
    yc = [torch.empty(C[j][0].shape[0], dtype=torch.float16, device="cuda") for j in range(count)]
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for _ in range(3):
            T.tern_gemv_step([(x0[j], A[j][0], A[j][1], ya[j]) for j in range(count)], stream=stream)
            T.tern_gemv_step([(ya[j], B[j][0], B[j][1], yb[j]) for j in range(count)], stream=stream)
            T.tern_gemv_step([(yb[j], C[j][0], C[j][1], yc[j]) for j in range(count)], stream=stream)
    T.tern_sync_status(stream)
    got = [t.clone() for t in ya + yb + yc]
    # the same calls one at a time, each after a full synchronisation
    for mats_fn in (
            lambda: [(x0[j], A[j][0], A[j][1], ya[j]) for j in range(count)],
            lambda: [(ya[j], B[j][0], B[j][1], yb[j]) for j in range(count)],
            lambda: [(yb[j], C[j][0], C[j][1], yc[j]) for j in range(count)]):
        torch.cuda.synchronize()
        T.tern_gemv_step(mats_fn())
        T.tern_sync_status()
    want = ya + yb + yc
    for i, (a, b) in enumerate(zip(got, want)):
        assert torch.equal(a, b), i


@pytest.mark.parametrize("M", [1, 2, 4, 8])
def test_long_rows_run_as_k_segments(T, orc, M, form):
    """Rows far longer than the staged x allows (K = 65536 at M = 1 and 4,
    K = 32768 at M = 8: four segments, the most a call takes) run as K
    segments; mixed with short products in one call; every output."""
    K = 65536 if M < 8 else 32768
    shapes = [(K, 48), (2048, 33), (K, 17)]
    mats, refs = make_mats(orc, shapes, seed=7800 + M, M=M)
    T.tern_gemv_step(mats, M)
    T.tern_sync_status()
    check_all(orc, mats, refs, f"step K segments M={M}")


@pytest.mark.parametrize("M", [2, 8])
def test_same_sign_rows_over_four_segments(T, orc, M):
    """The worst case for the K segments' fp16 roundings: every weight +1 with
    a positive scale and every x positive, so the running sum only grows and
    each segment's rounding of it can add up to 2^-11 of sum |x w|.  A row cut
    into four segments (the most a call takes: K = 65536 at M = 2, 32768 at
    M = 8) stays within the tolerance; every output."""
    K, N = (65536 if M == 2 else 32768), 40
    rng = np.random.default_rng(9100 + M)
    x = torch.from_numpy(rng.uniform(0.5, 1.0, size=(M, K)).astype(np.float16))
    codes = torch.ones((N, K), dtype=torch.int8)
    scales = torch.from_numpy(rng.uniform(0.005, 0.05, size=(N, K // 128)).astype(np.float16))
    xn, cn, sn = np_inputs(x, codes, scales)
    slots, sc, bad, _ = orc.pack(cn, sn)
    assert bad == 0
    y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    mats = [(x.cuda(), torch.from_numpy(slots).cuda(), scales.cuda(), y)]
    T.tern_gemv_step(mats, M)
    T.tern_sync_status()
    check_all(orc, mats, [(xn, slots, sc)], f"same-sign four segments M={M}")


def test_concurrent_calls_from_two_host_threads(T):
    """Two host threads call tern_gemv_step at the same time on their own
    streams (120 products each, two launches per call); every output equals
    the same call made alone."""
    import threading
    from ternary_weight_only_b200 import synth
    g = synth.gen(7900, "cuda")
    sets = []
    for t in range(2):
        mats = []
        for j in range(120):
            N = 64 + 16 * ((j + t) % 5)
            codes = synth.codes_sparse(N, 1024 * (1 + j % 3), g, device="cuda")
            slots, sc = T.tern_pack_g128(codes, synth.scales_uniform(N, codes.shape[1], g, device="cuda"))
            x = synth.activations(1, codes.shape[1], g, device="cuda")[0]
            mats.append((x, slots, sc, torch.empty(N, dtype=torch.float16, device="cuda")))
        sets.append(mats)
    torch.cuda.synchronize()
    # alone, one after the other
    want = []
    for mats in sets:
        T.tern_gemv_step(mats)
        T.tern_sync_status()
        want.append([m[3].clone() for m in mats])
        for m in mats:
            m[3].fill_(float("nan"))
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream() for _ in sets]
    errors = []

    def worker(i):
        try:
            for _ in range(20):
                T.tern_gemv_step(sets[i], stream=streams[i])
            streams[i].synchronize()
        except Exception as e:  # reported below
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for th in threads:
        th.start()
    for th in threads:
        th.join()
    assert not errors, errors
    T.tern_sync_status()
    for mats, w in zip(sets, want):
        for m, y in zip(mats, w):
            assert torch.equal(m[3], y)


def _range_cases(M, K, seed):
    """Activations that stress a fixed point per 128-k group: every group has
    its own pattern (cycled): all zeros; values 2^-e with e in [0, 12]
    (within 2^13 of the group's largest); fp16 subnormals only; values near
    +-30000; x all +1; x all 20 (same sign); ordinary N(0,1)."""
    gen = torch.Generator().manual_seed(seed)
    x = torch.empty(M, K)
    for m in range(M):
        for gi in range(K // 128):
            kind = (gi + 3 * m) % 7
            sl = slice(gi * 128, (gi + 1) * 128)
            sign = torch.where(torch.rand(128, generator=gen) < 0.5, -1.0, 1.0)
            if kind == 0:
                v = torch.zeros(128)
            elif kind == 1:
                v = sign * torch.pow(2.0, -torch.randint(0, 13, (128,), generator=gen).float())
            elif kind == 2:
                v = sign * torch.randint(1, 1024, (128,), generator=gen).float() * 2.0 ** -24
            elif kind == 3:
                v = sign * (30000.0 - torch.randint(0, 2000, (128,), generator=gen).float())
            elif kind == 4:
                v = torch.ones(128)
            elif kind == 5:
                v = torch.full((128,), 20.0)
            else:
                v = torch.randn(128, generator=gen)
            x[m, sl] = v
    return x.half()


@pytest.mark.parametrize("M", [1, 2])
def test_activation_range_cases(T, orc, M, form):
    """Per-group activation patterns (zeros, a 2^12 range, subnormals, values
    near 30000, same-sign runs) on mixed shapes; scales 1/1024 keep every sum
    finite in fp16; every output against the oracle."""
    from ternary_weight_only_b200 import synth
    shapes = [(2048, 96), (5120, 40), (1024, 17)]
    mats, refs = [], []
    for j, (K, N) in enumerate(shapes):
        x = _range_cases(M, K, seed=31 + j + 10 * M)
        g = synth.gen(8100 + j + 10 * M)
        codes = synth.codes_sparse(N, K, g)
        if j == 0:
            codes[: N // 2, :] = 1  # all +1 rows: no cancellation
        scales = torch.full((N, K // 128), 1.0 / 1024).half()
        xn, cn, sn = np_inputs(x, codes, scales)
        slots, sc, bad, _ = orc.pack(cn, sn)
        assert bad == 0
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        xd = x.cuda()
        mats.append((xd[0] if M == 1 else xd, torch.from_numpy(slots).cuda(), scales.cuda(), y[0] if M == 1 else y))
        refs.append((xn, slots, sc))
    T.tern_gemv_step(mats, M)
    T.tern_sync_status()
    check_all(orc, mats, refs, f"range cases M={M}")


@pytest.mark.parametrize("M", [1, 2, 4])
def test_slot_value_3_is_finite_and_local(T, orc, M, form):
    """Slot value 3 (not a valid code) in some rows: those rows give finite
    values and every other row is still within the tolerance."""
    from ternary_weight_only_b200 import synth
    K, N = 3072, 160
    x, codes, scales = synth.case(M, K, N, seed=8200 + M, codes="sparse", outlier_p=0.01)
    xn, cn, sn = np_inputs(x, codes, scales)
    slots, sc, bad, _ = orc.pack(cn, sn)
    assert bad == 0
    dirty = np.array([0, 5, 17, 18, 64, 159])
    bad_slots = slots.copy()
    rng = np.random.default_rng(M)
    for r in dirty:
        cols = rng.choice(K // 4, size=40, replace=False)
        bad_slots[r, cols] = 0xFF  # four code-3 fields per byte
    y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    xd = x.cuda()
    T.tern_gemv_step([(xd[0] if M == 1 else xd, torch.from_numpy(bad_slots).cuda(), scales.cuda(),
                       y[0] if M == 1 else y)], M)
    T.tern_sync_status()
    got = y.float().cpu()
    assert bool(torch.isfinite(got).all())
    clean = np.setdiff1d(np.arange(N), dirty)
    y_ref, bound = orc.matmul(xn, slots, sc, threads=NCPU)
    check_close(got[:, clean], y_ref[:, clean], bound[:, clean], f"clean rows with slot value 3 elsewhere M={M}")


@pytest.mark.parametrize("M", [3, 4])
def test_digit_form_at_three_and_four_rows(T, orc, M):
    """The digit form at three and four token rows (TERN_OPT_STEP_FORM = 2:
    two column sets of two tokens per group): mixed shapes, a decode layer,
    and a row long enough to run as K segments; every output."""
    from ternary_weight_only_b200 import synth
    shapes = [(1024, 1), (2048, 17), (5120, 100), (3072, 333), (17408, 40)]
    shapes += [(K, N) for _, K, N in synth.LAYER_PROJ] + [(32768, 24)]
    mats, refs = make_mats(orc, shapes, seed=8300 + M, M=M)
    T.tern_set_option(T.TERN_OPT_STEP_FORM, 2)
    try:
        T.tern_gemv_step(mats, M)
        T.tern_sync_status()
    finally:
        T.tern_set_option(T.TERN_OPT_STEP_FORM, 0)
    check_all(orc, mats, refs, f"digit form M={M}")
