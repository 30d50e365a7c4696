"""GPU tensor-core prefill kernel (tcgen05) against the fp64 oracle.

Small and ragged shapes are compared in full; the prefill shapes (M = 2048 and
8192 token rows, K x N = 5120 x 17408 and 17408 x 5120) run at full size and
are compared on sampled token rows (every output of those rows).
Tolerance: |y - y_ref| <= 2e-3 * sum_k |x_k w_k| + 1e-5.
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


def run_case(T, orc, x, codes, scales, what="", force_tc=True):
    xn, cn, sn = np_inputs(x, codes, scales)
    slots, sc, bad, _ = orc.pack(cn, sn)
    assert bad == 0
    if force_tc:
        T.tern_set_option(T.TERN_OPT_GEMM_PATH, 2)
    try:
        yd = T.tern_gemm(x.cuda(), torch.from_numpy(slots).cuda(), scales.cuda())
        T.tern_sync_status()
    finally:
        T.tern_set_option(T.TERN_OPT_GEMM_PATH, 0)
    y_ref, bound = orc.matmul(xn, slots, sc, threads=NCPU)
    return check_close(yd, y_ref, bound, what)


@pytest.mark.parametrize("M,K,N", [
    (256, 128, 128), (256, 256, 256), (1, 128, 128), (17, 384, 200), (300, 640, 129),
    (512, 1024, 384), (64, 5120, 256), (100, 17408, 128), (1000, 2048, 1000), (33, 128, 1),
])
def test_small_and_ragged(T, orc, M, K, N):
    from ternary_weight_only_b200 import synth
    x, codes, scales = synth.case(M, K, N, seed=M + K + N, codes="uniform")
    run_case(T, orc, x, codes, scales, f"M={M} K={K} N={N}")


def test_dispatch_threshold(T, orc):
    """Default dispatch: M >= 32 runs on the tensor cores, 8 < M < 32 in chunks."""
    from ternary_weight_only_b200 import synth
    for M in (9, 31, 32, 40):
        x, codes, scales = synth.case(M, 512, 96, seed=M, codes="sparse", outlier_p=0.01)
        run_case(T, orc, x, codes, scales, f"M={M}", force_tc=False)


def test_exact_cases(T, orc):
    from ternary_weight_only_b200 import synth
    M, K, N = 256, 1024, 256
    x, codes, scales = synth.case(M, K, N, seed=5)
    T.tern_set_option(T.TERN_OPT_GEMM_PATH, 2)
    try:
        slots, _ = T.tern_pack_g128(torch.zeros_like(codes).cuda(), scales.cuda())
        y = T.tern_gemm(x.cuda(), slots, scales.cuda())
        T.tern_sync_status()
        assert torch.all(y == 0)
    finally:
        T.tern_set_option(T.TERN_OPT_GEMM_PATH, 0)
    ones = torch.ones_like(codes)
    unit = torch.ones_like(scales)
    xs = (torch.randn(M, K) * 0.05).half()
    run_case(T, orc, xs, ones, unit, "row sums")
    one = torch.zeros_like(codes)
    for n in range(N):
        one[n, (n * 53 + 7) % K] = 1 if n % 3 else -1
    run_case(T, orc, x, one, scales, "single non-zero")


def test_adversarial(T, orc):
    M, K, N = 256, 2048, 128
    codes = torch.ones((N, K), dtype=torch.int8)
    codes[::2, 256:] = -1
    scales = torch.full((N, K // 128), 0.0499).half()
    x = torch.ones((M, K)).half()
    x[::3, ::5] = 20.0
    run_case(T, orc, x, codes, scales, "same sign")


@pytest.mark.parametrize("case_idx", [0, 1])
@pytest.mark.parametrize("M", [2048, 8192])
def test_prefill_full_size_sampled_rows(T, orc, case_idx, M):
    """The prefill shapes at full size; 64 token rows (first, last, random) checked in full."""
    from ternary_weight_only_b200 import synth
    K, N = synth.PREFILL[case_idx]
    g = synth.gen(3000 + 10 * case_idx + (0 if M == 2048 else 1), "cuda")
    codes = synth.codes_uniform(N, K, g, device="cuda")
    scales = synth.scales_uniform(N, K, g, device="cuda")
    x = synth.activations(M, K, g, device="cuda")
    slots, sc = T.tern_pack_g128(codes, scales)
    y = T.tern_gemm(x, slots, sc)
    T.tern_sync_status()
    rows = np.unique(np.concatenate([[0, M - 1], np.random.default_rng(M + case_idx).choice(M, 62, replace=False)]))
    xn, cn, sn = np_inputs(x[torch.from_numpy(rows).cuda()].cpu(), codes.cpu(), scales.cpu())
    ref_slots, ref_sc, _, _ = orc.pack(cn, sn)
    y_ref, bound = orc.matmul(xn, ref_slots, ref_sc, threads=NCPU)
    check_close(y[torch.from_numpy(rows).cuda()], y_ref, bound, f"prefill {K}x{N} M={M}")


def test_timeout_path_reports_and_recovers(T, orc):
    """A wait that can never complete (the loader issues nothing) gives up after
    its limit; the status is reported on the host and the context stays usable."""
    from ternary_weight_only_b200 import synth
    x, codes, scales = synth.case(256, 1024, 512, seed=77)
    xd, cd, sd = x.cuda(), codes.cuda(), scales.cuda()
    slots, sc = T.tern_pack_g128(cd, sd)
    T.tern_sync_status()
    T.tern_set_option(T.TERN_OPT_GEMM_PATH, 2)
    T.tern_set_option(T.TERN_OPT_TEST_STALL_US, 2000)
    try:
        T.tern_gemm(xd, slots, sc)
        with pytest.raises(T.TernError) as ei:
            T.tern_sync_status()
        assert ei.value.status == T.TERN_ERR_TIMEOUT
    finally:
        T.tern_set_option(T.TERN_OPT_TEST_STALL_US, 0)
        T.tern_set_option(T.TERN_OPT_GEMM_PATH, 0)
    T.tern_sync_status()  # record cleared
    run_case(T, orc, x, codes, scales, "after timeout")
