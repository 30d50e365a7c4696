"""tern_gemv_noalloc: the M = 1 product for callers that cannot allocate device
memory (code running while a CUDA graph is captured into a pool it does not
own, runtimes that forbid allocation after start-up, plug-ins whose host
framework owns all device memory).  It takes its split-K scratch from a static
area compiled into the library instead of a caller workspace.

The test calls it through the C ABI twice in a row and checks both results
against the fp64 oracle's product (|y - y_ref| <= 2e-3 * sum_k |x_k w_k| +
1e-5, the tolerance of every parity test) and against the existing entry
point tern_gemv within the same tolerance, and that a shape needing more
scratch than the area holds is refused without launching.  It needs no state
from other tests, so it passes alone in a fresh process and after the rest of
the suite.
"""
import os

import numpy as np
import pytest
import torch

from helpers import ATOL, RTOL, check_close, f16_to_f64, np_inputs

pytestmark = pytest.mark.gpu
NCPU = os.cpu_count() or 1


@pytest.fixture(scope="module")
def T():
    from ternary_weight_only_b200 import build
    build.build()
    from ternary_weight_only_b200 import tern
    return tern


def _noalloc(T, x, slots, scales, y):
    N, K = slots.shape[0], x.shape[-1]
    st = T.lib.tern_gemv_noalloc(x.data_ptr(), slots.data_ptr(), scales.data_ptr(), y.data_ptr(), N, K,
                                 torch.cuda.current_stream().cuda_stream)
    return st


@pytest.mark.parametrize("N,K", [(5120, 17408), (17408, 5120), (151936, 5120)])
def test_noalloc_matches_gemv_on_two_calls(T, orc, N, K):
    from ternary_weight_only_b200 import synth
    g = synth.gen(7000 + N + K, "cuda")
    codes = synth.codes_sparse(N, K, g, device="cuda")
    scales = synth.scales_uniform(N, K, g, device="cuda")
    x = synth.activations(1, K, g, device="cuda")
    slots, sc = T.tern_pack_g128(codes, scales)
    y_ref_gpu = T.tern_gemv(x[0], slots, sc)            # the existing entry point
    y1 = torch.full((N,), float("nan"), dtype=torch.float16, device="cuda")
    y2 = torch.full((N,), float("nan"), dtype=torch.float16, device="cuda")
    assert _noalloc(T, x[0], slots, sc, y1) == T.TERN_OK, T.lib.tern_last_error()
    assert _noalloc(T, x[0], slots, sc, y2) == T.TERN_OK, T.lib.tern_last_error()
    T.tern_sync_status()

    xn, cn, sn = np_inputs(x.cpu(), codes.cpu(), scales.cpu())
    ref_slots, ref_sc, _, _ = orc.pack(cn, sn)
    y_ref, bound = orc.matmul(xn, ref_slots, ref_sc, threads=NCPU)
    tol = RTOL * bound[0] + ATOL
    a = f16_to_f64(y_ref_gpu)
    for call, y in enumerate((y1, y2)):
        check_close(y.view(1, N), y_ref, bound, f"no-allocation call {call + 1} against the oracle")
        b = f16_to_f64(y)
        assert np.all(np.abs(b - a) <= tol), float(np.max(np.abs(b - a) - tol))


def test_noalloc_refuses_shapes_beyond_its_area(T):
    """A shape whose scratch exceeds the static area returns TERN_ERR_WORKSPACE
    and writes nothing."""
    # Long rows over few tiles make the planner split most: K = 131072 with a
    # few hundred tiles needs ~5 MB of scratch on a 148-SM B200.
    K = 131072
    N = None
    for cand in (76800, 128000, 51200):
        T.tern_set_option(T.TERN_OPT_GEMV_VARIANT, T.GEMV_VARIANT_TC)
        need = T.tern_workspace_bytes(1, cand, K)
        T.tern_set_option(T.TERN_OPT_GEMV_VARIANT, 0)
        if need > (4 << 20):
            N = cand
            break
    assert N is not None
    slots = torch.empty((N, K // 4), dtype=torch.uint8, device="cuda")
    scales = torch.empty((N, K // 128), dtype=torch.float16, device="cuda")
    x = torch.zeros(K, dtype=torch.float16, device="cuda")
    y = torch.full((N,), 7.0, dtype=torch.float16, device="cuda")
    assert _noalloc(T, x, slots, scales, y) == T.TERN_ERR_WORKSPACE
    assert b"scratch" in T.lib.tern_last_error()
    torch.cuda.synchronize()
    assert bool(torch.all(y == 7.0))
