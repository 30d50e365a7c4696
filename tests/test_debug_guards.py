"""The debug build (libtern_debug.so: in-kernel index checks in the
decode-step kernels, failed checks counted in a device word and reported by
tern_sync_status as TERN_ERR_GUARD, no trap) on legal shapes: every form the
step kernels take -- the three weight storages, one, two and four token rows in the
digit form, the fp16 group-per-column form at 1, 2, 4 and 8 rows, products
cut into K segments, several matrices per CTA -- reports no failed check and
still matches the oracle.  This stands in for a memory checker where none
can be run.
"""
import ctypes
import os

import numpy as np
import pytest
import torch

from helpers import check_close, np_inputs

pytestmark = pytest.mark.gpu
NCPU = os.cpu_count() or 1


@pytest.fixture(scope="module")
def D():
    from ternary_weight_only_b200 import build
    path = build.build(debug=True)
    from ternary_weight_only_b200 import tern
    lib = ctypes.CDLL(path)
    lib.tern_set_option.argtypes = [ctypes.c_int, ctypes.c_int64]
    lib.tern_sync_status.argtypes = [ctypes.c_void_p]
    for fn in ("tern_gemv_step", "tern_b1_gemv_step", "tern_t5_gemv_step"):
        getattr(lib, fn).argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p]
    yield lib, tern
    lib.tern_set_option(tern.TERN_OPT_STEP_FORM, 0)


@pytest.mark.parametrize("fmt", ["tern", "b1", "t5"])
@pytest.mark.parametrize("M,form", [(1, 0), (2, 0), (3, 2), (4, 2), (1, 1), (2, 1), (4, 1), (8, 1)])
def test_no_index_check_fails(D, orc, fmt, M, form):
    lib, T = D
    if fmt == "b1" and M > 4:
        pytest.skip("the 1-bit step takes M <= 4")
    from ternary_weight_only_b200 import synth
    # the last row is long enough to run as K segments (five-per-byte at
    # M = 8 fits K = 24576 in four segments of its shorter x room, the most
    # a call takes)
    shapes = [(1024, 40), (3072, 333), (17408, 48), (2048, 17), (65536 if M <= 2 else 24576, 20)]
    kind = "sign" if fmt == "b1" else "sparse"
    pack = {"tern": T.tern_pack_g128, "b1": T.tern_b1_pack, "t5": T.tern_t5_pack}[fmt]
    orc_pack = {"tern": orc.pack, "b1": orc.b1_pack, "t5": orc.t5_pack}[fmt]
    orc_mm = {"tern": orc.matmul, "b1": orc.b1_matmul, "t5": orc.t5_matmul}[fmt]
    mats, refs = [], []
    for j, (K, N) in enumerate(shapes):
        x, codes, scales = synth.case(M, K, N, seed=8600 + 7 * j + M, codes=kind, outlier_p=0.01)
        w_d, sc_d = pack(codes.cuda(), scales.cuda())
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        xd = x.cuda()
        mats.append((xd[0] if M == 1 else xd, w_d, sc_d, y[0] if M == 1 else y))
        refs.append((x, codes, scales))
    lib.tern_set_option(T.TERN_OPT_STEP_FORM, form)
    stream = torch.cuda.current_stream().cuda_stream
    fn = {"tern": lib.tern_gemv_step, "b1": lib.tern_b1_gemv_step, "t5": lib.tern_t5_gemv_step}[fmt]
    st = fn(T._step_descs(mats), len(mats), M, stream)
    assert st == T.TERN_OK, st
    st = lib.tern_sync_status(stream)
    assert st == T.TERN_OK, f"status {st}: an in-kernel index check failed"
    lib.tern_set_option(T.TERN_OPT_STEP_FORM, 0)
    for (x, codes, scales), m in zip(refs, mats):
        xn, cn, sn = np_inputs(x, codes, scales)
        w, sc, bad, _ = orc_pack(cn, sn)
        assert bad == 0
        y_ref, bound = orc_mm(xn, w, sc, threads=NCPU)
        check_close(m[3].reshape(y_ref.shape), y_ref, bound, f"debug build {fmt} M={M} form={form}")
