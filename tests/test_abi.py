"""The C ABI without a GPU: the library loads, exports every entry point that
include/tern.h declares, and rejects bad arguments on the host before any
launch."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tern.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tern_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from ternary_weight_only_b200 import build
    build.build()
    from ternary_weight_only_b200 import tern
    return tern.lib


def test_header_declares_the_boundary():
    names = _declared()
    for n in ["tern_pack_g128", "tern_unpack_g128", "tern_gemv", "tern_gemm",
              "tern_gemv_grouped", "tern_gemv_step", "tern_embed_gather", "tern_workspace_bytes",
              "tern_b1_pack", "tern_b1_unpack", "tern_b1_gemv_step", "tern_t5_bytes", "tern_t5_pack",
              "tern_t5_unpack", "tern_t5_gemv_step",
              "tern_slots_bytes",
              "tern_scales_bytes", "tern_status_string", "tern_last_error", "tern_set_option",
              "tern_version"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    from ternary_weight_only_b200 import build
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True,
                         text=True, check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    for name in _declared():
        assert name in exported, name
        assert hasattr(lib, name)


def test_sizes(lib):
    assert lib.tern_slots_bytes(256, 512) == 256 * 128
    assert lib.tern_scales_bytes(256, 512) == 256 * 4 * 2
    assert lib.tern_slots_bytes(151936, 5120) + lib.tern_scales_bytes(151936, 5120) == \
        151936 * 5120 * 17 // 64
    for bad in [(0, 128), (4, 0), (4, 100), (-1, 128), (4, -128)]:
        assert lib.tern_slots_bytes(*bad) == 0 and lib.tern_scales_bytes(*bad) == 0
    assert lib.tern_version() >= 100


def test_workspace_sizes(lib):
    """With the tcgen05 bandwidth kernel selected, workspace is planned for
    M <= 4 (it splits K), none for M = 5..8 and for the prefill kernel; invalid
    shapes give 0; a grouped query for one matrix equals the single-matrix
    query.  The default kernel needs none."""
    from ternary_weight_only_b200 import tern
    assert lib.tern_workspace_bytes(1, 5120, 17408) == 0
    assert lib.tern_set_option(7, 3) == 0
    for M in (1, 2, 4):
        n = lib.tern_workspace_bytes(M, 5120, 17408)
        assert n > 0 and n % 4 == 0
    for M in (5, 8, 64, 2048):
        assert lib.tern_workspace_bytes(M, 1024, 5120) == 0
    for bad in [(0, 1024, 5120), (1, 0, 5120), (1, 1024, 100)]:
        assert lib.tern_workspace_bytes(*bad) == 0
    arr = (tern.tern_gemv_desc * 1)()
    arr[0].N, arr[0].K = 17408, 5120
    assert lib.tern_gemv_grouped_workspace_bytes(arr, 1, 1) == lib.tern_workspace_bytes(1, 17408, 5120)
    assert lib.tern_gemv_grouped_workspace_bytes(arr, 0, 1) == 0
    assert lib.tern_gemv_grouped_workspace_bytes(None, 1, 1) == 0
    assert lib.tern_set_option(7, 0) == 0


def test_status_strings(lib):
    for st in range(8):
        assert lib.tern_status_string(st)
    assert lib.tern_status_string(99) == b"unknown status"


A = 1 << 20  # a fake 16-byte-aligned address: never dereferenced, checks fail first


@pytest.mark.parametrize("args,status", [
    ((None, A, A, A, 8, 128, None, 0, None), 1),          # null x
    ((A, A, A, A, 8, 100, None, 0, None), 3),             # K % 128
    ((A, A, A, A, 0, 128, None, 0, None), 3),             # N = 0
    ((A + 2, A, A, A, 8, 128, None, 0, None), 2),         # misaligned x
    ((A, A + 4, A, A, 8, 128, None, 0, None), 2),         # misaligned slots
    ((A, A, A + 2, A, 8, 128, None, 0, None), 2),         # misaligned scales
    ((A, A, A, A + 8, 8, 128, None, 0, None), 2),         # misaligned y
])
def test_gemv_rejects(lib, args, status):
    assert lib.tern_gemv(*args) == status
    assert lib.tern_last_error()


def test_gemm_rejects(lib):
    assert lib.tern_gemm(A, A, A, A, 0, 8, 128, None, 0, None) == 3
    assert lib.tern_gemm(A, A, A, A, 4, 8, 130, None, 0, None) == 3
    assert lib.tern_gemm(A, A, A, None, 4, 8, 128, None, 0, None) == 1


def test_pack_rejects(lib):
    assert lib.tern_pack_g128(None, A, 4, 128, A, A, None, None) == 1
    assert lib.tern_pack_g128(A, A, 4, 96, A, A, None, None) == 3
    assert lib.tern_pack_g128(A + 1, A, 4, 128, A, A, None, None) == 2
    assert lib.tern_pack_g128(A, A + 1, 4, 128, A, A, None, None) == 2
    assert lib.tern_pack_g128(A, A, 4, 128, A, A, A + 2, None) == 2
    assert lib.tern_unpack_g128(A, 4, 128, A + 3, None) == 2
    assert lib.tern_unpack_g128(A, 4, 127, A, None) == 3


def test_grouped_rejects(lib):
    from ternary_weight_only_b200 import tern
    arr = (tern.tern_gemv_desc * 2)()
    for d in arr:
        d.x, d.slots, d.scales, d.y, d.N, d.K = A, A, A, A, 16, 256
    assert lib.tern_gemv_grouped(None, 1, 1, None, 0, None) == 1
    assert lib.tern_gemv_grouped(arr, 0, 1, None, 0, None) == 1
    assert lib.tern_gemv_grouped(arr, 17, 1, None, 0, None) == 1
    assert lib.tern_gemv_grouped(arr, 2, 9, None, 0, None) == 3
    arr[1].K = 200
    assert lib.tern_gemv_grouped(arr, 2, 1, None, 0, None) == 3
    arr[1].K = 256
    arr[1].y = A + 2
    assert lib.tern_gemv_grouped(arr, 2, 1, None, 0, None) == 2


@pytest.mark.parametrize("fn", ["tern_gemv_step", "tern_b1_gemv_step", "tern_t5_gemv_step"])
def test_step_rejects(lib, fn):
    """tern_gemv_step and its 1-bit twin: argument errors return before any launch."""
    from ternary_weight_only_b200 import tern
    arr = (tern.tern_gemv_desc * 3)()
    for d in arr:
        d.x, d.slots, d.scales, d.y, d.N, d.K = A, A, A, A, 16, 2048

    class _L:
        tern_gemv_step = getattr(lib, fn)
    lib = _L
    mmax = 4 if fn == "tern_b1_gemv_step" else 8
    assert lib.tern_gemv_step(None, 1, 1, None) == 1
    assert lib.tern_gemv_step(arr, 0, 1, None) == 1
    assert lib.tern_gemv_step(arr, tern.TERN_MAX_STEP + 1, 1, None) == 1
    assert lib.tern_gemv_step(arr, 3, 0, None) == 3
    assert lib.tern_gemv_step(arr, 3, mmax + 1, None) == 3
    arr[1].K = 1536                      # a multiple of 128 but not of 1024
    assert lib.tern_gemv_step(arr, 3, 1, None) == 3
    arr[1].K = 1000                      # not a multiple of 128
    assert lib.tern_gemv_step(arr, 3, 1, None) == 3
    arr[1].K = 2048
    arr[2].N = 0
    assert lib.tern_gemv_step(arr, 3, 1, None) == 3
    arr[2].N = 16
    arr[2].slots = A + 8
    assert lib.tern_gemv_step(arr, 3, 1, None) == 2
    arr[2].slots = A
    arr[0].x = None
    assert lib.tern_gemv_step(arr, 3, 1, None) == 1
    arr[0].x = A
    arr[1].K = 204800                    # x beyond four K segments that fit shared memory
    assert lib.tern_gemv_step(arr, 3, mmax, None) == 3


def test_step_takes_at_most_four_k_segments(lib):
    """At M = 8 a row of K = 40960 would need five K segments, each rounding
    the running sum to fp16 once more, and is refused before any launch;
    K = 32768 (four segments) passes the planning and, with no usable device,
    fails later with a CUDA status instead."""
    import torch
    from ternary_weight_only_b200 import tern
    arr = (tern.tern_gemv_desc * 1)()
    arr[0].x, arr[0].slots, arr[0].scales, arr[0].y, arr[0].N = A, A, A, A, 16
    arr[0].K = 40960
    assert lib.tern_gemv_step(arr, 1, 8, None) == 3
    if torch.cuda.is_available():
        return
    arr[0].K = 32768
    assert lib.tern_gemv_step(arr, 1, 8, None) in (5, 7)


def test_b1_pack_rejects(lib):
    """tern_b1_pack / tern_b1_unpack: argument errors return before any launch."""
    assert lib.tern_b1_pack(None, A, 4, 256, A, A, None, None) == 1
    assert lib.tern_b1_pack(A, A, 4, 200, A, A, None, None) == 3
    assert lib.tern_b1_pack(A, A, 0, 256, A, A, None, None) == 3
    assert lib.tern_b1_pack(A + 8, A, 4, 256, A, A, None, None) == 2
    assert lib.tern_b1_pack(A, A, 4, 256, A + 8, A, None, None) == 2
    assert lib.tern_b1_pack(A, A + 1, 4, 256, A, A, None, None) == 2
    assert lib.tern_b1_pack(A, A, 4, 256, A, A, A + 2, None) == 2
    assert lib.tern_b1_unpack(None, 4, 256, A, None) == 1
    assert lib.tern_b1_unpack(A, 4, 100, A, None) == 3
    assert lib.tern_b1_unpack(A + 4, 4, 256, A, None) == 2


def test_t5_sizes_and_rejects(lib):
    """tern_t5_bytes: 26 bytes per 128-weight group, rows padded to 16 bytes;
    tern_t5_pack / tern_t5_unpack argument errors return before any launch."""
    assert lib.tern_t5_bytes(3, 128) == 3 * 32
    assert lib.tern_t5_bytes(2, 5120) == 2 * 1040
    assert lib.tern_t5_bytes(151936, 5120) + lib.tern_scales_bytes(151936, 5120) == 151936 * 5120 * 7 // 32
    for bad in [(0, 128), (4, 0), (4, 100), (-1, 128)]:
        assert lib.tern_t5_bytes(*bad) == 0
    assert lib.tern_t5_pack(None, A, 4, 256, A, A, None, None) == 1
    assert lib.tern_t5_pack(A, A, 4, 200, A, A, None, None) == 3
    assert lib.tern_t5_pack(A + 8, A, 4, 256, A, A, None, None) == 2
    assert lib.tern_t5_pack(A, A, 4, 256, A + 8, A, None, None) == 2
    assert lib.tern_t5_pack(A, A + 1, 4, 256, A, A, None, None) == 2
    assert lib.tern_t5_pack(A, A, 4, 256, A, A, A + 2, None) == 2
    assert lib.tern_t5_unpack(None, 4, 256, A, None) == 1
    assert lib.tern_t5_unpack(A, 4, 100, A, None) == 3
    assert lib.tern_t5_unpack(A + 4, 4, 256, A, None) == 2


def test_embed_rejects(lib):
    """tern_embed_gather: argument errors return before any launch."""
    assert lib.tern_embed_gather(None, 4, A, A, 100, 256, A, None, None) == 1
    assert lib.tern_embed_gather(A, 4, A, A, 100, 200, A, None, None) == 3
    assert lib.tern_embed_gather(A, 4, A, A, 0, 256, A, None, None) == 3
    assert lib.tern_embed_gather(A, -1, A, A, 100, 256, A, None, None) == 3
    assert lib.tern_embed_gather(A + 2, 4, A, A, 100, 256, A, None, None) == 2
    assert lib.tern_embed_gather(A, 4, A + 8, A, 100, 256, A, None, None) == 2
    assert lib.tern_embed_gather(A, 4, A, A + 1, 100, 256, A, None, None) == 2
    assert lib.tern_embed_gather(A, 4, A, A, 100, 256, A + 8, None, None) == 2
    assert lib.tern_embed_gather(A, 4, A, A, 100, 256, A, A + 2, None) == 2
    assert lib.tern_embed_gather(A, 0, A, A, 100, 256, A, None, None) == 0


def test_options(lib):
    assert lib.tern_set_option(99, 1) == 1
    assert lib.tern_set_option(1, -1) == 1
    assert lib.tern_set_option(1, 0) == 0


def test_valid_call_without_gpu_reports_cuda_error(lib):
    """With no usable device a well-formed call fails cleanly with a status."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    st = lib.tern_gemv(A, A, A, A, 16, 256, None, 0, None)
    assert st in (5, 7)
    assert lib.tern_last_error()


def test_option_values(lib):
    """Kernel variants 1 and 5 were removed and are refused; the step form
    takes 0, 1 and 2 only; 0 restores every default."""
    from ternary_weight_only_b200 import tern as T
    for v in (1, 5, 7):
        assert lib.tern_set_option(T.TERN_OPT_GEMV_VARIANT, v) == T.TERN_ERR_INVALID_ARG
    for v in (0, 2, 3, 4, 6, 0):
        assert lib.tern_set_option(T.TERN_OPT_GEMV_VARIANT, v) == T.TERN_OK
    assert lib.tern_set_option(T.TERN_OPT_STEP_FORM, 3) == T.TERN_ERR_INVALID_ARG
    assert lib.tern_set_option(T.TERN_OPT_STEP_FORM, 2) == T.TERN_OK
    assert lib.tern_set_option(T.TERN_OPT_STEP_FORM, 1) == T.TERN_OK
    assert lib.tern_set_option(T.TERN_OPT_STEP_FORM, 0) == T.TERN_OK
