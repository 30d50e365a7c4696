"""Python binding of libtern (include/tern.h): argument marshalling only.

Every function here has the name of the C entry point it calls and takes
PyTorch CUDA tensors; PyTorch supplies device memory and the current stream.
All arithmetic runs in the CUDA kernels of libtern.so.  If the library is
missing this module raises on import: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np
import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtern.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"libtern.so not found at {_LIB_PATH}; build it with "
        "`python -m ternary_weight_only_b200.build` (nvcc, sm_100a)")
_L = ctypes.CDLL(_LIB_PATH)

TERN_OK = 0
TERN_ERR_INVALID_ARG = 1
TERN_ERR_ALIGN = 2
TERN_ERR_SHAPE = 3
TERN_ERR_WORKSPACE = 4
TERN_ERR_CUDA = 5
TERN_ERR_TIMEOUT = 6
TERN_ERR_DEVICE = 7
TERN_ERR_GUARD = 8

TERN_OPT_GEMV_KSPLIT = 1
TERN_OPT_GEMV_CLUSTER = 2
TERN_OPT_GEMV_CTAS = 3
TERN_OPT_GEMM_PATH = 4
TERN_OPT_GEMM_MIN_M = 5
TERN_OPT_TEST_STALL_US = 6
TERN_OPT_GEMV_VARIANT = 7
TERN_OPT_GEMV_GRID = 8
TERN_OPT_GEMV_PREFETCH = 9
TERN_OPT_STEP_FORM = 10
GEMV_VARIANT_DEFAULT, GEMV_VARIANT_TMA, GEMV_VARIANT_TC, GEMV_VARIANT_PC = 0, 2, 3, 4
TERN_MAX_GROUP = 16
TERN_MAX_STEP = 512
GEMV_VARIANT_PC_TOKEN_COLUMNS = 6

_i64, _vp, _sz, _i32, _int = ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int


class tern_gemv_desc(ctypes.Structure):
    _fields_ = [("x", _vp), ("slots", _vp), ("scales", _vp), ("y", _vp), ("N", _i64), ("K", _i64)]


_SIGS = {
    "tern_version": ([], _int),
    "tern_status_string": ([_int], ctypes.c_char_p),
    "tern_last_error": ([], ctypes.c_char_p),
    "tern_slots_bytes": ([_i64, _i64], _sz),
    "tern_scales_bytes": ([_i64, _i64], _sz),
    "tern_workspace_bytes": ([_i64, _i64, _i64], _sz),
    "tern_pack_g128": ([_vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp], _int),
    "tern_unpack_g128": ([_vp, _i64, _i64, _vp, _vp], _int),
    "tern_gemv": ([_vp, _vp, _vp, _vp, _i64, _i64, _vp, _sz, _vp], _int),
    "tern_gemm": ([_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _sz, _vp], _int),
    "tern_gemv_grouped": ([ctypes.POINTER(tern_gemv_desc), _i32, _i64, _vp, _sz, _vp], _int),
    "tern_set_option": ([_int, _i64], _int),
    "tern_sync_status": ([_vp], _int),
    "tern_gemv_grouped_workspace_bytes": ([ctypes.POINTER(tern_gemv_desc), _i32, _i64], _sz),
    "tern_gemv_noalloc": ([_vp, _vp, _vp, _vp, _i64, _i64, _vp], _int),
    "tern_gemv_step": ([ctypes.POINTER(tern_gemv_desc), _i32, _i64, _vp], _int),
    "tern_embed_gather": ([_vp, _i64, _vp, _vp, _i64, _i64, _vp, _vp, _vp], _int),
    "tern_b1_pack": ([_vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp], _int),
    "tern_b1_unpack": ([_vp, _i64, _i64, _vp, _vp], _int),
    "tern_b1_gemv_step": ([ctypes.POINTER(tern_gemv_desc), _i32, _i64, _vp], _int),
    "tern_t5_bytes": ([_i64, _i64], _sz),
    "tern_t5_pack": ([_vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp], _int),
    "tern_t5_unpack": ([_vp, _i64, _i64, _vp, _vp], _int),
    "tern_t5_gemv_step": ([ctypes.POINTER(tern_gemv_desc), _i32, _i64, _vp], _int),
    "tern_step_plan": ([_vp, _vp, _i32, _i64, _i32, _vp], _int),
}
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(_L, _name)
    _f.argtypes = _args
    _f.restype = _res

lib = _L  # raw C-ABI access (pointers and sizes), used by the tests


class TernError(RuntimeError):
    def __init__(self, status: int, fn: str):
        self.status = status
        detail = _L.tern_last_error().decode(errors="replace")
        super().__init__(f"{fn}: {_L.tern_status_string(status).decode()} ({status}): {detail}")


def _check(st: int, fn: str):
    if st != TERN_OK:
        raise TernError(st, fn)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev(t: torch.Tensor, name: str, dtype=None) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def tern_version() -> int:
    return _L.tern_version()


def tern_slots_bytes(N: int, K: int) -> int:
    return _L.tern_slots_bytes(N, K)


def tern_scales_bytes(N: int, K: int) -> int:
    return _L.tern_scales_bytes(N, K)


def tern_workspace_bytes(M: int, N: int, K: int) -> int:
    return _L.tern_workspace_bytes(M, N, K)


# Zero-initialised workspaces owned by this binding, one per (device, stream):
# the library leaves a workspace zeroed after every call that completes, so a
# cached buffer can be reused by later calls on the same stream.
_WS: dict = {}
_WS_RETIRED: list = []  # outgrown buffers stay alive: a captured graph may still use them


def _workspace(nbytes: int, device: torch.device, stream: int):
    if nbytes <= 0:
        return None, 0
    key = (device.index, stream)
    buf = _WS.get(key)
    if buf is None or buf.numel() < nbytes:
        if buf is not None:
            _WS_RETIRED.append(buf)
        buf = torch.zeros(((nbytes + 255) // 256) * 256, dtype=torch.uint8, device=device)
        _WS[key] = buf
    return buf.data_ptr(), buf.numel()


def tern_reset_workspaces():
    """Zero every cached workspace (needed after a call reported TERN_ERR_TIMEOUT)."""
    for buf in list(_WS.values()) + _WS_RETIRED:
        buf.zero_()


def _ws_args(workspace, nbytes, device, stream):
    if workspace is False:
        return None, 0
    if isinstance(workspace, torch.Tensor):
        return _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    return _workspace(nbytes, device, stream)


def tern_set_option(option: int, value: int):
    _check(_L.tern_set_option(option, value), "tern_set_option")


def tern_sync_status(stream=None):
    """Wait for the stream; raise TernError if a kernel gave up a bounded wait."""
    _check(_L.tern_sync_status(_stream(stream)), "tern_sync_status")


def tern_pack_g128(codes: torch.Tensor, scales: torch.Tensor, slots_out: Optional[torch.Tensor] = None,
                   scales_out: Optional[torch.Tensor] = None,
                   invalid_count: Optional[torch.Tensor] = None, stream=None):
    """codes int8 [N,K], scales fp16 [N,K/128] -> (slots uint8 [N,K/4], scales fp16 [N,K/128])."""
    N, K = codes.shape
    if slots_out is None:
        slots_out = torch.empty((N, K // 4), dtype=torch.uint8, device=codes.device)
    if scales_out is None:
        scales_out = torch.empty_like(scales)
    ic = 0 if invalid_count is None else _dev(invalid_count, "invalid_count", torch.int32)
    _check(_L.tern_pack_g128(_dev(codes, "codes", torch.int8), _dev(scales, "scales", torch.float16),
                             N, K, _dev(slots_out, "slots_out", torch.uint8),
                             _dev(scales_out, "scales_out", torch.float16), ic or None,
                             _stream(stream)), "tern_pack_g128")
    return slots_out, scales_out


def tern_unpack_g128(slots: torch.Tensor, K: int, codes_out: Optional[torch.Tensor] = None, stream=None):
    N = slots.shape[0]
    if codes_out is None:
        codes_out = torch.empty((N, K), dtype=torch.int8, device=slots.device)
    _check(_L.tern_unpack_g128(_dev(slots, "slots", torch.uint8), N, K,
                               _dev(codes_out, "codes_out", torch.int8), _stream(stream)),
           "tern_unpack_g128")
    return codes_out


def tern_gemv(x: torch.Tensor, slots: torch.Tensor, scales: torch.Tensor,
              y: Optional[torch.Tensor] = None, stream=None, workspace=None):
    """x fp16 [K] -> y fp16 [N].  workspace: None = a cached zeroed buffer of
    tern_workspace_bytes(1, N, K) bytes, False = none, or a uint8 CUDA tensor."""
    N = slots.shape[0]
    K = x.shape[-1]
    if y is None:
        y = torch.empty((N,), dtype=torch.float16, device=x.device)
    st = _stream(stream)
    wp, wn = _ws_args(workspace, _L.tern_workspace_bytes(1, N, K) if workspace is None else 0, x.device, st)
    _check(_L.tern_gemv(_dev(x, "x", torch.float16), _dev(slots, "slots", torch.uint8),
                        _dev(scales, "scales", torch.float16), _dev(y, "y", torch.float16), N, K,
                        wp, wn, st), "tern_gemv")
    return y


def tern_gemv_noalloc(x: torch.Tensor, slots: torch.Tensor, scales: torch.Tensor,
                      y: torch.Tensor, stream=None):
    """x fp16 [K] -> y fp16 [N] (preallocated); the library uses its static
    scratch area and allocates nothing.  Calls must not overlap on the GPU."""
    N = slots.shape[0]
    K = x.shape[-1]
    _check(_L.tern_gemv_noalloc(_dev(x, "x", torch.float16), _dev(slots, "slots", torch.uint8),
                                _dev(scales, "scales", torch.float16), _dev(y, "y", torch.float16), N, K,
                                _stream(stream)), "tern_gemv_noalloc")
    return y


def tern_gemm(x: torch.Tensor, slots: torch.Tensor, scales: torch.Tensor,
              y: Optional[torch.Tensor] = None, stream=None, workspace=None):
    """x fp16 [M,K] -> y fp16 [M,N].  workspace as for tern_gemv."""
    M, K = x.shape
    N = slots.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.float16, device=x.device)
    st = _stream(stream)
    wp, wn = _ws_args(workspace, _L.tern_workspace_bytes(M, N, K) if workspace is None else 0, x.device, st)
    _check(_L.tern_gemm(_dev(x, "x", torch.float16), _dev(slots, "slots", torch.uint8),
                        _dev(scales, "scales", torch.float16), _dev(y, "y", torch.float16), M, N, K,
                        wp, wn, st), "tern_gemm")
    return y


def tern_gemv_grouped(mats: Sequence, M: int, stream=None, workspace=None):
    """mats: sequence of (x [M,K], slots [N,K/4], scales [N,K/128], y [M,N]) CUDA tensors.
    workspace as for tern_gemv (sized by tern_gemv_grouped_workspace_bytes)."""
    arr = (tern_gemv_desc * len(mats))()
    for i, (x, s, sc, y) in enumerate(mats):
        arr[i].x = _dev(x, "x", torch.float16)
        arr[i].slots = _dev(s, "slots", torch.uint8)
        arr[i].scales = _dev(sc, "scales", torch.float16)
        arr[i].y = _dev(y, "y", torch.float16)
        arr[i].N = s.shape[0]
        arr[i].K = x.shape[-1]
    st = _stream(stream)
    need = _L.tern_gemv_grouped_workspace_bytes(arr, len(mats), M) if workspace is None else 0
    wp, wn = _ws_args(workspace, need, mats[0][0].device, st)
    _check(_L.tern_gemv_grouped(arr, len(mats), M, wp, wn, st), "tern_gemv_grouped")


def tern_embed_gather(ids: torch.Tensor, slots: torch.Tensor, scales: torch.Tensor, K: int,
                      out: Optional[torch.Tensor] = None, bad_count: Optional[torch.Tensor] = None,
                      stream=None) -> torch.Tensor:
    """ids int32 [M]; slots uint8 [V,K/4]; scales fp16 [V,K/128] -> out fp16 [M,K]
    (rows s * t of the ternary table); bad_count: optional int32 [1] counter."""
    M = ids.shape[0]
    V = slots.shape[0]
    if out is None:
        out = torch.empty((M, K), dtype=torch.float16, device=slots.device)
    bc = None if bad_count is None else _dev(bad_count, "bad_count", torch.int32)
    _check(_L.tern_embed_gather(_dev(ids, "ids", torch.int32), M, _dev(slots, "slots", torch.uint8),
                                _dev(scales, "scales", torch.float16), V, K, _dev(out, "out", torch.float16),
                                bc, _stream(stream)), "tern_embed_gather")
    return out


def _step_descs(mats: Sequence):
    arr = (tern_gemv_desc * len(mats))()
    for i, (x, s, sc, y) in enumerate(mats):
        arr[i].x = _dev(x, "x", torch.float16)
        arr[i].slots = _dev(s, "slots", torch.uint8)
        arr[i].scales = _dev(sc, "scales", torch.float16)
        arr[i].y = _dev(y, "y", torch.float16)
        arr[i].N = s.shape[0]
        arr[i].K = x.shape[-1]
    return arr


def tern_step_plan(shapes: Sequence, M: int = 1, grid: int = 148):
    """shapes: sequence of (N, K) of one launch's products (host only).
    Returns the grid + 1 tile boundaries: CTA c streams the 16-row tiles
    [first[c], first[c + 1]) of the flat list."""
    n = np.ascontiguousarray([int(a) for a, _ in shapes], dtype=np.int64)
    k = np.ascontiguousarray([int(b) for _, b in shapes], dtype=np.int64)
    out = np.zeros(grid + 1, dtype=np.int32)
    _check(_L.tern_step_plan(n.ctypes.data, k.ctypes.data, len(shapes), M, grid, out.ctypes.data), "tern_step_plan")
    return out.tolist()


def tern_gemv_step(mats: Sequence, M: int = 1, stream=None):
    """mats: sequence of (x [M,K] (or [K] for M = 1), slots [N,K/4],
    scales [N,K/128], y [M,N] (or [N])) CUDA tensors, M in 1..8, every K a
    multiple of 1024: one persistent launch."""
    _check(_L.tern_gemv_step(_step_descs(mats), len(mats), M, _stream(stream)), "tern_gemv_step")


def tern_b1_pack(codes: torch.Tensor, scales: torch.Tensor, bits_out: Optional[torch.Tensor] = None,
                 scales_out: Optional[torch.Tensor] = None,
                 invalid_count: Optional[torch.Tensor] = None, stream=None):
    """1-bit variant: codes int8 [N,K] in {-1,+1}, scales fp16 [N,K/128] ->
    (bits uint8 [N,K/8], scales fp16 [N,K/128])."""
    N, K = codes.shape
    if bits_out is None:
        bits_out = torch.empty((N, K // 8), dtype=torch.uint8, device=codes.device)
    if scales_out is None:
        scales_out = torch.empty_like(scales)
    ic = None if invalid_count is None else _dev(invalid_count, "invalid_count", torch.int32)
    _check(_L.tern_b1_pack(_dev(codes, "codes", torch.int8), _dev(scales, "scales", torch.float16), N, K,
                           _dev(bits_out, "bits_out", torch.uint8), _dev(scales_out, "scales_out", torch.float16),
                           ic, _stream(stream)), "tern_b1_pack")
    return bits_out, scales_out


def tern_b1_unpack(bits: torch.Tensor, K: int, codes_out: Optional[torch.Tensor] = None, stream=None):
    N = bits.shape[0]
    if codes_out is None:
        codes_out = torch.empty((N, K), dtype=torch.int8, device=bits.device)
    _check(_L.tern_b1_unpack(_dev(bits, "bits", torch.uint8), N, K, _dev(codes_out, "codes_out", torch.int8),
                             _stream(stream)), "tern_b1_unpack")
    return codes_out


def tern_b1_gemv_step(mats: Sequence, M: int = 1, stream=None):
    """1-bit variant of tern_gemv_step: mats as there with bits uint8 [N,K/8]
    in place of the slots."""
    _check(_L.tern_b1_gemv_step(_step_descs(mats), len(mats), M, _stream(stream)), "tern_b1_gemv_step")


def tern_gemv_grouped_workspace_bytes(mats: Sequence, M: int) -> int:
    arr = (tern_gemv_desc * len(mats))()
    for i, (x, s, sc, y) in enumerate(mats):
        arr[i].N = s.shape[0]
        arr[i].K = x.shape[-1]
    return _L.tern_gemv_grouped_workspace_bytes(arr, len(mats), M)


def tern_t5_pack(codes: torch.Tensor, scales: torch.Tensor, bytes_out: Optional[torch.Tensor] = None,
                 scales_out: Optional[torch.Tensor] = None,
                 invalid_count: Optional[torch.Tensor] = None, stream=None):
    """Five trits per byte: codes int8 [N,K], scales fp16 [N,K/128] ->
    (bytes uint8 [N,R], scales fp16 [N,K/128]), R = tern_t5_bytes(N, K) / N."""
    N, K = codes.shape
    if bytes_out is None:
        R = _L.tern_t5_bytes(N, K) // max(N, 1)
        bytes_out = torch.empty((N, R), dtype=torch.uint8, device=codes.device)
    if scales_out is None:
        scales_out = torch.empty_like(scales)
    ic = None if invalid_count is None else _dev(invalid_count, "invalid_count", torch.int32)
    _check(_L.tern_t5_pack(_dev(codes, "codes", torch.int8), _dev(scales, "scales", torch.float16), N, K,
                           _dev(bytes_out, "bytes_out", torch.uint8), _dev(scales_out, "scales_out", torch.float16),
                           ic, _stream(stream)), "tern_t5_pack")
    return bytes_out, scales_out


def tern_t5_unpack(packed: torch.Tensor, K: int, codes_out: Optional[torch.Tensor] = None, stream=None):
    N = packed.shape[0]
    if codes_out is None:
        codes_out = torch.empty((N, K), dtype=torch.int8, device=packed.device)
    _check(_L.tern_t5_unpack(_dev(packed, "bytes", torch.uint8), N, K, _dev(codes_out, "codes_out", torch.int8),
                             _stream(stream)), "tern_t5_unpack")
    return codes_out


def tern_t5_gemv_step(mats: Sequence, M: int = 1, stream=None):
    """Five-per-byte variant of tern_gemv_step: mats as there with the bytes
    uint8 [N,R] in place of the slots."""
    _check(_L.tern_t5_gemv_step(_step_descs(mats), len(mats), M, _stream(stream)), "tern_t5_gemv_step")
