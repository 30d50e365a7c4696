"""fp64 CPU oracle for the ternary-g128 weight-only matmul -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or calls it, and the two share no
code.  The arithmetic lives in ``tern_oracle.c`` (plain C, fp64); this module
only compiles it with gcc and marshals numpy arrays through ctypes.

Format followed (see the header of ``tern_oracle.c`` for the passages):
w = s_g * t with t in {-1,0,+1} and one fp16 scale s_g per 128 consecutive
weights along K; y = x * W^T.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tern_oracle.c")
_LIB_DEFAULT = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_cache: dict[str, "Oracle"] = {}


def lib_path(mutant: int = 0) -> str:
    if mutant == 0:
        return _LIB_DEFAULT
    return os.path.join(_HERE, f"liboracle_mutant{mutant}.so")


def build(mutant: int = 0, force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no intrinsics).  ``mutant``
    plants one deliberate mistake (tests only)."""
    out = lib_path(mutant)
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(_SRC):
        return out
    cmd = ["gcc", "-std=c99", "-O2", "-fPIC", "-shared", "-fopenmp",
           f"-DORC_MUTANT={int(mutant)}", _SRC, "-o", out + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


def _ptr(a: np.ndarray) -> ctypes.c_void_p:
    return ctypes.c_void_p(a.ctypes.data)


class Oracle:
    """numpy-facing wrapper around one build of ``tern_oracle.c``."""

    def __init__(self, path: str):
        self.path = path
        L = ctypes.CDLL(path)
        i64, vp, dbl, i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_double, ctypes.c_int
        L.orc_half_to_double.argtypes = [ctypes.c_uint16]
        L.orc_half_to_double.restype = dbl
        L.orc_slots_bytes.argtypes = [i64, i64]
        L.orc_slots_bytes.restype = i64
        L.orc_scales_bytes.argtypes = [i64, i64]
        L.orc_scales_bytes.restype = i64
        L.orc_pack_g128.argtypes = [vp, vp, i64, i64, vp, vp, ctypes.POINTER(i64)]
        L.orc_pack_g128.restype = i64
        L.orc_unpack_g128.argtypes = [vp, i64, i64, vp]
        L.orc_unpack_g128.restype = i64
        L.orc_weight.argtypes = [vp, vp, i64, i64, i64]
        L.orc_weight.restype = dbl
        L.orc_dequant.argtypes = [vp, vp, i64, i64, vp]
        L.orc_dequant.restype = None
        L.orc_matmul.argtypes = [vp, i64, i64, vp, vp, i64, vp, vp, i32]
        L.orc_matmul.restype = i32
        L.orc_matmul_at.argtypes = [vp, i64, i64, vp, vp, i64, vp, vp, i64, vp, vp, i32]
        L.orc_matmul_at.restype = i32
        L.orc_matvec_rows.argtypes = [vp, i64, i64, vp, vp, i64, vp, vp, i32]
        L.orc_matvec_rows.restype = i32
        L.orc_embed.argtypes = [vp, vp, i64, i64, vp, i64, vp]
        L.orc_embed.restype = i64
        L.orc_b1_slots_bytes.argtypes = [i64, i64]
        L.orc_b1_slots_bytes.restype = i64
        L.orc_pack_b1.argtypes = [vp, vp, i64, i64, vp, vp, ctypes.POINTER(i64)]
        L.orc_pack_b1.restype = i64
        L.orc_unpack_b1.argtypes = [vp, i64, i64, vp]
        L.orc_unpack_b1.restype = i64
        L.orc_b1_weight.argtypes = [vp, vp, i64, i64, i64]
        L.orc_b1_weight.restype = dbl
        L.orc_b1_matmul.argtypes = [vp, i64, i64, vp, vp, i64, vp, vp, i32]
        L.orc_b1_matmul.restype = i32
        L.orc_t5_row_bytes.argtypes = [i64]
        L.orc_t5_row_bytes.restype = i64
        L.orc_pack_t5.argtypes = [vp, vp, i64, i64, vp, vp, ctypes.POINTER(i64)]
        L.orc_pack_t5.restype = i64
        L.orc_unpack_t5.argtypes = [vp, i64, i64, vp]
        L.orc_unpack_t5.restype = i64
        L.orc_t5_weight.argtypes = [vp, vp, i64, i64, i64]
        L.orc_t5_weight.restype = dbl
        L.orc_t5_matmul.argtypes = [vp, i64, i64, vp, vp, i64, vp, vp, i32]
        L.orc_t5_matmul.restype = i32
        self.L = L
        self.threads_used = 1

    # -- scalar helpers ---------------------------------------------------
    def half_to_double(self, bits: int) -> float:
        return self.L.orc_half_to_double(int(bits) & 0xFFFF)

    def slots_bytes(self, N: int, K: int) -> int:
        return self.L.orc_slots_bytes(N, K)

    def scales_bytes(self, N: int, K: int) -> int:
        return self.L.orc_scales_bytes(N, K)

    # -- format -----------------------------------------------------------
    def pack(self, codes: np.ndarray, scales_bits: np.ndarray):
        """codes int8 [N,K]; scales_bits uint16 [N,K/128] -> (slots uint8 [N,K/4],
        scales uint16 [N,K/128], invalid_count, first_bad_index)."""
        codes = np.ascontiguousarray(codes, dtype=np.int8)
        scales_bits = np.ascontiguousarray(scales_bits, dtype=np.uint16)
        N, K = codes.shape
        slots = np.zeros((N, max(K // 4, 0)), dtype=np.uint8)
        sc = np.zeros((N, max(K // 128, 0)), dtype=np.uint16)
        first = ctypes.c_int64(-1)
        bad = self.L.orc_pack_g128(_ptr(codes), _ptr(scales_bits), N, K, _ptr(slots), _ptr(sc),
                                   ctypes.byref(first))
        if bad < 0:
            raise ValueError("oracle pack: K must be a positive multiple of 128")
        return slots, sc, int(bad), int(first.value)

    def unpack(self, slots: np.ndarray, K: int):
        slots = np.ascontiguousarray(slots, dtype=np.uint8)
        N = slots.shape[0]
        codes = np.zeros((N, K), dtype=np.int8)
        bad = self.L.orc_unpack_g128(_ptr(slots), N, K, _ptr(codes))
        if bad < 0:
            raise ValueError("oracle unpack: K must be a positive multiple of 128")
        return codes, int(bad)

    def dequant(self, slots: np.ndarray, scales_bits: np.ndarray, K: int) -> np.ndarray:
        slots = np.ascontiguousarray(slots, dtype=np.uint8)
        scales_bits = np.ascontiguousarray(scales_bits, dtype=np.uint16)
        N = slots.shape[0]
        w = np.zeros((N, K), dtype=np.float64)
        self.L.orc_dequant(_ptr(slots), _ptr(scales_bits), N, K, _ptr(w))
        return w

    # -- matmul -----------------------------------------------------------
    def matmul(self, x_bits: np.ndarray, slots: np.ndarray, scales_bits: np.ndarray,
               threads: int = 1):
        """x_bits uint16 [M,K] (fp16 bit patterns) -> (y fp64 [M,N], bound fp64 [M,N])."""
        x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
        slots = np.ascontiguousarray(slots, dtype=np.uint8)
        scales_bits = np.ascontiguousarray(scales_bits, dtype=np.uint16)
        M, K = x_bits.shape
        N = slots.shape[0]
        y = np.zeros((M, N), dtype=np.float64)
        b = np.zeros((M, N), dtype=np.float64)
        self.threads_used = self.L.orc_matmul(_ptr(x_bits), M, K, _ptr(slots), _ptr(scales_bits),
                                              N, _ptr(y), _ptr(b), int(threads))
        return y, b

    def matmul_at(self, x_bits, slots, scales_bits, m_idx, n_idx, threads: int = 1):
        x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
        slots = np.ascontiguousarray(slots, dtype=np.uint8)
        scales_bits = np.ascontiguousarray(scales_bits, dtype=np.uint16)
        m_idx = np.ascontiguousarray(m_idx, dtype=np.int64)
        n_idx = np.ascontiguousarray(n_idx, dtype=np.int64)
        M, K = x_bits.shape
        N = slots.shape[0]
        if m_idx.size and (m_idx.min() < 0 or m_idx.max() >= M or n_idx.min() < 0 or n_idx.max() >= N):
            raise IndexError("oracle matmul_at: index out of range")
        y = np.zeros(m_idx.size, dtype=np.float64)
        b = np.zeros(m_idx.size, dtype=np.float64)
        self.threads_used = self.L.orc_matmul_at(_ptr(x_bits), M, K, _ptr(slots), _ptr(scales_bits),
                                                 N, _ptr(m_idx), _ptr(n_idx), m_idx.size, _ptr(y),
                                                 _ptr(b), int(threads))
        return y, b

    def matvec_rows(self, x_bits, row_slots: list, row_scales: list, threads: int = 1):
        """Rows given one by one (each uint8 [K/4] / uint16 [K/128]) -> y [M,R], bound [M,R]."""
        x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
        M, K = x_bits.shape
        R = len(row_slots)
        rs = [np.ascontiguousarray(r, dtype=np.uint8) for r in row_slots]
        rc = [np.ascontiguousarray(r, dtype=np.uint16) for r in row_scales]
        for a, c in zip(rs, rc):
            if a.size != K // 4 or c.size != K // 128:
                raise ValueError("oracle matvec_rows: row size does not match K")
        ps = (ctypes.c_void_p * R)(*[a.ctypes.data for a in rs])
        pc = (ctypes.c_void_p * R)(*[c.ctypes.data for c in rc])
        y = np.zeros((M, R), dtype=np.float64)
        b = np.zeros((M, R), dtype=np.float64)
        self.threads_used = self.L.orc_matvec_rows(_ptr(x_bits), M, K, ps, pc, R, _ptr(y), _ptr(b),
                                                   int(threads))
        return y, b


    # -- embedding lookup ------------------------------------------------
    def embed(self, slots: np.ndarray, scales_bits: np.ndarray, K: int, ids: np.ndarray):
        """Rows ids of the packed table -> (out fp64 [M,K] = s * t, count of ids
        outside [0, V), whose rows are +0)."""
        slots = np.ascontiguousarray(slots, dtype=np.uint8)
        scales_bits = np.ascontiguousarray(scales_bits, dtype=np.uint16)
        ids = np.ascontiguousarray(ids, dtype=np.int32)
        V = slots.shape[0]
        out = np.zeros((ids.size, K), dtype=np.float64)
        bad = self.L.orc_embed(_ptr(slots), _ptr(scales_bits), V, K, _ptr(ids), ids.size, _ptr(out))
        return out, int(bad)


    # -- the 1-bit variant ---------------------------------------------
    def b1_slots_bytes(self, N: int, K: int) -> int:
        return self.L.orc_b1_slots_bytes(N, K)

    def b1_pack(self, codes: np.ndarray, scales_bits: np.ndarray):
        """codes int8 [N,K] in {-1,+1}; scales uint16 [N,K/128] -> (bits uint8
        [N,K/8], scales, invalid_count, first_bad_index)."""
        codes = np.ascontiguousarray(codes, dtype=np.int8)
        scales_bits = np.ascontiguousarray(scales_bits, dtype=np.uint16)
        N, K = codes.shape
        bits = np.zeros((N, max(K // 8, 0)), dtype=np.uint8)
        sc = np.zeros((N, max(K // 128, 0)), dtype=np.uint16)
        first = ctypes.c_int64(-1)
        bad = self.L.orc_pack_b1(_ptr(codes), _ptr(scales_bits), N, K, _ptr(bits), _ptr(sc), ctypes.byref(first))
        if bad < 0:
            raise ValueError("oracle b1 pack: K must be a positive multiple of 128")
        return bits, sc, int(bad), int(first.value)

    def b1_unpack(self, bits: np.ndarray, K: int) -> np.ndarray:
        bits = np.ascontiguousarray(bits, dtype=np.uint8)
        N = bits.shape[0]
        codes = np.zeros((N, K), dtype=np.int8)
        if self.L.orc_unpack_b1(_ptr(bits), N, K, _ptr(codes)) < 0:
            raise ValueError("oracle b1 unpack: K must be a positive multiple of 128")
        return codes

    def b1_matmul(self, x_bits: np.ndarray, bits: np.ndarray, scales_bits: np.ndarray, threads: int = 1):
        x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
        bits = np.ascontiguousarray(bits, dtype=np.uint8)
        scales_bits = np.ascontiguousarray(scales_bits, dtype=np.uint16)
        M, K = x_bits.shape
        N = bits.shape[0]
        y = np.zeros((M, N), dtype=np.float64)
        b = np.zeros((M, N), dtype=np.float64)
        self.threads_used = self.L.orc_b1_matmul(_ptr(x_bits), M, K, _ptr(bits), _ptr(scales_bits), N,
                                                 _ptr(y), _ptr(b), int(threads))
        return y, b


    # -- five trits per byte -------------------------------------------
    def t5_row_bytes(self, K: int) -> int:
        return self.L.orc_t5_row_bytes(K)

    def t5_pack(self, codes: np.ndarray, scales_bits: np.ndarray):
        """codes int8 [N,K]; scales uint16 [N,K/128] -> (bytes uint8 [N,R],
        scales, invalid_count, first_bad_index), R = t5_row_bytes(K)."""
        codes = np.ascontiguousarray(codes, dtype=np.int8)
        scales_bits = np.ascontiguousarray(scales_bits, dtype=np.uint16)
        N, K = codes.shape
        out = np.zeros((N, max(self.t5_row_bytes(K), 0)), dtype=np.uint8)
        sc = np.zeros((N, max(K // 128, 0)), dtype=np.uint16)
        first = ctypes.c_int64(-1)
        bad = self.L.orc_pack_t5(_ptr(codes), _ptr(scales_bits), N, K, _ptr(out), _ptr(sc), ctypes.byref(first))
        if bad < 0:
            raise ValueError("oracle t5 pack: K must be a positive multiple of 128")
        return out, sc, int(bad), int(first.value)

    def t5_unpack(self, packed: np.ndarray, K: int) -> np.ndarray:
        packed = np.ascontiguousarray(packed, dtype=np.uint8)
        N = packed.shape[0]
        codes = np.zeros((N, K), dtype=np.int8)
        if self.L.orc_unpack_t5(_ptr(packed), N, K, _ptr(codes)) < 0:
            raise ValueError("oracle t5 unpack: K must be a positive multiple of 128")
        return codes

    def t5_matmul(self, x_bits: np.ndarray, packed: np.ndarray, scales_bits: np.ndarray, threads: int = 1):
        x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
        packed = np.ascontiguousarray(packed, dtype=np.uint8)
        scales_bits = np.ascontiguousarray(scales_bits, dtype=np.uint16)
        M, K = x_bits.shape
        N = packed.shape[0]
        y = np.zeros((M, N), dtype=np.float64)
        b = np.zeros((M, N), dtype=np.float64)
        self.threads_used = self.L.orc_t5_matmul(_ptr(x_bits), M, K, _ptr(packed), _ptr(scales_bits), N,
                                                 _ptr(y), _ptr(b), int(threads))
        return y, b


def load(mutant: int = 0) -> Oracle:
    """Build (if needed) and load the oracle library."""
    with _lock:
        key = str(mutant)
        if key not in _cache:
            _cache[key] = Oracle(build(mutant))
        return _cache[key]
