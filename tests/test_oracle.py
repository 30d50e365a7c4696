"""Pins for the fp64 CPU oracle, each against something other than the oracle.

The oracle follows the format w = s_g * t_i, t in {-1,0,+1}, one fp16 scale per
128 weights along K ("Bonsai 27B ternary / 1-bit quantization", ThakiCloud
blog, section "How compression works"), stored in 2-bit slots ("Ternary
quantization: 27B in 7 GB", devnsb blog, section "Limits") with the byte layout
of include/tern.h.  Each pin below checks it against a hand-worked fixture
(tests/golden/), a closed form printed on the pages, a library routine (numpy),
an exact algebraic identity, or brute force.  ``test_planted_mistakes_are_caught``
rebuilds the oracle with one deliberate mistake at a time and checks that some
pin fails for each.
"""
import itertools
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f16bits(a):
    return np.asarray(a, dtype=np.float16).view(np.uint16)


def _rng(seed):
    return np.random.default_rng(seed)


def _rand_case(rng, M, K, N, lo=0.005, hi=0.05):
    codes = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    scales = _f16bits(rng.uniform(lo, hi, size=(N, K // 128)))
    x = _f16bits(rng.standard_normal((M, K)))
    return x, codes, scales


def _np_dequant(codes, scales_bits):
    """W[n,k] = s[n, k//128] * t[n,k], built directly with numpy."""
    s = scales_bits.view(np.float16).astype(np.float64)
    return np.repeat(s, 128, axis=1) * codes.astype(np.float64)


# ---------------------------------------------------------------- pins ----

def pin_half_decode(o):
    """Every binary16 bit pattern decodes like numpy's float16."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([o.half_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def pin_golden_bytes(o):
    rows = []
    with open(os.path.join(GOLDEN, "pack_bytes.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            *ts, hb = line.split()
            rows.append(([int(t) for t in ts], int(hb, 16)))
    for ts, want in rows:
        codes = np.zeros((1, 128), dtype=np.int8)
        codes[0, :4] = ts
        slots, _, bad, _ = o.pack(codes, np.zeros((1, 1), dtype=np.uint16))
        assert bad == 0
        assert slots[0, 0] == want, (ts, hex(slots[0, 0]), hex(want))
        assert np.all(slots[0, 1:] == 0x55)
        back, bad = o.unpack(slots, 128)
        assert bad == 0 and np.array_equal(back, codes)


def _load_matmul_golden():
    y, b, rows, sc = {}, {}, {}, {}
    with open(os.path.join(GOLDEN, "matmul_k128.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            p = line.split()
            if p[0] == "y":
                y[(int(p[1]), int(p[2]))] = float(p[3])
            elif p[0] == "bound":
                b[(int(p[1]), int(p[2]))] = float(p[3])
            elif p[0] == "slots_row":
                r = np.full(32, int(p[3], 16), dtype=np.uint8)
                if len(p) > 4:
                    for kv in p[5:]:
                        i, v = kv.split("=")
                        r[int(i)] = int(v, 16)
                rows[int(p[1])] = r
            elif p[0] == "scale":
                sc[int(p[1])] = int(p[2], 16)
    return y, b, rows, sc


def _golden_inputs():
    x = np.ones((2, 128))
    x[1, 64:] = -0.5
    codes = np.zeros((3, 128), dtype=np.int8)
    codes[0, :] = 1
    codes[1, 0::2] = 1
    codes[1, 1::2] = -1
    codes[2, 5] = -1
    codes[2, 100] = 1
    scales = _f16bits([[0.5], [2.0], [0.25]])
    return _f16bits(x), codes, scales


def pin_golden_matmul(o):
    gy, gb, grows, gsc = _load_matmul_golden()
    x, codes, scales = _golden_inputs()
    slots, sc, bad, _ = o.pack(codes, scales)
    assert bad == 0
    for r in range(3):
        assert np.array_equal(slots[r], grows[r]), r
        assert sc[r, 0] == gsc[r]
    y, b = o.matmul(x, slots, sc)
    for (m, n), v in gy.items():
        assert y[m, n] == v, (m, n, y[m, n], v)
    for (m, n), v in gb.items():
        assert b[m, n] == v, (m, n, b[m, n], v)


def pin_exhaustive_bytes(o):
    """All 3^4 = 81 valid 4-tuples map to 81 distinct bytes and back; every
    other byte value holds at least one code 3 and unpacks as invalid."""
    seen = {}
    for ts in itertools.product((-1, 0, 1), repeat=4):
        codes = np.zeros((1, 128), dtype=np.int8)
        codes[0, :4] = ts
        slots, _, bad, _ = o.pack(codes, np.zeros((1, 1), dtype=np.uint16))
        assert bad == 0
        byte = int(slots[0, 0])
        assert byte not in seen
        seen[byte] = ts
        back, bad = o.unpack(slots, 128)
        assert bad == 0 and tuple(back[0, :4]) == ts
    assert len(seen) == 81
    for byte in range(256):
        fields = [(byte >> (2 * j)) & 3 for j in range(4)]
        slots = np.full((1, 32), 0x55, dtype=np.uint8)
        slots[0, 0] = byte
        back, bad = o.unpack(slots, 128)
        if byte in seen:
            assert 3 not in fields and bad == 0
        else:
            assert 3 in fields and bad == fields.count(3)
            assert all(back[0, j] == 2 for j in range(4) if fields[j] == 3)


def pin_roundtrip_random(o):
    rng = _rng(7)
    for N, K in [(1, 128), (3, 256), (17, 512), (64, 1024)]:
        codes = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
        scales = rng.integers(0, 65536, size=(N, K // 128)).astype(np.uint16)
        slots, sc, bad, first = o.pack(codes, scales)
        assert bad == 0 and first == -1
        assert slots.shape == (N, K // 4)
        assert np.array_equal(sc, scales)
        back, bad = o.unpack(slots, K)
        assert bad == 0 and np.array_equal(back, codes)


def pin_invalid_codes(o):
    codes = np.zeros((2, 128), dtype=np.int8)
    codes[0, 9] = 2
    codes[1, 0] = -2
    codes[1, 127] = 127
    slots, _, bad, first = o.pack(codes, np.zeros((2, 1), dtype=np.uint16))
    assert bad == 3 and first == 9
    assert (slots[0, 2] >> 2) & 3 == 3
    assert slots[1, 0] & 3 == 3
    assert (slots[1, 31] >> 6) & 3 == 3
    back, nb = o.unpack(slots, 128)
    assert nb == 3 and back[0, 9] == 2 and back[1, 0] == 2 and back[1, 127] == 2


def pin_byte_count(o):
    """Slot bytes + scale bytes = K*N/4 + 2*K*N/128, i.e. 2.125 bits/weight, and
    the pages' size arithmetic: log2(3) + 16/128 ~= 1.71 bits/weight ideal,
    ~9.4x smaller than fp16; binary 1 + 16/128 = 1.125, ~14.2x ("Bonsai 27B
    ternary / 1-bit quantization", ThakiCloud blog, section "How compression
    works").  The slot layout's 2.125 against the 1.71 ideal matches the
    deployed ~7.17 GB against the ideal ~5.9 GB ("Ternary quantization: 27B in
    7 GB", devnsb blog, section "Deploy size and hardware"): 24.8 B language +
    2.5 B embedding/head weights at 2.125 bpw, and those plus the 0.46 B vision
    tower at 1.71 bpw (parameter counts: ThakiCloud blog, section "What it is")."""
    for N, K in [(256, 512), (6144, 5120), (5120, 17408), (151936, 5120), (1, 128)]:
        total = o.slots_bytes(N, K) + o.scales_bytes(N, K)
        assert total == K * N // 4 + 2 * K * N // 128
        assert total * 8 / (N * K) == 2.125
    ideal = math.log2(3) + 16 / 128
    assert round(ideal, 2) == 1.71
    assert round(16 / ideal, 1) == 9.4
    assert 1 + 16 / 128 == 1.125 and round(16 / 1.125, 1) == 14.2
    assert abs((24.8e9 + 0.46e9 + 2.5e9) * ideal / 8 / 1e9 - 5.9) < 0.05
    assert abs((24.8e9 + 2.5e9) * 2.125 / 8 / 1e9 - 7.17) / 7.17 < 0.02
    # workload totals: tiny GEMV, one decode layer, one 64-layer decode step + head
    layer = [(5120, 6144), (5120, 1024), (5120, 1024), (6144, 5120),
             (5120, 17408), (5120, 17408), (17408, 5120)]
    f = lambda K, N: o.slots_bytes(N, K) + o.scales_bytes(N, K)
    assert f(512, 256) == 34816
    assert sum(f(K, N) for K, N in layer) == 90521600
    assert 64 * sum(f(K, N) for K, N in layer) + f(5120, 151936) == 6000015360


def pin_numpy_crosscheck(o):
    """Tiny shapes: oracle == numpy float64 x @ W.T (W built by numpy from the codes)."""
    rng = _rng(11)
    for M, K, N in [(1, 128, 1), (3, 128, 7), (8, 256, 64), (5, 512, 33), (2, 384, 5)]:
        x, codes, scales = _rand_case(rng, M, K, N)
        slots, sc, _, _ = o.pack(codes, scales)
        y, b = o.matmul(x, slots, sc)
        xf = x.view(np.float16).astype(np.float64)
        W = _np_dequant(codes, scales)
        ref = xf @ W.T
        refb = np.abs(xf) @ np.abs(W).T
        assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * refb.max())
        assert np.allclose(b, refb, rtol=1e-12, atol=0)
        # the dequantised matrix itself
        assert np.array_equal(o.dequant(slots, sc, K), W)


def pin_row_sums(o):
    """All codes +1 with unit scales: y[m][n] = sum_k x[m][k] for every n."""
    rng = _rng(13)
    M, K, N = 3, 640, 5
    x = _f16bits(rng.standard_normal((M, K)))
    codes = np.ones((N, K), dtype=np.int8)
    scales = _f16bits(np.ones((N, K // 128)))
    slots, sc, _, _ = o.pack(codes, scales)
    y, b = o.matmul(x, slots, sc)
    xf = x.view(np.float16).astype(np.float64)
    for m in range(M):
        want = math.fsum(xf[m])
        wantb = math.fsum(np.abs(xf[m]))
        for n in range(N):
            assert abs(y[m, n] - want) <= 1e-13 * wantb
            assert abs(b[m, n] - wantb) <= 1e-13 * wantb


def pin_exact_cases(o):
    """Zero codes give exactly 0; one non-zero gives exactly s*t*x; negating
    every code negates y exactly; doubling every scale doubles y exactly."""
    rng = _rng(17)
    M, K, N = 4, 384, 9
    x, codes, scales = _rand_case(rng, M, K, N)
    # all zero
    z = np.zeros_like(codes)
    slots, sc, _, _ = o.pack(z, scales)
    y, b = o.matmul(x, slots, sc)
    assert np.all(y == 0) and np.all(b == 0)
    # single non-zero per row, at a different place per row
    one = np.zeros_like(codes)
    pos = [(n * 37 + 5) % K for n in range(N)]
    sgn = [1 if n % 2 else -1 for n in range(N)]
    for n in range(N):
        one[n, pos[n]] = sgn[n]
    slots, sc, _, _ = o.pack(one, scales)
    y, _ = o.matmul(x, slots, sc)
    xf = x.view(np.float16).astype(np.float64)
    sf = scales.view(np.float16).astype(np.float64)
    for m in range(M):
        for n in range(N):
            assert y[m, n] == sf[n, pos[n] // 128] * sgn[n] * xf[m, pos[n]]
    # negation and scaling
    slots, sc, _, _ = o.pack(codes, scales)
    y0, _ = o.matmul(x, slots, sc)
    slots_n, sc_n, _, _ = o.pack(-codes, scales)
    yn, _ = o.matmul(x, slots_n, sc_n)
    assert np.array_equal(yn, -y0)
    s2 = _f16bits(scales.view(np.float16).astype(np.float64) * 2)
    slots2, sc2, _, _ = o.pack(codes, s2)
    y2, _ = o.matmul(x, slots2, sc2)
    assert np.array_equal(y2, 2 * y0)


def pin_brute_force(o):
    """K = 128, N = 81 (row r starts with the r-th of the 81 valid 4-tuples),
    and, at K = N = 128, one-hot x = e_k reads W out column by column."""
    tuples = list(itertools.product((-1, 0, 1), repeat=4))
    rng = _rng(19)
    for N, K in [(81, 128), (128, 128)]:
        codes = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
        for r in range(min(N, 81)):
            codes[r, :4] = tuples[r]
        scales = _f16bits(rng.uniform(0.005, 0.05, size=(N, 1)))
        slots, sc, _, _ = o.pack(codes, scales)
        X = _f16bits(np.eye(K))
        y, _ = o.matmul(X, slots, sc)  # y[k][n] = w[n][k]
        W = _np_dequant(codes, scales)
        assert np.array_equal(y, W.T)


def pin_sampled_paths(o):
    """matmul_at and matvec_rows agree exactly with the full product."""
    rng = _rng(23)
    M, K, N = 3, 256, 40
    x, codes, scales = _rand_case(rng, M, K, N)
    slots, sc, _, _ = o.pack(codes, scales)
    y, b = o.matmul(x, slots, sc)
    mi = rng.integers(0, M, 50)
    ni = rng.integers(0, N, 50)
    ya, ba = o.matmul_at(x, slots, sc, mi, ni)
    assert np.array_equal(ya, y[mi, ni]) and np.array_equal(ba, b[mi, ni])
    rows = [5, 0, 39, 17]
    yr, br = o.matvec_rows(x, [slots[r] for r in rows], [sc[r] for r in rows])
    assert np.array_equal(yr, y[:, rows]) and np.array_equal(br, b[:, rows])


def pin_embed(o):
    """Embedding rows equal codes[id] * s[id, k // 128] built with numpy from
    the unpacked codes (values and the sign of zeros); ids outside [0, V)
    give +0 rows and are counted."""
    rng = _rng(31)
    V, K = 57, 384
    codes = rng.integers(-1, 2, size=(V, K)).astype(np.int8)
    scales = _f16bits(rng.uniform(-0.05, 0.05, size=(V, K // 128)))  # negative scales too
    slots, sc, _, _ = o.pack(codes, scales)
    ids = np.array([0, V - 1, 3, 3, -1, V, 2 ** 31 - 1, 17, -5, 40], dtype=np.int32)
    out, bad = o.embed(slots, sc, K, ids)
    W = _np_dequant(codes, scales)
    ok = (ids >= 0) & (ids < V)
    assert bad == int((~ok).sum())
    want = np.zeros((ids.size, K))
    want[ok] = W[ids[ok]]
    assert np.array_equal(out, want)
    assert np.array_equal(np.signbit(out), np.signbit(want))
    assert not np.signbit(out[~ok]).any()


def pin_b1_format(o):
    """The 1-bit variant: the byte count is the closed form K*N/8 + 2*K*N/128
    = 1.125 bits/weight, 16/1.125 = 14.2x smaller than fp16 (the figures the
    ThakiCloud blog prints in "How compression works"); all 256 byte values
    unpack to their bits (LSB first, 1 -> +1, 0 -> -1) and pack back; a
    hand-worked row; random round trips; invalid inputs are counted."""
    N, K = 3, 256
    assert o.b1_slots_bytes(N, K) + o.scales_bytes(N, K) == K * N * 1.125 / 8
    assert round(16 / 1.125, 1) == 14.2
    # every byte value, 16 bytes per row of K = 128
    bytes_ = np.arange(256, dtype=np.uint8).reshape(16, 16)
    codes = o.b1_unpack(bytes_, 128)
    want = np.where((bytes_[:, :, None] >> np.arange(8)) & 1, 1, -1).reshape(16, 128)
    assert np.array_equal(codes, want)
    back, _, bad, _ = o.b1_pack(codes, np.zeros((16, 1), np.uint16))
    assert bad == 0 and np.array_equal(back, bytes_)
    # hand-worked: codes +1,-1,-1,+1,+1,+1,-1,+1 -> bits 1,0,0,1,1,1,0,1 (LSB first) = 0b10111001 = 0xB9
    row = np.full((1, 128), -1, dtype=np.int8)
    row[0, :8] = [1, -1, -1, 1, 1, 1, -1, 1]
    b, _, _, _ = o.b1_pack(row, np.zeros((1, 1), np.uint16))
    assert b[0, 0] == 0xB9 and not b[0, 1:].any()
    rng = _rng(41)
    codes = rng.choice(np.array([-1, 1], dtype=np.int8), size=(7, 384))
    b, _, bad, _ = o.b1_pack(codes, np.zeros((7, 3), np.uint16))
    assert bad == 0 and np.array_equal(o.b1_unpack(b, 384), codes)
    codes[2, 5] = 0
    codes[6, 383] = 3
    _, _, bad, first = o.b1_pack(codes, np.zeros((7, 3), np.uint16))
    assert bad == 2 and first == 2 * 384 + 5


def pin_b1_matmul(o):
    """The 1-bit product equals numpy float64 x @ (s*t).T, and all-(+1) codes
    with unit scales give row sums."""
    rng = _rng(43)
    M, K, N = 3, 384, 29
    codes = rng.choice(np.array([-1, 1], dtype=np.int8), size=(N, K))
    scales = _f16bits(rng.uniform(-0.05, 0.05, size=(N, K // 128)))
    x = _f16bits(rng.standard_normal((M, K)))
    bits, sc, _, _ = o.b1_pack(codes, scales)
    y, b = o.b1_matmul(x, bits, sc)
    W = _np_dequant(codes, scales)
    X = x.view(np.float16).astype(np.float64)
    ref = X @ W.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(b, np.abs(X) @ np.abs(W).T, rtol=1e-12, atol=1e-12)
    ones = np.ones((N, K), dtype=np.int8)
    bits, sc, _, _ = o.b1_pack(ones, _f16bits(np.ones((N, K // 128))))
    y, _ = o.b1_matmul(x, bits, sc)
    assert np.array_equal(y, np.repeat(X.sum(axis=1, keepdims=True), N, axis=1))


def pin_t5_format(o):
    """Five trits per byte: the row length closed form (26 bytes per group of
    128) and the size against the pages' arithmetic (1.625 + 16/128 = 1.75
    bits/weight, within 2.5 % of the log2(3) + 16/128 ~= 1.71 ideal of the
    ThakiCloud blog, "How compression works"; 17.6 % below 2-bit slots);
    every valid byte value decodes to its base-3 digits (numpy's base_repr),
    the invalid ones to the sentinel; a hand-worked byte; each group starts a
    new byte; round trips; invalid codes are counted."""
    assert [o.t5_row_bytes(K) for K in (128, 5120, 6144, 17408)] == [32, 1040, 1248, 3536]
    K, N = 5120, 6
    bpw = (o.t5_row_bytes(K) * N * 8 + o.scales_bytes(N, K) * 8) / (K * N)
    assert bpw == 1.75 and abs(bpw / (np.log2(3) + 16 / 128) - 1) < 0.025
    assert round(1 - 1.75 / 2.125, 3) == 0.176
    # all byte values as the first byte of a row of K = 128 (weights 0..4)
    rows = np.zeros((256, 32), dtype=np.uint8)
    rows[:, 0] = np.arange(256)
    codes = o.t5_unpack(rows, 128)
    for v in range(256):
        if v < 243:
            digits = [int(ch) for ch in np.base_repr(v, 3).zfill(5)[::-1]]
            assert list(codes[v, :5]) == [d - 1 for d in digits], v
        else:
            assert list(codes[v, :5]) == [2] * 5, v
        assert not (codes[v, 5:] + 1).any()  # zero bytes: code 0, t = -1
    # hand-worked: t = +1, 0, -1, +1, 0 -> digits 2, 1, 0, 2, 1 -> 2 + 3 + 0 + 54 + 81 = 140;
    # weights 5..9 = -1 -> byte 1 = 0; weight 127 (byte 25, digit 2) = +1 -> 2 * 9 = 18
    row = np.full((1, 128), -1, dtype=np.int8)
    row[0, :5] = [1, 0, -1, 1, 0]
    row[0, 125:128] = [-1, -1, 1]
    b, _, _, _ = o.t5_pack(row, np.zeros((1, 1), np.uint16))
    assert b.shape == (1, 32) and b[0, 0] == 140 and b[0, 25] == 18
    assert not b[0, 1:25].any() and not b[0, 26:].any()
    # the second group starts at byte 26: weight 128 = +1, weight 133 = 0 -> bytes 26, 27 = 2, 1
    row = np.full((1, 256), -1, dtype=np.int8)
    row[0, 128] = 1
    row[0, 133] = 0
    b, _, _, _ = o.t5_pack(row, np.zeros((1, 2), np.uint16))
    assert b.shape == (1, 64) and b[0, 26] == 2 and b[0, 27] == 1
    assert not b[0, :26].any() and not b[0, 28:].any()
    rng = _rng(47)
    for K in (128, 384, 1152):
        codes = rng.integers(-1, 2, size=(5, K), dtype=np.int8)
        b, _, bad, _ = o.t5_pack(codes, np.zeros((5, K // 128), np.uint16))
        assert bad == 0 and np.array_equal(o.t5_unpack(b, K), codes)
        assert int(b.max()) < 243
    codes[3, 7] = 5
    codes[4, 1000] = -2
    b, _, bad, first = o.t5_pack(codes, np.zeros((5, 9), np.uint16))
    assert bad == 2 and first == 3 * 1152 + 7 and o.t5_unpack(b, 1152)[3, 7] == 0


def pin_t5_matmul(o):
    """The five-per-byte product equals numpy float64 x @ (s*t).T."""
    rng = _rng(53)
    M, K, N = 3, 640, 21
    codes = rng.integers(-1, 2, size=(N, K), dtype=np.int8)
    scales = _f16bits(rng.uniform(-0.05, 0.05, size=(N, K // 128)))
    x = _f16bits(rng.standard_normal((M, K)))
    b, sc, _, _ = o.t5_pack(codes, scales)
    y, bound = o.t5_matmul(x, b, sc)
    W = _np_dequant(codes, scales)
    X = x.view(np.float16).astype(np.float64)
    assert np.allclose(y, X @ W.T, rtol=1e-12, atol=1e-12)
    assert np.allclose(bound, np.abs(X) @ np.abs(W).T, rtol=1e-12, atol=1e-12)


def pin_formats_agree(o):
    """The same weights give bit-identical fp64 products whatever the
    storage: ternary codes as 2-bit slots and as five trits per byte; +-1
    codes as 2-bit slots, five per byte and 1-bit signs (the three oracle
    paths share no packing code, so a slip in one shows as a difference)."""
    rng = _rng(59)
    M, K, N = 2, 384, 13
    x = _f16bits(rng.standard_normal((M, K)))
    scales = _f16bits(rng.uniform(-0.05, 0.05, size=(N, K // 128)))
    tern = rng.integers(-1, 2, size=(N, K), dtype=np.int8)
    sgn = rng.choice(np.array([-1, 1], dtype=np.int8), size=(N, K))
    s2, sc2, _, _ = o.pack(tern, scales)
    t5, sc5, _, _ = o.t5_pack(tern, scales)
    y2, b2 = o.matmul(x, s2, sc2)
    y5, b5 = o.t5_matmul(x, t5, sc5)
    assert np.array_equal(y2, y5) and np.array_equal(b2, b5)
    s2, sc2, _, _ = o.pack(sgn, scales)
    t5, sc5, _, _ = o.t5_pack(sgn, scales)
    b1, sc1, _, _ = o.b1_pack(sgn, scales)
    ya, _ = o.matmul(x, s2, sc2)
    yb, _ = o.t5_matmul(x, t5, sc5)
    yc, _ = o.b1_matmul(x, b1, sc1)
    assert np.array_equal(ya, yb) and np.array_equal(ya, yc)


PINS = [pin_half_decode, pin_golden_bytes, pin_golden_matmul, pin_exhaustive_bytes,
        pin_roundtrip_random, pin_invalid_codes, pin_byte_count, pin_numpy_crosscheck,
        pin_row_sums, pin_exact_cases, pin_brute_force, pin_sampled_paths, pin_embed, pin_b1_format,
        pin_b1_matmul, pin_t5_format, pin_t5_matmul, pin_formats_agree]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_threads_do_not_change_results(orc):
    rng = _rng(29)
    x, codes, scales = _rand_case(rng, 4, 512, 100)
    slots, sc, _, _ = orc.pack(codes, scales)
    y1, b1 = orc.matmul(x, slots, sc, threads=1)
    y4, b4 = orc.matmul(x, slots, sc, threads=4)
    assert np.array_equal(y1, y4) and np.array_equal(b1, b4)


def test_rejects_bad_k(orc):
    with pytest.raises(ValueError):
        orc.pack(np.zeros((1, 100), dtype=np.int8), np.zeros((1, 0), dtype=np.uint16))


@pytest.mark.parametrize("mutant", [1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12, 13])
def test_planted_mistakes_are_caught(mutant):
    """Each planted mistake in the oracle (bit order, code sign, group size,
    transposed operand, dropped term, subnormal decode; in the 1-bit variant
    bit order, bit meaning, scale group; in the five-per-byte packing digit
    order, base, row padding, digits running across groups) fails at least
    one pin."""
    bad = oracle.Oracle(oracle.build(mutant))
    failed = []
    for pin in PINS:
        try:
            pin(bad)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"mutant {mutant} passed every pin"
