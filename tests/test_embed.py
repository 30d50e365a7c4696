"""Ternary embedding lookup (tern_embed_gather) against the fp64 oracle.

Outputs are s * t, exactly representable in fp16, so the comparison is exact:
every value and the sign of every zero.  Ids outside [0, V) give zero rows
and are counted.
"""
import numpy as np
import pytest
import torch

from helpers import np_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def T():
    from ternary_weight_only_b200 import build
    build.build()
    from ternary_weight_only_b200 import tern
    return tern


def table(orc, V, K, seed, neg=False):
    rng = np.random.default_rng(seed)
    codes = torch.from_numpy(rng.integers(-1, 2, size=(V, K)).astype(np.int8))
    lo = -0.05 if neg else 0.005
    scales = torch.from_numpy(rng.uniform(lo, 0.05, size=(V, K // 128))).half()
    _, cn, sn = np_inputs(torch.zeros(1, K, dtype=torch.float16), codes, scales)
    slots, sc, bad, _ = orc.pack(cn, sn)
    assert bad == 0
    return slots, sc


def check(T, orc, slots, sc, K, ids):
    ids_d = torch.from_numpy(ids).cuda()
    bad = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = T.tern_embed_gather(ids_d, torch.from_numpy(slots).cuda(), torch.from_numpy(sc.view(np.int16)).cuda().view(torch.float16),
                              K, bad_count=bad)
    T.tern_sync_status()
    want, nbad = orc.embed(slots, sc, K, ids)
    got = out.cpu().float().double().numpy()
    assert int(bad.item()) == nbad
    assert np.array_equal(got, want)
    assert np.array_equal(np.signbit(got), np.signbit(want))


@pytest.mark.parametrize("V,K", [(1, 128), (100, 640), (1000, 5120), (37, 17408), (3000, 1152)])
def test_gather(T, orc, V, K):
    rng = np.random.default_rng(V + K)
    ids = rng.integers(0, V, size=257).astype(np.int32)
    ids[:3] = [0, V - 1, 0]
    slots, sc = table(orc, V, K, seed=V * 7 + K, neg=True)
    check(T, orc, slots, sc, K, ids)


def test_invalid_ids_zero_rows_and_counted(T, orc):
    V, K = 50, 1024
    slots, sc = table(orc, V, K, seed=3)
    ids = np.array([-1, 0, V, 49, 2 ** 31 - 1, -(2 ** 31), 7, 7], dtype=np.int32)
    check(T, orc, slots, sc, K, ids)


def test_many_rows_and_single_row(T, orc):
    """70000 rows at K = 256 and a single row."""
    V, K = 200, 256
    slots, sc = table(orc, V, K, seed=5)
    rng = np.random.default_rng(9)
    check(T, orc, slots, sc, K, rng.integers(-2, V + 2, size=70000).astype(np.int32))
    check(T, orc, slots, sc, K, np.array([123], dtype=np.int32))


def test_grid_stride_reuse_and_tail_guard(T, orc):
    """More 64-weight items than the capped grid holds (70000 rows x K = 512
    -> 560000 items against 148 SMs x 16 blocks x 4 warps x 32 = 303104), so
    every warp takes a second pass and reuses its shared-memory stage; the
    row count leaves a ragged last warp item; a canary written after the
    output must be untouched."""
    V, K = 300, 512
    slots, sc = table(orc, V, K, seed=6, neg=True)
    rng = np.random.default_rng(10)
    ids = rng.integers(-2, V + 2, size=70001).astype(np.int32)
    M = ids.size
    canary = 4096
    buf = torch.full((M * K + canary,), -7.0, dtype=torch.float16, device="cuda")
    out = buf[: M * K].view(M, K)
    bad = torch.zeros(1, dtype=torch.int32, device="cuda")
    T.tern_embed_gather(torch.from_numpy(ids).cuda(), torch.from_numpy(slots).cuda(),
                        torch.from_numpy(sc.view(np.int16)).cuda().view(torch.float16), K, out=out, bad_count=bad)
    T.tern_sync_status()
    want, nbad = orc.embed(slots, sc, K, ids)
    got = out.cpu().float().double().numpy()
    assert int(bad.item()) == nbad
    assert np.array_equal(got, want)
    assert np.array_equal(np.signbit(got), np.signbit(want))
    assert bool(torch.all(buf[M * K:] == -7.0)), "the gather wrote past its output"


def test_tied_head_table(T, orc):
    """A head-shaped table (K = 5120) packed once and read both as the
    embedding table and as the output head: the gathered row of token v,
    dotted with x on the host, equals the head product's output v."""
    V, K = 4096, 5120
    slots, sc = table(orc, V, K, seed=11)
    sl_d = torch.from_numpy(slots).cuda()
    sc_d = torch.from_numpy(sc.view(np.int16)).cuda().view(torch.float16)
    ids = np.array([5, 4095, 1000], dtype=np.int32)
    rows = T.tern_embed_gather(torch.from_numpy(ids).cuda(), sl_d, sc_d, K)
    rng = np.random.default_rng(12)
    x = torch.from_numpy(rng.standard_normal(K)).half()
    y = T.tern_gemv(x.cuda(), sl_d, sc_d)
    T.tern_sync_status()
    want, _ = orc.embed(slots, sc, K, ids)
    assert np.array_equal(rows.cpu().double().numpy(), want)
    dots = want @ x.double().numpy()
    bound = np.abs(want) @ np.abs(x.double().numpy())
    got = y.cpu().double().numpy()[ids]
    assert np.all(np.abs(got - dots) <= 2e-3 * bound + 1e-5)
