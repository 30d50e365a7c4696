"""GPU slot packing against the oracle: bit-exact."""
import itertools

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


def _pack_both(T, orc, codes, scales):
    slots, sc = T.tern_pack_g128(codes.cuda(), scales.cuda())
    torch.cuda.synchronize()
    _, cn, sn = np_inputs(torch.zeros(1, 1, dtype=torch.float16), codes, scales)
    ref_slots, ref_sc, bad, _ = orc.pack(cn, sn)
    return slots.cpu().numpy(), sc.view(torch.int16).cpu().numpy().view(np.uint16), ref_slots, ref_sc, bad


def test_tiny_and_layer_shapes(T, orc):
    from ternary_weight_only_b200 import synth
    cases = [synth.tiny_gemv()] + [synth.decode_proj(i) for i in range(len(synth.LAYER_PROJ))]
    for x, codes, scales in cases:
        s, sc, rs, rsc, bad = _pack_both(T, orc, codes, scales)
        assert bad == 0
        assert np.array_equal(s, rs)
        assert np.array_equal(sc, rsc)


@pytest.mark.parametrize("N,K", [(1, 128), (3, 256), (17, 384), (100, 1024), (5, 17408)])
def test_ragged_shapes(T, orc, N, K):
    from ternary_weight_only_b200 import synth
    _, codes, scales = synth.case(1, K, N, seed=N * 7 + K)
    s, sc, rs, rsc, _ = _pack_both(T, orc, codes, scales)
    assert np.array_equal(s, rs) and np.array_equal(sc, rsc)


def test_exhaustive_bytes_and_roundtrip(T, orc):
    tuples = list(itertools.product((-1, 0, 1), repeat=4))
    codes = torch.zeros((81, 128), dtype=torch.int8)
    for r, t in enumerate(tuples):
        codes[r, :4] = torch.tensor(t, dtype=torch.int8)
        codes[r, 4:8] = torch.tensor(tuples[(r * 7) % 81], dtype=torch.int8)
    scales = torch.rand((81, 1)).half()
    s, sc, rs, rsc, _ = _pack_both(T, orc, codes, scales)
    assert np.array_equal(s, rs)
    assert len(set(s[:, 0].tolist())) == 81
    back = T.tern_unpack_g128(torch.from_numpy(s).cuda(), 128).cpu()
    assert torch.equal(back, codes)


def test_unpack_all_256_bytes(T, orc):
    slots = np.tile(np.arange(256, dtype=np.uint8), (1, 1)).reshape(8, 32)
    got = T.tern_unpack_g128(torch.from_numpy(slots).cuda(), 128).cpu().numpy()
    want, bad = orc.unpack(slots, 128)
    assert np.array_equal(got, want)
    assert bad == int(sum(((b >> (2 * j)) & 3) == 3 for b in range(256) for j in range(4)))


def test_invalid_codes_counted(T, orc):
    codes = torch.zeros((4, 256), dtype=torch.int8)
    codes[0, 3] = 2
    codes[1, 200] = -2
    codes[3, 255] = 127
    codes[2, 0] = -128
    scales = torch.ones((4, 2)).half()
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    slots, _ = T.tern_pack_g128(codes.cuda(), scales.cuda(), invalid_count=cnt)
    torch.cuda.synchronize()
    assert int(cnt.item()) == 4
    _, cn, sn = np_inputs(torch.zeros(1, 1).half(), codes, scales)
    rs, _, bad, _ = orc.pack(cn, sn)
    assert bad == 4 and np.array_equal(slots.cpu().numpy(), rs)


def test_in_place_scales(T, orc):
    from ternary_weight_only_b200 import synth
    _, codes, scales = synth.case(1, 512, 64, seed=5)
    sd = scales.cuda()
    slots, sc = T.tern_pack_g128(codes.cuda(), sd, scales_out=sd)
    torch.cuda.synchronize()
    assert sc.data_ptr() == sd.data_ptr() and torch.equal(sc.cpu(), scales)


def test_head_shape_sampled_rows(T, orc):
    """The 5120 -> 151936 head: packed on the GPU in full, 2048 rows checked."""
    from ternary_weight_only_b200 import synth
    N, K = 151936, 5120
    g = synth.gen(77, "cuda")
    codes = synth.codes_sparse(N, K, g, device="cuda")
    scales = synth.scales_uniform(N, K, g, device="cuda")
    slots, sc = T.tern_pack_g128(codes, scales)
    torch.cuda.synchronize()
    rows = torch.from_numpy(np.random.default_rng(0).choice(N, 2048, replace=False)).cuda()
    rows = torch.cat([rows, torch.tensor([0, N - 1], device="cuda")])
    c_rows = codes[rows].cpu()
    s_rows = scales[rows].cpu()
    _, cn, sn = np_inputs(torch.zeros(1, 1).half(), c_rows, s_rows)
    rs, rsc, bad, _ = orc.pack(cn, sn)
    assert bad == 0
    assert np.array_equal(slots[rows].cpu().numpy(), rs)
    assert np.array_equal(sc[rows].view(torch.int16).cpu().numpy().view(np.uint16), rsc)
