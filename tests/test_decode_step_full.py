"""The decode step exactly as bench.py times it, against the fp64 oracle.

bench.py's DecodeModel: 64 synthetic layers (q 5120->6144, k/v 5120->1024,
o 6144->5120, gate/up 5120->17408, down 17408->5120) plus the 5120->151936
head, packed on the GPU by tern_pack_g128; one step is one tern_gemv_step
call over all 449 products (five launches), captured in a CUDA graph and
replayed.  Checked:
  * two whole layers (the first and the last) and the head: the codes are
    drawn again from the same seeds, packed by the oracle and compared with
    the GPU's slots and scales byte for byte, and every output is compared
    with the oracle's product;
  * every projection of the other 62 layers: 4096 rows (all rows where N is
    smaller) drawn at random, their slots and scales copied back, their
    outputs compared with the oracle's product of those rows.
The pages tie generation speed to the weight bytes read per token ("Bonsai
27B ternary / 1-bit quantization", ThakiCloud blog, section "Throughput and
speculative decoding"), which is why this is the configuration the benchmark
reports; this test proves its numbers come from correct products.
"""
import os

import numpy as np
import pytest
import torch

from helpers import check_close

pytestmark = pytest.mark.gpu
NCPU = os.cpu_count() or 1
SAMPLE_ROWS = 4096


def _bits(t):
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


@pytest.fixture(scope="module")
def stepped():
    from ternary_weight_only_b200 import build
    build.build()
    from ternary_weight_only_b200 import tern as T
    import bench
    model = bench.DecodeModel(T)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        model.step()  # first-call set-up outside capture, as bench.py does
        stream.synchronize()
        model.y_all.fill_(float("nan"))
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            model.step()
        graph.replay()
        graph.replay()
    stream.synchronize()
    T.tern_sync_status()
    yield T, model
    del graph


def _full_check(orc, T, model, name, K, N, codes, scales, slots_d, sc_d, x_d, y_d):
    cn = codes.cpu().numpy()
    sb = _bits(scales)
    slots, sc, bad, _ = orc.pack(cn, sb)
    assert bad == 0
    assert np.array_equal(slots_d.cpu().numpy(), slots), f"{name}: GPU slots differ from the oracle's"
    assert np.array_equal(_bits(sc_d), sc), f"{name}: GPU scales differ from the oracle's"
    y_ref, bound = orc.matmul(_bits(x_d).reshape(1, K), slots, sc, threads=NCPU)
    check_close(y_d.view(1, N), y_ref, bound, name)


def test_whole_layers_and_head(stepped, orc):
    from ternary_weight_only_b200 import synth
    T, model = stepped
    for l in (0, synth.N_LAYERS - 1):
        g = synth.gen(4000 + l, "cuda")
        for i, (name, K, N) in enumerate(synth.LAYER_PROJ):
            codes = synth.codes_sparse(N, K, g, device="cuda")
            scales = synth.scales_uniform(N, K, g, device="cuda")
            x_d, slots_d, sc_d, y_d = model.groups[l][i]
            _full_check(orc, T, model, f"layer {l} {name}", K, N, codes, scales, slots_d, sc_d, x_d, y_d)
    g = synth.gen(4000 + synth.N_LAYERS, "cuda")
    _, K, N = synth.HEAD
    codes = synth.codes_sparse(N, K, g, device="cuda")
    scales = synth.scales_uniform(N, K, g, device="cuda")
    _, _, _, slots_d, sc_d = model.head
    _full_check(orc, T, model, "head", K, N, codes, scales, slots_d, sc_d, model.head_io[0], model.head_io[1])


def test_sampled_rows_of_every_other_projection(stepped, orc):
    from ternary_weight_only_b200 import synth
    T, model = stepped
    rng = np.random.default_rng(4242)
    for l in range(1, synth.N_LAYERS - 1):
        for i, (name, K, N) in enumerate(synth.LAYER_PROJ):
            x_d, slots_d, sc_d, y_d = model.groups[l][i]
            n = min(SAMPLE_ROWS, N)
            rows = np.sort(rng.choice(N, size=n, replace=False))
            idx = torch.from_numpy(rows).cuda()
            slots = slots_d.index_select(0, idx).cpu().numpy()
            sc = _bits(sc_d.index_select(0, idx))
            y_ref, bound = orc.matmul(_bits(x_d).reshape(1, K), slots, sc, threads=NCPU)
            check_close(y_d.index_select(0, idx).view(1, n), y_ref, bound, f"layer {l} {name} (sampled rows)")
