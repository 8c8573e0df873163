"""The metric's FLOP accounting: allowed (query, key, head) triples counted
from the mask, against their closed forms.  A document of length S with a
window W sees sum_i min(i + 1, W) = W(W + 1)/2 + (S - W) W keys (S >= W), or
S(S + 1)/2 with no window; the forward does 4 D and the backward 10 D flop
per triple (two and five D-long dot products, two flop each)."""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.join(os.path.dirname(__file__), ".."))


def _closed_form(S, W, docs, Hq):
    per_doc = S * (S + 1) // 2 if W <= 0 or W >= S else W * (W + 1) // 2 + (S - W) * W
    return per_doc * docs * Hq


def test_pairs_match_closed_forms():
    import bench
    from sink_sliding_window_b200 import synth
    for S, docs in ((4096, 4), (61440, 1), (128, 1), (1, 3)):
        cu = synth.uniform_cu_seqlens(docs, S)
        for W in (0, 1, 32, 128, 4096, 100000):
            assert bench.pairs(cu, W, 64) == _closed_form(S, W, docs, 64), (S, docs, W)


def test_headline_shapes():
    import bench
    from sink_sliding_window_b200 import synth
    cu4k = synth.uniform_cu_seqlens(4, 4096)
    assert bench.pairs(cu4k, 128, 64) == 132_136_960
    assert bench.pairs(cu4k, 0, 64) == 2_148_007_936
    cu60k = synth.uniform_cu_seqlens(1, 61440)
    assert bench.pairs(cu60k, 0, 64) == 120_797_921_280
    assert bench.pairs(cu60k, 128, 64) == 502_796_288
    fwd, bwd = bench.layer_flops(128)
    assert (fwd, bwd) == (4 * 64 * 132_136_960, 10 * 64 * 132_136_960)
    assert bench.step_flops() == sum(14 * 64 * bench.pairs(cu4k, w, 64) for w in bench.LAYERS)


def test_packed_documents_count_each_document_alone():
    import bench
    lens = [5, 0, 300, 129, 1]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    for W in (0, 128):
        want = sum(_closed_form(L, W, 1, 8) for L in lens if L > 0)
        assert bench.pairs(cu, W, 8) == want
