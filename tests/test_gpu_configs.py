"""GPU parity at the full sizes of the five benchmark workloads, in the launch
configuration the benchmark times (one plan per mask, one forward each).

The oracle computes sampled rows one by one (first, middle and last rows of every
sequence plus random ones); tile classes of the GPU plans (host planner or device scan
of the packed bits) are compared bit for bit with the oracle's dense-mask classes; the
two descriptor forms of the chunk-causal and block-dense workloads must give identical
outputs.
"""
import numpy as np
import pytest
import torch

import workloads as W
import oracle
import masked_flash_attention_attn_b200 as M
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(attn_lib):
    assert torch.cuda.is_available()


def _classes_match(wl, spec, plan):
    cls = M.attn_plan_get_tile_classes(plan)
    assert np.array_equal(cls, oracle.tile_classes(spec, G.lengths(wl)))
    return cls


def test_config1_prefix_lm_full_compare():
    wl = W.config(1)
    G.check_full(wl, wl.masks[0], "config 1")


def test_config2_gemma2_local_global():
    wl = W.config(2)
    inputs = G.device_inputs(wl)
    res = []
    for spec in wl.masks:
        out, lse, plan = G.run(wl, spec, inputs)
        _classes_match(wl, spec, plan)
        G.check_sampled(wl, spec, out, lse, G.sample_rows(wl, 64, seed=2), f"config 2 {spec.kind}")
        res.append(out)
    # the window bites on the longest sequence: the two masks must differ there
    b = int(np.argmax([wl.lq(i) for i in range(wl.batch)]))
    last = int(wl.cu_seqlens_q[b + 1]) - 1
    assert wl.lq(b) > 4096 and not torch.equal(res[0][last], res[1][last])


def test_config3_tree_verify_paged_custom():
    wl = W.config(3)
    spec = wl.masks[0]
    out, lse, plan = G.run(wl, spec)
    _classes_match(wl, spec, plan)
    assert plan.stats["heads_per_tile"] == 2
    G.check_sampled(wl, spec, out, lse, G.sample_rows(wl, 96, seed=3), "config 3")


def test_config4_chunk_causal_both_forms():
    wl = W.config(4)
    inputs = G.device_inputs(wl)
    outs = []
    for spec in wl.masks:
        out, lse, plan = G.run(wl, spec, inputs)
        st = plan.stats
        assert (st["tiles_empty"], st["tiles_full"], st["tiles_partial"]) == (8 * 2016, 8 * 2016, 8 * 64)
        assert st["unmasked_pairs"] == 8 * 33560576
        outs.append((out, lse))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    G.check_sampled(wl, wl.masks[0], outs[0][0], outs[0][1], G.sample_rows(wl, 64, seed=4), "config 4")


def test_config5_block_dense_packed_vs_ranges():
    wl = W.config(5)
    inputs = G.device_inputs(wl)
    outs = []
    for spec in wl.masks:
        out, lse, plan = G.run(wl, spec, inputs)
        st = plan.stats
        assert (st["tiles_empty"], st["tiles_full"], st["tiles_partial"]) == (9202, 44544, 78)
        assert st["unmasked_pairs"] == 727112276
        outs.append((out, lse))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    rows = [24575, 24576, 24675, 24676, 27775, 27776, 29575, 0, 100]
    samples = [(0, h, i) for i, h in zip(rows, [0, 5, 9, 31, 16, 3, 30, 7, 8])]
    samples += G.sample_rows(wl, 40, seed=5)
    G.check_sampled(wl, wl.masks[0], outs[0][0], outs[0][1], samples, "config 5")
