"""GPU parity of split-KV: work items cut into consecutive key ranges, each writing partial
results (out / l and lse per row) that a second kernel merges by their lse. Forced splits
on small problems of every mask kind and head dim, contiguous and paged, against the fp64
oracle; rows that see no key at all or none inside some ranges; a forward without lse;
automatic splitting on a long-context tree-verify workload (few long work items)."""
import numpy as np
import pytest
import torch

import workloads as W
import oracle
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu

KINDS = ["FULL", "CAUSAL", "SLIDING_WINDOW", "PREFIX_LM", "CHUNK_CAUSAL", "RANGES", "CUSTOM", "BLOCK_SPARSE"]


@pytest.fixture(scope="module", autouse=True)
def _lib(attn_lib):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return attn_lib


def _check_split(wl, spec, kv_splits, what):
    out, lse, plan = G.run(wl, spec, kv_splits=kv_splits)
    st = plan.stats
    assert st["kv_splits_max"] > 1 and st["merge_tiles"] > 0, f"{what}: nothing was split ({st})"
    ref_out, ref_lse = oracle.masked_attention(wl, spec)
    cls = G.M.attn_plan_get_tile_classes(plan)
    assert np.array_equal(cls, oracle.tile_classes(spec, G.lengths(wl))), f"{what}: tile classes"
    return G.compare(out, lse, ref_out, ref_lse, what)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("kind", KINDS)
def test_forced_split_all_kinds(kind, d):
    wl = W.random_small(seed=300 + d + 7 * KINDS.index(kind), kind=kind, batch=3, hq=4, hkv=2, d=d,
                        lmin=129, lmax=900)
    _check_split(wl, wl.masks[0], 3, f"split {kind} d={d}")


@pytest.mark.parametrize("d", [64, 128, 256])
def test_forced_split_paged(d):
    wl = W.random_small(seed=40 + d, kind="CUSTOM", batch=3, hq=4, hkv=2, d=d, lmin=129, lmax=700, paged=True)
    _check_split(wl, wl.masks[0], 4, f"split paged d={d}")


@pytest.mark.parametrize("n", [2, 5, 64])
def test_split_counts(n):
    # more ranges than key tiles: every item is cut into one range per key tile
    wl = W.random_small(seed=n, kind="CAUSAL", batch=2, hq=2, hkv=1, d=128, lmin=300, lmax=1000)
    _check_split(wl, wl.masks[0], n, f"kv_splits={n}")


def test_never_split():
    wl = W.random_small(seed=9, kind="CAUSAL", batch=2, hq=2, hkv=1, d=128, lmin=300, lmax=1000)
    out, lse, plan = G.run(wl, wl.masks[0], kv_splits=1)
    assert plan.stats["kv_splits_max"] == 1 and plan.stats["merge_tiles"] == 0
    G.compare(out, lse, *oracle.masked_attention(wl, wl.masks[0]), "kv_splits=1")


def test_split_masked_rows_and_ranges():
    # rows 0..9 see no key at all; rows 10..29 only keys in [0, 40) (the first range); the
    # rest a random pattern: the merge must give out = 0 / lse = -inf, and ignore ranges
    # in which a row saw nothing
    rng = np.random.default_rng(11)
    lq, lk = [200, 150], [900, 700]
    dense = []
    for a, b in zip(lq, lk):
        m = rng.random((a, b)) < 0.3
        m[:10] = False
        m[10:30] = False
        m[10:30, :40] = True
        dense.append(m)
    words, offs = [], [0]
    for m in dense:
        w = W.pack_rows(m)
        words.append(w.reshape(-1))
        offs.append(offs[-1] + w.size)
    spec = W.MaskSpec("CUSTOM", bits=np.concatenate(words).astype(np.uint32), word_offsets=np.asarray(offs, np.int64))
    gen = torch.Generator().manual_seed(3)
    cq, ck = W.cu_from_lengths(lq), W.cu_from_lengths(lk)
    wl = W.Workload(name="split_masked", hq=4, hkv=2, d=128, scale=0.09, cu_seqlens_q=cq,
                    q=W.randn_bf16(gen, int(cq[-1]), 4, 128), masks=[spec], cu_seqlens_k=ck,
                    k=W.randn_bf16(gen, int(ck[-1]), 2, 128), v=W.randn_bf16(gen, int(ck[-1]), 2, 128), seed=3)
    _check_split(wl, spec, 6, "masked rows under split")


def test_split_without_lse():
    wl = W.random_small(seed=21, kind="SLIDING_WINDOW", batch=2, hq=4, hkv=2, d=128, lmin=300, lmax=900)
    q, k, v = G.device_inputs(wl)
    plan = G.make_plan(wl, wl.masks[0], kv_splits=3)
    assert plan.stats["merge_tiles"] > 0
    tq = int(wl.cu_seqlens_q[-1])
    out = torch.empty(tq, wl.hq, wl.d, dtype=torch.bfloat16, device="cuda")
    G.M.attn_masked_fwd(plan, q, k, v, out, None)
    assert G.M.attn_plan_check_status(plan) == 0
    ref_out, ref_lse = oracle.masked_attention(wl, wl.masks[0])
    G.compare(out.float().cpu(), torch.from_numpy(ref_lse), ref_out, ref_lse, "split, lse=NULL")


def test_auto_split_long_context_verify():
    # 4 requests x 8 KV heads = 32 work items over 16K-32K keys: automatic split-KV cuts
    # them; sampled rows against the oracle, and the unsplit plan agrees as well
    wl = W.config(6)
    spec = wl.masks[0]
    q, k, v = G.device_inputs(wl)
    samples = G.sample_rows(wl, 48, seed=6)
    results = {}
    for n in (0, 1):
        out, lse, plan = G.run(wl, spec, inputs=(q, k, v), kv_splits=n)
        st = plan.stats
        if n == 0:
            assert st["kv_splits_max"] >= 3, st
        else:
            assert st["kv_splits_max"] == 1, st
        G.check_sampled(wl, spec, out, lse, samples, f"long verify kv_splits={n}")
        results[n] = out
    assert (results[0] - results[1]).abs().max().item() <= 2e-2
