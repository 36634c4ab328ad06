"""Host-side planner invariants through attn_plan_dry_run (no GPU): the tile classes and
pair counts match attn_classify_host, query-row shards partition the work list for every
kind (with and without head packing), forced splits keep every job exactly once, and the
shard arguments are validated."""
import pytest

import workloads as W

KINDS = ["FULL", "CAUSAL", "SLIDING_WINDOW", "PREFIX_LM", "CHUNK_CAUSAL", "RANGES", "BLOCK_SPARSE"]


def _kw(wl, spec):
    return dict(hq=wl.hq, hkv=wl.hkv, head_dim=wl.d, cu_seqlens_q=wl.cu_seqlens_q, cu_seqlens_k=wl.cu_seqlens_k,
                mask=spec)


@pytest.mark.parametrize("kind", KINDS)
def test_dry_run_matches_classify_host(attn_lib, kind):
    wl = W.random_small(seed=11 + len(kind), kind=kind, batch=3, hq=4, hkv=2, d=128, lmin=1, lmax=700)
    st = attn_lib.attn_plan_dry_run(**_kw(wl, wl.masks[0]))
    cls, pairs = attn_lib.attn_classify_host(**_kw(wl, wl.masks[0]))
    assert st["unmasked_pairs"] == pairs
    assert (st["tiles_empty"], st["tiles_full"], st["tiles_partial"]) == tuple(int((cls == c).sum()) for c in (0, 1, 2))


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("lmax", [40, 900])   # 40: short queries, several heads per 128-row tile
def test_query_shards_partition(attn_lib, kind, lmax):
    M = attn_lib
    wl = W.random_small(seed=5 + lmax + len(kind), kind=kind, batch=3, hq=8, hkv=2, d=128, lmin=1, lmax=lmax)
    kw = _kw(wl, wl.masks[0])
    full = M.attn_plan_dry_run(kv_splits=1, **kw)
    lq_max = max(wl.lq(b) for b in range(wl.batch))
    rows = full["heads_per_tile"] and 128 // full["heads_per_tile"]
    for world in (2, 3):
        per = -(-lq_max // (world * rows)) * rows            # whole row blocks per shard
        st = [M.attn_plan_dry_run(kv_splits=1, q_rows=(r * per, (r + 1) * per), **kw) for r in range(world)]
        assert sum(x["jobs"] for x in st) == full["jobs"], (kind, lmax, world)
        assert sum(x["mask_tile_reads"] for x in st) == full["mask_tile_reads"]
        # the tile classes and pair counts describe the whole problem whatever the shard
        assert all(x["unmasked_pairs"] == full["unmasked_pairs"] for x in st)


@pytest.mark.parametrize("kind", ["CAUSAL", "RANGES", "BLOCK_SPARSE"])
def test_forced_split_keeps_jobs(attn_lib, kind):
    wl = W.random_small(seed=21, kind=kind, batch=2, hq=4, hkv=2, d=64, lmin=300, lmax=1500)
    kw = _kw(wl, wl.masks[0])
    base = attn_lib.attn_plan_dry_run(kv_splits=1, **kw)
    for n in (2, 3, 9):
        st = attn_lib.attn_plan_dry_run(kv_splits=n, **kw)
        assert st["jobs"] == base["jobs"] and st["mask_tile_reads"] == base["mask_tile_reads"]
        assert base["work_items"] < st["work_items"] <= n * base["work_items"]
        assert st["kv_splits_max"] <= n


def test_shard_validation_and_empty_shard(attn_lib):
    M = attn_lib
    wl = W.random_small(seed=3, kind="CAUSAL", batch=2, hq=2, hkv=1, d=64, lmin=50, lmax=200)
    kw = _kw(wl, wl.masks[0])
    with pytest.raises(M.AttnError) as e:
        M.attn_plan_dry_run(q_rows=(100, 50), **kw)
    assert e.value.status == 1
    with pytest.raises(M.AttnError) as e:
        M.attn_plan_dry_run(q_rows=(-1, 10), **kw)
    assert e.value.status == 1
    st = M.attn_plan_dry_run(q_rows=(10000, 20000), **kw)          # past every sequence
    assert st["work_items"] == 0 and st["jobs"] == 0


@pytest.mark.parametrize("kind", ["CAUSAL", "RANGES", "BLOCK_SPARSE"])
def test_job_lists_are_shared_across_heads(attn_lib, kind):
    """Items over the same row blocks read one job list whatever their KV head: going from
    1 to 8 KV heads (same group size) multiplies the items and jobs by 8 but adds to the
    workspace only the items and per-CTA lists, never another copy of the job lists."""
    wl = W.random_small(seed=31, kind=kind, batch=3, hq=2, hkv=1, d=128, lmin=200, lmax=1500)
    kw = _kw(wl, wl.masks[0])
    one = attn_lib.attn_plan_dry_run(kv_splits=1, **kw)
    kw.update(hq=16, hkv=8)
    eight = attn_lib.attn_plan_dry_run(kv_splits=1, **kw)
    assert eight["work_items"] == 8 * one["work_items"] and eight["jobs"] == 8 * one["jobs"]
    grown = eight["workspace_bytes"] - one["workspace_bytes"]
    # 64-byte items, one int32 per listed item and per CTA offset, plus alignment of the parts
    assert grown <= (eight["work_items"] - one["work_items"]) * (64 + 4) + 4 * (eight["ctas"] + 1) + 8 * 256
    # copies of the 16-byte jobs per head would exceed that bound by more than its slack
    assert 16 * (eight["jobs"] - one["jobs"]) > 8 * 256


def test_noalloc_size_limit_premise(attn_lib):
    """The GPU test of the allocation-free entry's size limit relies on this problem needing
    more than its 32 MiB array (the limit is checked on the same host plan)."""
    from tests import gpu_helpers as G
    cq, kw = G.noalloc_too_large_problem()
    st = attn_lib.attn_plan_dry_run(cu_seqlens_q=cq, cu_seqlens_k=cq, mask=W.MaskSpec("FULL"), kv_splits=1, **kw)
    assert st["workspace_bytes"] > 1.5 * attn_lib.NOALLOC_SCRATCH_BYTES
