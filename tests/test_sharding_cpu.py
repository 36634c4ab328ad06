"""Host side of the long-sequence multi-GPU path: query shards partition the work exactly
(attn_plan_dry_run), and the K/V all-gather of row shards over gloo groups of 2 and 3 ranks
rebuilds the full tensors on every rank."""
import multiprocessing as mp
import os

import pytest
import torch

import workloads as W
from masked_flash_attention_attn_b200 import sharding as S


def test_query_shards_partition_the_work(attn_lib):
    M = attn_lib
    wl = W.config(5)
    spec = wl.masks[1]   # the range form (analytic: plannable on the host)
    kw = dict(hq=wl.hq, hkv=wl.hkv, head_dim=wl.d, cu_seqlens_q=wl.cu_seqlens_q, cu_seqlens_k=wl.cu_seqlens_k,
              mask=spec)
    full = M.attn_plan_dry_run(**kw)
    L = wl.lq(0)
    for world in (2, 3, 8):
        shards = [S.query_shard(L, r, world) for r in range(world)]
        assert shards[0][0] == 0 and shards[-1][1] == L
        assert all(a[1] == b[0] for a, b in zip(shards, shards[1:]))
        st = [M.attn_plan_dry_run(q_rows=sh, **kw) for sh in shards]
        assert sum(x["work_items"] for x in st) == full["work_items"]
        assert sum(x["jobs"] for x in st) == full["jobs"]
        jobs = [x["jobs"] for x in st]
        assert max(jobs) <= 1.25 * (sum(jobs) / world)     # balanced for this mask


def _gather_worker(rank, world, port, rows, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        full = torch.arange(rows * 6, dtype=torch.float32).reshape(rows, 2, 3)
        a, b = S.row_shard(rows, rank, world)
        got = S.all_gather_rows(full[a:b].clone(), rows)
        q.put((rank, bool(torch.equal(got, full))))
    finally:
        dist.destroy_process_group()


def _row_gather_worker(rank, world, port, rows, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = S.RowGather(rows, (2, 3), torch.float32, "cpu")
        ok = True
        for step in range(3):   # the same buffers serve every call
            full = (torch.arange(rows * 6, dtype=torch.float32) + 1000 * step).reshape(rows, 2, 3)
            a, b = S.row_shard(rows, rank, world)
            got = g.gather(full[a:b].clone())
            ok = ok and bool(torch.equal(got, full)) and got.shape[0] == rows
        ok = ok and g.bytes_received == (world - 1) * ((rows + world - 1) // world) * 6 * 4
        q.put((rank, ok))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("rows,world", [(10, 2), (7, 3), (2, 3)])
def test_row_gather_reuses_its_buffers_gloo(rows, world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29750 + 10 * world + rows
    procs = [ctx.Process(target=_row_gather_worker, args=(r, world, port, rows, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(ok for _, ok in res)


@pytest.mark.parametrize("rows,world", [(10, 2), (7, 2), (7, 3), (2, 3)])   # (2, 3): a rank holds no rows
def test_all_gather_rows_gloo(rows, world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29650 + 10 * world + rows
    procs = [ctx.Process(target=_gather_worker, args=(r, world, port, rows, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(ok for _, ok in res)


def test_balanced_shards_even_out_causal_work(attn_lib):
    """For a causal batch, equal row counts give the last rank most of the tiles; the
    work-balanced shards (from the host tile classes) give every rank about the same number
    of jobs, and the shards still partition the work list exactly."""
    M = attn_lib
    L = 16384
    cq = W.cu_from_lengths([L, L // 2])
    kw = dict(hq=8, hkv=2, head_dim=128, cu_seqlens_q=cq, cu_seqlens_k=cq, mask=W.MaskSpec("CAUSAL"))
    cls, _ = M.attn_classify_host(**kw)
    lengths = [(L, L), (L // 2, L // 2)]
    full = M.attn_plan_dry_run(kv_splits=1, **kw)
    world = 4
    equal = [S.query_shard(L, r, world) for r in range(world)]
    bal = S.balanced_query_shards(cls, lengths, world)
    assert bal[0][0] == 0 and bal[-1][1] == L and all(a[1] == b[0] for a, b in zip(bal, bal[1:]))
    jobs_eq = [M.attn_plan_dry_run(kv_splits=1, q_rows=sh, **kw)["jobs"] for sh in equal]
    jobs_bal = [M.attn_plan_dry_run(kv_splits=1, q_rows=sh, **kw)["jobs"] for sh in bal]
    assert sum(jobs_bal) == full["jobs"] == sum(jobs_eq)
    assert max(jobs_eq) > 1.3 * (full["jobs"] / world)         # equal rows: imbalanced
    assert max(jobs_bal) < 1.15 * (full["jobs"] / world)       # balanced within 15 %


def test_bench_shard_rows_plan_partitions_the_sequence(attn_lib):
    """bench.py --shard-rows: the shards it plans cover every query row once, in order, for
    the long block-dense sequence (range form on the host) and a causal batch."""
    import bench
    for wl in (W.config(5), W.config(4)):
        lq_max = max(wl.lq(b) for b in range(wl.batch))
        for world in (1, 2, 4, 8):
            sh = bench.shard_rows_plan(attn_lib, wl, world)
            assert len(sh) == world and sh[0][0] == 0 and sh[-1][1] == lq_max
            assert all(a[1] == b[0] and a[0] <= a[1] for a, b in zip(sh, sh[1:]))
            assert all(b % 128 == 0 or b == lq_max for _, b in sh)
