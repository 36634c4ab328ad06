"""One long sequence over several GPUs: query-row shards plus one K/V all-gather.

Every rank computes a contiguous range of query rows of every sequence (attn_problem_t
q_begin / q_end, whole row blocks) against all keys; K and V are sharded by rows across
the ranks beforehand, so the exchange step is one all-gather that lands every rank's K/V
rows in every GPU's own memory (NCCL over NVLink; no peer memory is read by a kernel).
Outputs stay sharded by query rows. This module holds only the shard arithmetic and the
torch.distributed plumbing; the attention itself runs in the library's kernels.
"""
from __future__ import annotations


def query_shard(lq_max: int, rank: int, world: int, block: int = 128):
    """Sequence-local rows [begin, end) of `rank`: equal whole blocks of `block` rows."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad rank / world")
    blocks = (lq_max + block - 1) // block
    per = (blocks + world - 1) // world
    begin = min(lq_max, rank * per * block)
    end = min(lq_max, (rank + 1) * per * block)
    return begin, end


def row_shard(rows: int, rank: int, world: int):
    """Rows [begin, end) of a row-sharded tensor (K or V) owned by `rank`: equal parts, the
    last one shorter."""
    per = (rows + world - 1) // world
    return min(rows, rank * per), min(rows, (rank + 1) * per)


def all_gather_rows(local, rows: int, group=None):
    """All-gather a row-sharded tensor (this rank's rows from row_shard) into the full
    [rows, ...] tensor on every rank: one all_gather_into_tensor over equal padded parts."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    per = (rows + world - 1) // world
    buf = torch.zeros((per,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    buf[:local.shape[0]] = local
    out = torch.empty((per * world,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    dist.all_gather_into_tensor(out, buf, group=group)
    return out[:rows]


class RowGather:
    """all_gather_rows with buffers allocated once: every call sends this rank's rows of a
    row-sharded [rows, ...] tensor and receives the full tensor (one all_gather_into_tensor
    over equal padded parts; with one rank, a copy). For a step that repeats the gather (a
    timed loop, every layer of a model), so that no allocation happens per call."""

    def __init__(self, rows: int, feature_shape, dtype, device, group=None):
        import torch
        import torch.distributed as dist
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
        self.rows = rows
        self.per = (rows + self.world - 1) // self.world
        self.send = torch.zeros((self.per,) + tuple(feature_shape), dtype=dtype, device=device)
        self.full = torch.empty((self.per * self.world,) + tuple(feature_shape), dtype=dtype, device=device)

    def gather(self, local):
        """local: this rank's rows (row_shard(rows, rank, world)); returns the full [rows, ...]
        tensor (a view of the receive buffer, valid until the next call)."""
        import torch.distributed as dist
        n = local.shape[0]
        if n > self.per:
            raise ValueError("local rows exceed this rank's share")
        self.send[:n].copy_(local)
        if self.world == 1:
            self.full[:self.per].copy_(self.send)
        else:
            dist.all_gather_into_tensor(self.full, self.send, group=self.group)
        return self.full[:self.rows]

    @property
    def bytes_received(self) -> int:
        """Bytes that land on this rank per call (the other ranks' parts)."""
        return (self.world - 1) * self.send.numel() * self.send.element_size()


def balanced_query_shards(tile_classes, lengths, world: int, block: int = 128):
    """Row shards [begin, end) for every rank (sequence-local rows, whole `block`-row tiles)
    that give each rank about the same number of non-empty 128 x 128 tiles, summed over the
    sequences of the batch (causal masks put more work in later rows than equal row counts
    would). tile_classes: the classes attn_classify_host returns (sequence, query tile, key
    tile order; 0 = empty); lengths: [(L_q, L_k)] per sequence. Returns `world` pairs; ranks
    past the last row get empty shards."""
    import numpy as np
    if world <= 0:
        raise ValueError("bad world")
    n_qt_max = max(((lq + block - 1) // block for lq, _ in lengths), default=0)
    work = np.zeros(n_qt_max, np.int64)
    pos = 0
    for lq, lk in lengths:
        n_qt, n_kt = (lq + block - 1) // block, (lk + block - 1) // block
        cls = np.asarray(tile_classes[pos:pos + n_qt * n_kt]).reshape(n_qt, n_kt) if n_qt * n_kt else None
        if cls is not None:
            work[:n_qt] += (cls != 0).sum(axis=1) + 1     # + 1: per-tile fixed cost
        pos += n_qt * n_kt
    if pos != len(tile_classes):
        raise ValueError("tile_classes do not match lengths")
    cum = np.concatenate([[0], np.cumsum(work)])
    total = cum[-1]
    bounds = [0]
    for r in range(1, world):
        bounds.append(int(np.searchsorted(cum, total * r / world, side="left")))
    bounds.append(n_qt_max)
    bounds = np.maximum.accumulate(np.clip(bounds, 0, n_qt_max))
    lq_max = max((lq for lq, _ in lengths), default=0)
    return [(min(lq_max, int(a) * block), min(lq_max, int(b) * block)) for a, b in zip(bounds[:-1], bounds[1:])]
