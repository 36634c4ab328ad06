"""Dense boolean masks from each descriptor kind (oracle; test infrastructure only).

Conventions (the pages leave these open; the readings taken are listed in the
design notes):
  * L_q, L_k are the query and key lengths of one sequence; query row i sits at
    key-space position pos(i) = i + L_k - L_q (queries are the last tokens).
  * M[i, j] = True means query row i may attend to key j.

Sources for each kind
  CAUSAL          j <= pos(i).
  SLIDING_WINDOW  "feat: add Gemma2 sliding-window (local/global) attention",
                  Summary: the local mask is the causal mask AND-ed with the window;
                  a key is kept when 0 <= pos(i) - j < w.
  PREFIX_LM       "[Attention] feat: support PrefixLM", Highlights
                  (prefixlm_mask_mod): bidirectional inside the prefix, causal
                  after it; keys [0, p) are visible to every row.
  RANGES          "Feature request: chunk-causal mask type for Flex Flash
                  Attention", Current pattern / Proposed API: a list of
                  (q_range, k_range, type) whose union is the mask.
                  FULL: every (i, j) in q_range x k_range; CAUSAL: additionally
                  j <= i in sequence-local coordinates. The same page names
                  INV_CAUSAL and BI_CAUSAL (attn_type_map 2, 3; "Why existing mask
                  types are not enough": BI_CAUSAL is an aligned band/intersection):
                  INV_CAUSAL keeps j - k_start >= i - q_start (the causal triangle
                  aligned to the top-left corner of the range rectangle); BI_CAUSAL
                  additionally keeps j - k_end <= i - q_end (bottom-right aligned
                  causal), i.e. the band between the two aligned diagonals.
  CHUNK_CAUSAL    same page, Desired representation: query chunk c of
                  [q_start + c*cs, q_start + (c+1)*cs) attends keys
                  [k_start, q_start + (c+1)*cs), the chunk end clipped to q_end
                  and the keys to k_range. The convenience kind adds a CAUSAL
                  range over [0, q_start) before the chunked part.
  BLOCK_SPARSE    "Custom mask slows down attention." (the sparse API the thread
                  recommends for long sequences, equivalent to a custom mask): query i
                  sees key j iff block (i // block_q, j // block_k) is listed in the
                  sequence's block rows (CSR over all sequences' block rows in order;
                  bsr_seq_row0[b] is sequence b's first block row).
  CUSTOM          "Custom mask slows down attention." (bit-packed mask) and
                  "feat: support custom mask for flash attention" (custom_mask):
                  row-major [L_q][ceil(L_k/32)] uint32 words, key j is bit j%32
                  (least significant first) of word j//32; bits past L_k ignored.
"""
from __future__ import annotations

import numpy as np

CLASS_EMPTY, CLASS_FULL, CLASS_PARTIAL = 0, 1, 2
R_FULL, R_CAUSAL, R_INV_CAUSAL, R_BI_CAUSAL, R_CHUNK = 0, 1, 2, 3, 4
TILE = 128


def unpack_rows(words: np.ndarray, rows: int, lk: int) -> np.ndarray:
    """uint32 [rows * W] (W = ceil(lk/32)) -> bool [rows, lk]."""
    w = (lk + 31) // 32
    if rows == 0 or lk == 0:
        return np.zeros((rows, lk), dtype=bool)
    words = np.asarray(words, dtype=np.uint32).reshape(rows, w)
    shifts = np.arange(32, dtype=np.uint32)
    bits = ((words[:, :, None] >> shifts[None, None, :]) & np.uint32(1)).astype(bool)
    return bits.reshape(rows, w * 32)[:, :lk]


def _range_or_into(m: np.ndarray, rng, r0: int, r1: int) -> None:
    """OR one range (q_start, q_end, k_start, k_end, type, cs) into rows [r0, r1) of m.
    Rows outside q_range and keys outside k_range are untouched (False for this range)."""
    qs, qe, ks, ke, typ, cs = (int(x) for x in rng)
    lk = m.shape[1]
    a, b = max(qs, r0), min(qe, r1)
    c, d = max(ks, 0), min(ke, lk)
    if a >= b or c >= d:
        return
    i = np.arange(a, b)[:, None]
    j = np.arange(c, d)[None, :]
    if typ == R_FULL:
        sub = np.ones((b - a, d - c), dtype=bool)
    elif typ == R_CAUSAL:
        sub = j <= i
    elif typ == R_INV_CAUSAL:
        sub = (j - ks) >= (i - qs)
    elif typ == R_BI_CAUSAL:
        sub = ((j - ks) >= (i - qs)) & ((j - ke) <= (i - qe))
    elif typ == R_CHUNK:
        ch = (i - qs) // cs
        end = np.minimum(qs + (ch + 1) * cs, qe)
        sub = j < end
    else:
        raise ValueError(f"unknown range type {typ}")
    m[a - r0:b - r0, c:d] |= sub


def dense_mask_rows(spec, b: int, lq: int, lk: int, r0: int, r1: int) -> np.ndarray:
    """Rows [r0, r1) of sequence b's dense mask, bool [r1 - r0, lk]."""
    i = np.arange(r0, r1)[:, None]
    j = np.arange(lk)[None, :]
    pos = i + (lk - lq)
    kind = spec.kind
    if kind == "FULL":
        return np.ones((r1 - r0, lk), dtype=bool)
    if kind == "CAUSAL":
        return np.broadcast_to(j <= pos, (r1 - r0, lk)).copy()
    if kind == "SLIDING_WINDOW":
        return (j <= pos) & (pos - j < int(spec.window))
    if kind == "PREFIX_LM":
        p = int(spec.prefix_lens[b]) if spec.prefix_lens is not None else int(spec.prefix_len)
        return (j < p) | (j <= pos)
    if kind == "RANGES" or kind == "CHUNK_CAUSAL":
        if kind == "RANGES":
            ranges = spec.ranges[b]
        else:
            qs = int(spec.chunk[0])
            ranges = [(0, qs, 0, qs, R_CAUSAL, 0), tuple(spec.chunk)]
        m = np.zeros((r1 - r0, lk), dtype=bool)
        for rg in ranges:
            _range_or_into(m, rg, r0, r1)
        return m
    if kind == "BLOCK_SPARSE":
        bq, bk = int(spec.block_q), int(spec.block_k)
        row0 = int(spec.bsr_seq_row0[b])      # first block row of sequence b in the CSR
        m = np.zeros((r1 - r0, lk), dtype=bool)
        for R in range(r0 // bq, -(-r1 // bq)):
            a, e = max(r0, R * bq), min(r1, (R + 1) * bq)
            for c in spec.bsr_col_idx[spec.bsr_row_ptr[row0 + R]:spec.bsr_row_ptr[row0 + R + 1]]:
                m[a - r0:e - r0, int(c) * bk:min(lk, (int(c) + 1) * bk)] = True
        return m
    if kind == "CUSTOM":
        w = (lk + 31) // 32
        off = int(spec.word_offsets[b])
        return unpack_rows(spec.bits[off + r0 * w: off + r1 * w], r1 - r0, lk)
    raise ValueError(kind)


def dense_mask(spec, b: int, lq: int, lk: int) -> np.ndarray:
    return dense_mask_rows(spec, b, lq, lk, 0, lq)


def tile_classes(spec, lengths, tile: int = TILE, row_block: int = 2048) -> np.ndarray:
    """Class of every tile x tile (q, k) tile of every sequence over its valid sub-rectangle:
    0 = all False, 1 = all True, 2 = mixed. Order: sequence, q tile, k tile (row-major).
    ``lengths`` is a list of (L_q, L_k)."""
    out = []
    for b, (lq, lk) in enumerate(lengths):
        nqt, nkt = -(-lq // tile), -(-lk // tile)
        cnt = np.zeros((nqt, nkt), dtype=np.int64)
        for r0 in range(0, lq, row_block):
            r1 = min(lq, r0 + row_block)
            m = dense_mask_rows(spec, b, lq, lk, r0, r1)
            pad = np.zeros((r1 - r0, nkt * tile), dtype=np.int64)
            pad[:, :lk] = m
            col = pad.reshape(r1 - r0, nkt, tile).sum(axis=2)
            qt = np.arange(r0, r1) // tile
            np.add.at(cnt, qt, col)
        rows_valid = np.minimum(tile, lq - np.arange(nqt) * tile)[:, None]
        cols_valid = np.minimum(tile, lk - np.arange(nkt) * tile)[None, :]
        total = rows_valid * cols_valid
        cls = np.where(cnt == 0, CLASS_EMPTY, np.where(cnt == total, CLASS_FULL, CLASS_PARTIAL))
        out.append(cls.reshape(-1))
    return np.concatenate(out).astype(np.uint8) if out else np.zeros(0, np.uint8)


def unmasked_pairs(spec, lengths, row_block: int = 2048) -> int:
    """Number of True entries summed over sequences (one head)."""
    n = 0
    for b, (lq, lk) in enumerate(lengths):
        for r0 in range(0, lq, row_block):
            r1 = min(lq, r0 + row_block)
            n += int(dense_mask_rows(spec, b, lq, lk, r0, r1).sum())
    return n
