"""Seeded synthetic inputs for the masked attention forward.

This module is shared by the tests, the benchmark and the smoke check. It
holds none of the attention arithmetic: it only draws lengths, tensors,
tree parents and page permutations from seeds and writes the mask
descriptors in the formats the library accepts.

Randomness:
  * integers (lengths, prefixes, tree parents, page permutation) come from
    ``numpy.random.default_rng(seed)``;
  * tensors are fp32 N(0, 1) from a CPU ``torch.Generator`` seeded with the
    same seed, rounded to bf16 (round-to-nearest-even, torch's cast).

Mask descriptor (``MaskSpec``) kinds and parameters, in the notation of the
pages they come from:
  FULL, CAUSAL                          plain attention / causal attention
  SLIDING_WINDOW(window)                "feat: add Gemma2 sliding-window (local/global)
                                        attention", Summary: local mask = causal AND
                                        within the window
  PREFIX_LM(prefix_len | prefix_lens)   "[Attention] feat: support PrefixLM",
                                        Highlights: bidirectional prefix, causal suffix
  CHUNK_CAUSAL(chunk)                   "Feature request: chunk-causal mask type for Flex
                                        Flash Attention", Desired representation
  RANGES(ranges per sequence)           same page, Current pattern / Proposed API
                                        (q_ranges, k_ranges, attn_type_map, chunk_size_map)
  CUSTOM(bits, word_offsets)            "Custom mask slows down attention." (bit-packed
                                        custom mask); "feat: support custom mask for
                                        flash attention" (custom_mask input)
  BLOCK_SPARSE(block_q, block_k, BSR)   "Custom mask slows down attention." (the sparse API
                                        recommended for long sequences): listed blocks visible

Packed CUSTOM layout: for each sequence, row-major ``[L_q][ceil(L_k/32)]``
uint32 words; key ``j`` of row ``i`` is bit ``j % 32`` (least significant bit
first) of word ``i * W + j // 32``. Sequences are concatenated; the start word
of sequence ``b`` is ``word_offsets[b]``. One mask is shared by every head.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

# range types of the range-list descriptor (0-3 follow the attn_type_map values printed
# on the chunk-causal page; 4 is this library's code for CHUNK_CAUSAL)
RANGE_FULL = 0
RANGE_CAUSAL = 1
RANGE_INV_CAUSAL = 2
RANGE_BI_CAUSAL = 3
RANGE_CHUNK_CAUSAL = 4

KINDS = ("FULL", "CAUSAL", "SLIDING_WINDOW", "PREFIX_LM", "CHUNK_CAUSAL", "RANGES", "CUSTOM", "BLOCK_SPARSE")

Range = Tuple[int, int, int, int, int, int]  # q_start, q_end, k_start, k_end, type, chunk_size


@dataclasses.dataclass
class MaskSpec:
    kind: str
    window: int = 0
    prefix_len: int = 0
    prefix_lens: Optional[np.ndarray] = None          # int32 [B] or None
    chunk: Optional[Range] = None                      # CHUNK_CAUSAL convenience kind
    ranges: Optional[List[List[Range]]] = None         # RANGES: per-sequence lists
    bits: Optional[np.ndarray] = None                  # CUSTOM: uint32 words
    word_offsets: Optional[np.ndarray] = None          # CUSTOM: int64 [B+1]
    block_q: int = 0                                   # BLOCK_SPARSE block height
    block_k: int = 0                                   # BLOCK_SPARSE block width
    bsr_row_ptr: Optional[np.ndarray] = None           # BLOCK_SPARSE: int32 [total block rows + 1]
    bsr_col_idx: Optional[np.ndarray] = None           # BLOCK_SPARSE: int32 block columns
    bsr_seq_row0: Optional[np.ndarray] = None          # BLOCK_SPARSE: first block row of each sequence

    def __post_init__(self):
        if self.kind not in KINDS:
            raise ValueError(f"unknown mask kind {self.kind}")


@dataclasses.dataclass
class Workload:
    name: str
    hq: int
    hkv: int
    d: int
    scale: float
    cu_seqlens_q: np.ndarray            # int32 [B+1]
    q: torch.Tensor                     # bf16 [total_q, hq, d] (CPU)
    masks: List[MaskSpec]
    # contiguous KV
    cu_seqlens_k: Optional[np.ndarray] = None   # int32 [B+1]
    k: Optional[torch.Tensor] = None            # bf16 [total_k, hkv, d]
    v: Optional[torch.Tensor] = None
    # paged KV
    kv_lens: Optional[np.ndarray] = None        # int32 [B]
    page_table: Optional[np.ndarray] = None     # int32 [B, max_pages]
    page_size: int = 0
    k_cache: Optional[torch.Tensor] = None      # bf16 [num_pages, page_size, hkv, d]
    v_cache: Optional[torch.Tensor] = None
    seed: int = 0
    notes: str = ""

    @property
    def batch(self) -> int:
        return len(self.cu_seqlens_q) - 1

    @property
    def paged(self) -> bool:
        return self.page_table is not None

    def lq(self, b: int) -> int:
        return int(self.cu_seqlens_q[b + 1] - self.cu_seqlens_q[b])

    def lk(self, b: int) -> int:
        if self.paged:
            return int(self.kv_lens[b])
        return int(self.cu_seqlens_k[b + 1] - self.cu_seqlens_k[b])

    def kv_of_seq(self, b: int) -> Tuple[torch.Tensor, torch.Tensor]:
        """Contiguous [L_k, hkv, d] K and V of sequence b (gathers pages if paged)."""
        if not self.paged:
            s, e = int(self.cu_seqlens_k[b]), int(self.cu_seqlens_k[b + 1])
            return self.k[s:e], self.v[s:e]
        n = self.lk(b)
        npg = (n + self.page_size - 1) // self.page_size
        pages = torch.as_tensor(self.page_table[b, :npg].astype(np.int64))
        kk = self.k_cache[pages].reshape(-1, self.hkv, self.d)[:n]
        vv = self.v_cache[pages].reshape(-1, self.hkv, self.d)[:n]
        return kk, vv


def randn_bf16(gen: torch.Generator, *shape) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)


def quantize_e4m3(t: torch.Tensor):
    """Per-tensor e4m3 quantisation of an input: scale = max |t| / 448 and the e4m3 bytes of
    t / scale (the library's round-to-nearest-even conversion), as a uint8 tensor."""
    amax = float(t.float().abs().max()) if t.numel() else 0.0
    scale = amax / 448.0 if amax > 0 else 1.0
    return (t.float() / scale).to(torch.float8_e4m3fn).view(torch.uint8), scale


def pack_rows(dense: np.ndarray) -> np.ndarray:
    """Pack a bool [rows, L_k] array into uint32 words, LSB = lowest key."""
    rows, lk = dense.shape
    w = (lk + 31) // 32
    padded = np.zeros((rows, w * 32), dtype=np.uint8)
    padded[:, :lk] = dense
    by = np.packbits(padded.reshape(rows, w * 4, 8), axis=-1, bitorder="little").reshape(rows, w * 4)
    return by.view("<u4").reshape(rows, w).copy()


def cu_from_lengths(lengths: Sequence[int]) -> np.ndarray:
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return cu


def _contiguous(name, seed, lq, lk, hq, hkv, d, scale, masks, notes=""):
    gen = torch.Generator().manual_seed(seed)
    cq, ck = cu_from_lengths(lq), cu_from_lengths(lk)
    q = randn_bf16(gen, int(cq[-1]), hq, d)
    k = randn_bf16(gen, int(ck[-1]), hkv, d)
    v = randn_bf16(gen, int(ck[-1]), hkv, d)
    return Workload(name=name, hq=hq, hkv=hkv, d=d, scale=scale, cu_seqlens_q=cq, q=q,
                    masks=masks, cu_seqlens_k=ck, k=k, v=v, seed=seed, notes=notes)


# --------------------------------------------------------------------------
# the five workloads of the masked-attention benchmark suite
# --------------------------------------------------------------------------

def prefix_lm_small(seed: int = 1) -> Workload:
    """PREFIX_LM, 1 sequence L=256, Hq=Hkv=4, d=64, scale 1/8, prefix_len=64."""
    return _contiguous("prefix_lm_L256_d64", seed, [256], [256], 4, 4, 64, 1.0 / 8.0,
                       [MaskSpec("PREFIX_LM", prefix_len=64)])


def gemma2_local_global(seed: int = 2, batch: int = 4, lo: int = 1024, hi: int = 8192,
                        window: int = 4096) -> Workload:
    """Gemma2-style local/global pair: B=4 ragged lengths U[1024, 8192], Hq=16, Hkv=8,
    d=256, SLIDING_WINDOW(4096) and CAUSAL on the same tensors."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(lo, hi + 1, size=batch).tolist()
    return _contiguous("gemma2_sliding4096_causal_d256", seed, lens, lens, 16, 8, 256, 1.0 / 16.0,
                       [MaskSpec("SLIDING_WINDOW", window=window), MaskSpec("CAUSAL")],
                       notes=f"lengths={lens}")


def tree_parents(rng: np.random.Generator, n: int) -> np.ndarray:
    """Node 0 is the root; node t >= 1 has a parent uniform over 0..t-1."""
    par = np.full(n, -1, dtype=np.int64)
    for t in range(1, n):
        par[t] = rng.integers(0, t)
    return par


def tree_visible(par: np.ndarray) -> np.ndarray:
    """bool [n, n]: node t sees its ancestors and itself (the tree structure only)."""
    n = len(par)
    vis = np.zeros((n, n), dtype=bool)
    for t in range(n):
        a = t
        while a >= 0:
            vis[t, a] = True
            a = par[a]
    return vis


def tree_verify_paged(seed: int = 3, requests: int = 32, plo: int = 512, phi: int = 4096,
                      drafts: int = 64, page_size: int = 16, hq: int = 32, hkv: int = 8,
                      d: int = 128, spare_pages: int = 64) -> Workload:
    """Speculative tree verify over a paged KV cache: prefix P ~ U[512, 4096], 64 draft
    tokens whose K/V are the last 64 slots of the request, page size 16, pages randomly
    permuted; draft row t sees the whole prefix plus its ancestors and itself."""
    rng = np.random.default_rng(seed)
    prefix = rng.integers(plo, phi + 1, size=requests)
    kv_lens = (prefix + drafts).astype(np.int32)
    npages = (kv_lens + page_size - 1) // page_size
    total_pages = int(npages.sum()) + spare_pages
    perm = rng.permutation(total_pages).astype(np.int32)
    max_pages = int(npages.max())
    page_table = np.full((requests, max_pages), -1, dtype=np.int32)
    pos = 0
    for b in range(requests):
        page_table[b, :npages[b]] = perm[pos:pos + npages[b]]
        pos += int(npages[b])
    words, offs = [], [0]
    for b in range(requests):
        par = tree_parents(rng, drafts)
        dense = np.zeros((drafts, int(kv_lens[b])), dtype=bool)
        dense[:, :int(prefix[b])] = True
        dense[:, int(prefix[b]):] = tree_visible(par)
        w = pack_rows(dense)
        words.append(w.reshape(-1))
        offs.append(offs[-1] + w.size)
    bits = np.concatenate(words).astype(np.uint32)
    gen = torch.Generator().manual_seed(seed)
    cq = cu_from_lengths([drafts] * requests)
    q = randn_bf16(gen, int(cq[-1]), hq, d)
    k_cache = randn_bf16(gen, total_pages, page_size, hkv, d)
    v_cache = randn_bf16(gen, total_pages, page_size, hkv, d)
    return Workload(name="tree_verify_paged_d128", hq=hq, hkv=hkv, d=d, scale=1.0 / np.sqrt(d),
                    cu_seqlens_q=cq, q=q,
                    masks=[MaskSpec("CUSTOM", bits=bits, word_offsets=np.asarray(offs, np.int64))],
                    kv_lens=kv_lens, page_table=page_table, page_size=page_size,
                    k_cache=k_cache, v_cache=v_cache, seed=seed,
                    notes=f"prefix_lens={prefix.tolist()}")


def chunk_causal_ranges(seqs: int, L: int, prefix: int, cs: int) -> List[List[Range]]:
    """The FULL-range form of a causal prefix followed by chunk-causal pairs: one CAUSAL
    range over the prefix and one FULL range per chunk, q=[s, s+cs), k=[0, s+cs)."""
    one = [(0, prefix, 0, prefix, RANGE_CAUSAL, 0)]
    for s in range(prefix, L, cs):
        e = min(s + cs, L)
        one.append((s, e, 0, e, RANGE_FULL, 0))
    return [list(one) for _ in range(seqs)]


def chunk_causal_interleaved(seed: int = 4, seqs: int = 8, L: int = 8192, prefix: int = 4096,
                             cs: int = 2, h: int = 16, d: int = 128) -> Workload:
    """CHUNK_CAUSAL interleaved token/latent pairs: causal prefix of 4096, then
    q_range=[4096, 8192), k_range=[0, 8192), chunk_size=2; also given as FULL ranges."""
    masks = [MaskSpec("CHUNK_CAUSAL", chunk=(prefix, L, 0, L, RANGE_CHUNK_CAUSAL, cs)),
             MaskSpec("RANGES", ranges=chunk_causal_ranges(seqs, L, prefix, cs))]
    return _contiguous("chunk_causal_L8192_d128", seed, [L] * seqs, [L] * seqs, h, h, d,
                       1.0 / np.sqrt(d), masks)


def block_dense_rows(r0: int, r1: int, L: int, dense_rows: int, block: int) -> np.ndarray:
    """bool [r1-r0, L] rows of the long block-dense mask."""
    rows = np.arange(r0, r1)[:, None]
    cols = np.arange(L)[None, :]
    m = cols < dense_rows
    bs = dense_rows + ((rows - dense_rows) // block) * block
    tail = (rows >= dense_rows) & (cols >= bs) & (cols <= rows)
    return m | tail


def block_dense_custom(seed: int = 5, L: int = 29576, dense_rows: int = 24576, block: int = 100,
                       hq: int = 32, hkv: int = 8, d: int = 128) -> Workload:
    """Long block-dense custom mask: rows < 24576 see keys [0, 24576); the last 5000 rows
    see [0, 24576) plus causal attention inside their own 100-row block."""
    w = (L + 31) // 32
    bits = np.empty(L * w, dtype=np.uint32)
    step = 2048
    for r0 in range(0, L, step):
        r1 = min(L, r0 + step)
        bits[r0 * w:r1 * w] = pack_rows(block_dense_rows(r0, r1, L, dense_rows, block)).reshape(-1)
    ranges = [(0, dense_rows, 0, dense_rows, RANGE_FULL, 0)]
    for s in range(dense_rows, L, block):
        e = min(s + block, L)
        ranges.append((s, e, 0, dense_rows, RANGE_FULL, 0))
        ranges.append((s, e, s, e, RANGE_CAUSAL, 0))
    masks = [MaskSpec("CUSTOM", bits=bits, word_offsets=np.asarray([0, L * w], np.int64)),
             MaskSpec("RANGES", ranges=[ranges])]
    return _contiguous("block_dense_custom_L29576_d128", seed, [L], [L], hq, hkv, d,
                       1.0 / np.sqrt(d), masks)


def tree_verify_long_paged(seed: int = 6, requests: int = 4) -> Workload:
    """Long-context tree verify (split-KV case): the tree-verify recipe with 4 requests and
    prefixes P ~ U[16384, 32768]; 32 (request, KV head) work items alone would fill 32 of
    148 SMs, so the key range of every item is split."""
    wl = tree_verify_paged(seed=seed, requests=requests, plo=16384, phi=32768)
    wl.name = "tree_verify_long_paged_d128"
    return wl


WORKLOADS_BY_NUMBER = {
    1: prefix_lm_small,
    2: gemma2_local_global,
    3: tree_verify_paged,
    4: chunk_causal_interleaved,
    5: block_dense_custom,
    6: tree_verify_long_paged,
}


def config(n: int, **kw) -> Workload:
    return WORKLOADS_BY_NUMBER[n](**kw)


def random_small(seed: int, kind: str, batch: int = 3, hq: int = 4, hkv: int = 2, d: int = 64,
                 lmin: int = 1, lmax: int = 300, paged: bool = False, page_size: int = 16,
                 equal_qk: bool = False) -> Workload:
    """A small ragged problem with random lengths and a random descriptor of one kind,
    sized for exhaustive comparison with the oracle."""
    rng = np.random.default_rng(seed)
    lq = rng.integers(lmin, lmax + 1, size=batch)
    lk = lq.copy() if equal_qk else np.maximum(lq, rng.integers(lmin, lmax + 1, size=batch))
    spec = random_mask_spec(rng, kind, lq, lk)
    gen = torch.Generator().manual_seed(seed)
    cq = cu_from_lengths(lq)
    q = randn_bf16(gen, int(cq[-1]), hq, d)
    scale = 1.0 / np.sqrt(d)
    if not paged:
        ck = cu_from_lengths(lk)
        k = randn_bf16(gen, int(ck[-1]), hkv, d)
        v = randn_bf16(gen, int(ck[-1]), hkv, d)
        return Workload(name=f"random_{kind}", hq=hq, hkv=hkv, d=d, scale=scale, cu_seqlens_q=cq, q=q,
                        masks=[spec], cu_seqlens_k=ck, k=k, v=v, seed=seed)
    npages = (lk + page_size - 1) // page_size
    total = int(npages.sum()) + 7
    perm = rng.permutation(total).astype(np.int32)
    pt = np.full((batch, max(1, int(npages.max()))), -1, dtype=np.int32)
    pos = 0
    for b in range(batch):
        pt[b, :npages[b]] = perm[pos:pos + npages[b]]
        pos += int(npages[b])
    kc = randn_bf16(gen, total, page_size, hkv, d)
    vc = randn_bf16(gen, total, page_size, hkv, d)
    return Workload(name=f"random_{kind}_paged", hq=hq, hkv=hkv, d=d, scale=scale, cu_seqlens_q=cq, q=q,
                    masks=[spec], kv_lens=lk.astype(np.int32), page_table=pt, page_size=page_size,
                    k_cache=kc, v_cache=vc, seed=seed)


def random_mask_spec(rng: np.random.Generator, kind: str, lq, lk) -> MaskSpec:
    B = len(lq)
    if kind in ("FULL", "CAUSAL"):
        return MaskSpec(kind)
    if kind == "SLIDING_WINDOW":
        return MaskSpec(kind, window=int(rng.integers(1, max(2, int(max(lk))) + 1)))
    if kind == "PREFIX_LM":
        return MaskSpec(kind, prefix_lens=np.asarray([rng.integers(0, int(x) + 1) for x in lk], np.int32))
    if kind == "CHUNK_CAUSAL":
        L = int(min(min(lq), min(lk)))
        qs = int(rng.integers(0, L + 1))
        return MaskSpec(kind, chunk=(qs, L, 0, L, RANGE_CHUNK_CAUSAL, int(rng.integers(1, 9))))
    if kind == "RANGES":
        per = []
        for b in range(B):
            rs = []
            for _ in range(int(rng.integers(0, 6))):
                a, c = sorted(rng.integers(0, int(lq[b]) + 1, size=2).tolist())
                e, f = sorted(rng.integers(0, int(lk[b]) + 1, size=2).tolist())
                t = int(rng.choice([RANGE_FULL, RANGE_CAUSAL, RANGE_INV_CAUSAL, RANGE_BI_CAUSAL,
                                    RANGE_CHUNK_CAUSAL]))
                rs.append((a, c, e, f, t, int(rng.integers(1, 6)) if t == RANGE_CHUNK_CAUSAL else 0))
            per.append(rs)
        return MaskSpec(kind, ranges=per)
    if kind == "BLOCK_SPARSE":
        bq, bk = int(rng.choice([16, 64, 128, 100])), int(rng.choice([32, 128, 77]))
        ptr, cols, row0 = [0], [], []
        for b in range(B):
            nbr, nbc = -(-int(lq[b]) // bq), -(-int(lk[b]) // bk)
            row0.append(len(ptr) - 1)
            for _ in range(nbr):
                sel = np.nonzero(rng.random(nbc) < rng.choice([0.1, 0.5, 0.9]))[0]
                cols.extend(rng.permutation(sel).tolist())   # unsorted on purpose
                ptr.append(len(cols))
        return MaskSpec(kind, block_q=bq, block_k=bk, bsr_row_ptr=np.asarray(ptr, np.int32),
                        bsr_col_idx=np.asarray(cols, np.int32), bsr_seq_row0=np.asarray(row0, np.int64))
    if kind == "CUSTOM":
        words, offs = [], [0]
        for b in range(B):
            dense = rng.random((int(lq[b]), int(lk[b]))) < rng.choice([0.02, 0.5, 0.97])
            # add structure: some fully visible and some empty column blocks
            if lk[b] > 150:
                dense[:, : int(lk[b]) // 3] = True
            w = pack_rows(dense)
            # the padding bits past L_k are undefined in the format: fill them with ones
            if lk[b] % 32:
                w[:, -1] |= np.uint32((0xFFFFFFFF << (int(lk[b]) % 32)) & 0xFFFFFFFF)
            words.append(w.reshape(-1))
            offs.append(offs[-1] + w.size)
        return MaskSpec(kind, bits=np.concatenate(words).astype(np.uint32) if words else np.zeros(0, np.uint32),
                        word_offsets=np.asarray(offs, np.int64))
    raise ValueError(kind)
