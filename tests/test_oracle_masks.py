"""Pins of the oracle's mask builders and tile classifier (CPU).

Each test checks the oracle against something other than itself: the worked
example and equivalences printed on the pages, closed-form counts derived by
hand for the benchmark workloads, and a hand-written bit-format fixture.
"""
import os

import numpy as np
import pytest

import workloads as W
from oracle import masks as OM

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _ranges_spec(per_seq):
    return W.MaskSpec("RANGES", ranges=per_seq)


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ---- "Feature request: chunk-causal mask type for Flex Flash Attention" -------------

def test_chunk_causal_worked_example_matches_printed_full_ranges():
    rows = _read_golden("chunk_causal_worked_example.txt")
    chunk = [int(x) for x in rows[0][1:]]
    qs, qe, ks, ke, cs = chunk
    printed = [[int(x) for x in r[1:]] for r in rows[1:]]
    L = qe
    cc = _ranges_spec([[(qs, qe, ks, ke, W.RANGE_CHUNK_CAUSAL, cs)]])
    m = OM.dense_mask(cc, 0, L, L)
    # every printed FULL range: its rows see exactly k_range and nothing else
    for a, b, c, d in printed:
        for i in range(a, b):
            want = np.zeros(L, bool)
            want[c:d] = True
            assert np.array_equal(m[i], want), (i, a, b, c, d)
    # the whole progression (first two entries fix the step, the last closes it)
    step = printed[1][0] - printed[0][0]
    assert printed[1][3] - printed[0][3] == step
    full = [(s, s + step, 0, s + step, W.RANGE_FULL, 0) for s in range(printed[0][0], printed[-1][1], step)]
    assert full[-1][:4] == tuple(printed[-1])
    mf = OM.dense_mask(_ranges_spec([full]), 0, L, L)
    assert np.array_equal(m, mf)
    # rows before q_start are outside every range
    assert not m[:qs].any()


def test_chunk_causal_is_not_causal_token_sees_latent():
    """The page: under CAUSAL token_i cannot attend to latent_i; under CHUNK_CAUSAL it can."""
    L, qs = 200, 100
    cc = OM.dense_mask(_ranges_spec([[(qs, L, 0, L, W.RANGE_CHUNK_CAUSAL, 2)]]), 0, L, L)
    ca = OM.dense_mask(_ranges_spec([[(qs, L, 0, L, W.RANGE_CAUSAL, 0)]]), 0, L, L)
    for t in range(qs, L, 2):            # token_t at even offset, latent_t right after it
        assert cc[t, t + 1] and not ca[t, t + 1]
    assert not np.array_equal(cc, ca)
    # every chunk of size >= 2 differs from causal
    for cs in (2, 3, 5, 8):
        m = OM.dense_mask(_ranges_spec([[(qs, L, 0, L, W.RANGE_CHUNK_CAUSAL, cs)]]), 0, L, L)
        assert not np.array_equal(m, ca)


@pytest.mark.parametrize("L,qs", [(37, 0), (64, 10), (130, 129)])
def test_chunk_size_one_equals_causal(L, qs):
    one = OM.dense_mask(_ranges_spec([[(qs, L, 0, L, W.RANGE_CHUNK_CAUSAL, 1)]]), 0, L, L)
    ca = OM.dense_mask(_ranges_spec([[(qs, L, 0, L, W.RANGE_CAUSAL, 0)]]), 0, L, L)
    assert np.array_equal(one, ca)


def test_chunk_causal_convenience_kind_equals_range_form():
    L = 300
    for qs, cs in [(100, 2), (0, 7), (300, 3), (257, 4)]:
        a = OM.dense_mask(W.MaskSpec("CHUNK_CAUSAL", chunk=(qs, L, 0, L, W.RANGE_CHUNK_CAUSAL, cs)), 0, L, L)
        b = OM.dense_mask(_ranges_spec(W.chunk_causal_ranges(1, L, qs, cs)), 0, L, L)
        assert np.array_equal(a, b), (qs, cs)
    # with the prefix covering everything it is plain causal
    a = OM.dense_mask(W.MaskSpec("CHUNK_CAUSAL", chunk=(L, L, 0, L, W.RANGE_CHUNK_CAUSAL, 2)), 0, L, L)
    assert np.array_equal(a, OM.dense_mask(W.MaskSpec("CAUSAL"), 0, L, L))


def test_chunk_clipped_at_q_end_and_k_range():
    # last chunk shorter than chunk_size; keys limited to k_range
    m = OM.dense_mask(_ranges_spec([[(2, 9, 1, 8, W.RANGE_CHUNK_CAUSAL, 3)]]), 0, 10, 10)
    # chunks: [2,5) -> keys [1,5); [5,8) -> [1,8); [8,9) -> [1, min(9, 8)) = [1,8)
    exp = np.zeros((10, 10), bool)
    exp[2:5, 1:5] = True
    exp[5:8, 1:8] = True
    exp[8, 1:8] = True
    assert np.array_equal(m, exp)


# ---- "feat: add Gemma2 sliding-window (local/global) attention" --------------------

def test_sliding_window_inert_equals_causal_and_biting_differs():
    g = dict((r[0], int(r[1])) for r in _read_golden("sliding_window_inert.txt"))
    L, w, w_min = g["max_seq"], g["window_default"], g["window_inert_min"]
    assert w >= w_min == L
    ca = OM.dense_mask(W.MaskSpec("CAUSAL"), 0, L, L)
    assert np.array_equal(OM.dense_mask(W.MaskSpec("SLIDING_WINDOW", window=w), 0, L, L), ca)
    assert np.array_equal(OM.dense_mask(W.MaskSpec("SLIDING_WINDOW", window=w_min), 0, L, L), ca)
    bite = OM.dense_mask(W.MaskSpec("SLIDING_WINDOW", window=w_min - 1), 0, L, L)
    assert not np.array_equal(bite, ca)
    # the local mask is the causal mask AND the window: never more keys than causal
    assert not (bite & ~ca).any()
    # window w keeps exactly min(w, pos+1) keys per row
    for w in (1, 2, 17, 128):
        m = OM.dense_mask(W.MaskSpec("SLIDING_WINDOW", window=w), 0, L, L)
        assert np.array_equal(m.sum(1), np.minimum(w, np.arange(L) + 1))


def test_sliding_window_ragged_queries_bottom_right():
    lq, lk = 5, 12
    m = OM.dense_mask(W.MaskSpec("SLIDING_WINDOW", window=3), 0, lq, lk)
    for i in range(lq):
        p = i + lk - lq
        assert set(np.nonzero(m[i])[0]) == {p - 2, p - 1, p}


# ---- "[Attention] feat: support PrefixLM" ------------------------------------------

def test_prefix_lm_zero_is_causal_and_prefix_is_bidirectional():
    L = 70
    ca = OM.dense_mask(W.MaskSpec("CAUSAL"), 0, L, L)
    assert np.array_equal(OM.dense_mask(W.MaskSpec("PREFIX_LM", prefix_len=0), 0, L, L), ca)
    p = 20
    m = OM.dense_mask(W.MaskSpec("PREFIX_LM", prefix_len=p), 0, L, L)
    assert m[:p, :p].all()                      # bidirectional inside the prefix
    assert not m[:p, p:].any()                  # prefix rows do not see the suffix
    assert np.array_equal(m[p:], ca[p:] | (np.arange(L) < p)[None, :])
    assert np.array_equal(m[p:, p:], ca[p:, p:])  # causal after the prefix
    # prefix covering the sequence is FULL
    assert OM.dense_mask(W.MaskSpec("PREFIX_LM", prefix_len=L), 0, L, L).all()


# ---- causal, full ---------------------------------------------------------------------

def test_causal_decode_row_sees_everything_and_full():
    m = OM.dense_mask(W.MaskSpec("CAUSAL"), 0, 1, 33)
    assert m.all()
    m = OM.dense_mask(W.MaskSpec("CAUSAL"), 0, 4, 4)
    assert np.array_equal(m, np.tril(np.ones((4, 4), bool)))
    assert OM.dense_mask(W.MaskSpec("FULL"), 0, 3, 5).all()


# ---- CUSTOM bit format -------------------------------------------------------------

def test_custom_bit_format_fixture():
    # row 0: keys 0 and 2 (word 0b101); row 1: key 33 only (bit 1 of word 1) ; L_k = 35
    words = np.array([0x5, 0x0, 0x0, 0x2 | 0xFFFFFFF8], dtype=np.uint32)  # bits past L_k are ignored
    m = OM.unpack_rows(words, 2, 35)
    exp = np.zeros((2, 35), bool)
    exp[0, [0, 2]] = True
    exp[1, 33] = True
    assert np.array_equal(m, exp)
    spec = W.MaskSpec("CUSTOM", bits=words, word_offsets=np.array([0, 4], np.int64))
    assert np.array_equal(OM.dense_mask(spec, 0, 2, 35), exp)


@pytest.mark.parametrize("lk", [1, 31, 32, 33, 200])
def test_custom_pack_unpack_round_trip(lk):
    rng = np.random.default_rng(lk)
    d = rng.random((7, lk)) < 0.4
    assert np.array_equal(OM.unpack_rows(W.pack_rows(d).reshape(-1), 7, lk), d)


def test_custom_equals_descriptor_for_every_kind():
    rng = np.random.default_rng(0)
    lq, lk = 45, 77
    for kind in ("FULL", "CAUSAL", "SLIDING_WINDOW", "PREFIX_LM", "RANGES", "CHUNK_CAUSAL"):
        spec = W.random_mask_spec(rng, kind, np.array([lq]), np.array([lk]))
        d = OM.dense_mask(spec, 0, lq, lk)
        bits = W.pack_rows(d).reshape(-1)
        cu = W.MaskSpec("CUSTOM", bits=bits, word_offsets=np.array([0, bits.size], np.int64))
        assert np.array_equal(OM.dense_mask(cu, 0, lq, lk), d)


def test_tree_mask_structure():
    rng = np.random.default_rng(3)
    par = W.tree_parents(rng, 64)
    vis = W.tree_visible(par)
    assert vis[0, 0] and vis[0].sum() == 1
    for t in range(1, 64):
        assert 0 <= par[t] < t
        assert vis[t, t] and vis[t, par[t]]
        assert np.array_equal(vis[t] & ~np.eye(64, dtype=bool)[t], vis[par[t]])


# ---- tile classes and pair counts of the benchmark workloads (closed forms) ----------

def _counts(cls):
    return (int((cls == 0).sum()), int((cls == 1).sum()), int((cls == 2).sum()))


def test_config1_prefix_lm_tiles_and_pairs():
    spec = W.MaskSpec("PREFIX_LM", prefix_len=64)
    # 2x2 tiles: (0,0) partial (row 0 sees only the prefix), (0,1) empty, (1,0) full, (1,1) diagonal
    assert list(OM.tile_classes(spec, [(256, 256)])) == [2, 0, 1, 2]
    # sum_i max(64, i+1) = 64*64 + sum_{i=64}^{255} (i+1)
    assert OM.unmasked_pairs(spec, [(256, 256)]) == 64 * 64 + (65 + 256) * 192 // 2 == 34912


def test_config4_chunk_causal_tiles_and_pairs_one_sequence():
    L, p = 8192, 4096
    spec = W.MaskSpec("CHUNK_CAUSAL", chunk=(p, L, 0, L, W.RANGE_CHUNK_CAUSAL, 2))
    cls = OM.tile_classes(spec, [(L, L)])
    # q tiles 0..31: causal -> F below the diagonal (496), 32 diagonal P;
    # q tiles 32..63: every row sees up to its chunk end (<= its tile end) -> F = sum_{i=32}^{63} i
    assert _counts(cls) == (2016, 2016, 64)
    # causal prefix sum_{i<4096}(i+1); chunk part: odd rows see i+1 keys, even rows i+2
    pairs = p * (p + 1) // 2 + ((p + 1) + L) * (L - p) // 2 + (L - p) // 2
    assert pairs == 33560576
    assert OM.unmasked_pairs(spec, [(L, L)]) == pairs
    rng_spec = W.MaskSpec("RANGES", ranges=W.chunk_causal_ranges(1, L, p, 2))
    assert np.array_equal(OM.tile_classes(rng_spec, [(L, L)]), cls)


def test_config5_block_dense_tiles_pairs_and_packed_equals_ranges():
    L, dense, blk = 29576, 24576, 100
    w = (L + 31) // 32
    ranges = [(0, dense, 0, dense, W.RANGE_FULL, 0)]
    for s in range(dense, L, blk):
        e = min(s + blk, L)
        ranges += [(s, e, 0, dense, W.RANGE_FULL, 0), (s, e, s, e, W.RANGE_CAUSAL, 0)]
    rng_spec = W.MaskSpec("RANGES", ranges=[ranges])
    cls = OM.tile_classes(rng_spec, [(L, L)])
    # 232x232 tiles: F = 192*192 (dense block) + 40*192 (tail rows over the dense keys);
    # P = 40 diagonal + 38 sub-diagonal (a 100-row block straddles every 128-row tile
    # boundary except the one at relative row 3200 = 25*128); E = the rest
    assert _counts(cls) == (232 * 232 - 44544 - 78, 44544, 78) == (9202, 44544, 78)
    pairs = dense * dense + (L - dense) * dense + (L - dense) // blk * (blk * (blk + 1) // 2)
    assert pairs == 727112276
    assert OM.unmasked_pairs(rng_spec, [(L, L)]) == pairs
    # the packed form of the generator equals the range form, checked on row blocks that
    # include the dense/tail boundary, a straddling block and the ragged last tile
    for r0, r1 in [(0, 64), (24500, 24700), (27700, 27900), (29400, 29576)]:
        packed = W.pack_rows(W.block_dense_rows(r0, r1, L, dense, blk)).reshape(-1)
        spec_b = W.MaskSpec("CUSTOM", bits=np.concatenate([np.zeros(r0 * w, np.uint32), packed]),
                            word_offsets=np.array([0, r1 * w], np.int64))
        a = OM.dense_mask_rows(spec_b, 0, L, L, r0, r1)
        b = OM.dense_mask_rows(rng_spec, 0, L, L, r0, r1)
        assert np.array_equal(a, b), (r0, r1)


def test_tile_classes_ragged_valid_rectangle():
    # L_q = 130, L_k = 129: the tile (1, 1) has 2 valid rows and 1 valid column
    spec = W.MaskSpec("FULL")
    assert list(OM.tile_classes(spec, [(130, 129)])) == [1, 1, 1, 1]
    spec = W.MaskSpec("CAUSAL")
    # pos(i) = i - 1: rows 128, 129 of tile (1,1) see key 128 only for i = 129
    assert list(OM.tile_classes(spec, [(130, 129)])) == [2, 0, 1, 2]
    assert list(OM.tile_classes(spec, [(0, 5)])) == []


# ---- INV_CAUSAL and BI_CAUSAL range types (the page names them; readings in the header) ----

def _one_range(typ, qs, qe, ks, ke, L=None):
    L = L or max(qe, ke)
    return OM.dense_mask(_ranges_spec([[(qs, qe, ks, ke, typ, 0)]]), 0, L, L)


def test_inv_causal_square_is_transposed_causal():
    L = 37
    inv = _one_range(W.RANGE_INV_CAUSAL, 0, L, 0, L)
    ca = _one_range(W.RANGE_CAUSAL, 0, L, 0, L)
    assert np.array_equal(inv, ca.T)
    assert np.array_equal(inv | ca, np.ones((L, L), bool))     # together they cover the square
    assert np.array_equal(inv & ca, np.eye(L, dtype=bool))     # and meet on the diagonal


def test_bi_causal_is_an_aligned_band():
    # square: the band of width 1 is the diagonal; with L_k - L_q = 5 every row keeps 6 keys
    assert np.array_equal(_one_range(W.RANGE_BI_CAUSAL, 0, 20, 0, 20), np.eye(20, dtype=bool))
    m = _one_range(W.RANGE_BI_CAUSAL, 3, 13, 2, 17, L=20)
    rows = m.sum(1)
    assert list(rows[3:13]) == [6] * 10 and rows[:3].sum() == 0 and rows[13:].sum() == 0
    for i in range(3, 13):
        keys = np.nonzero(m[i])[0]
        # top-left aligned lower edge, bottom-right aligned upper edge
        assert keys[0] == 2 + (i - 3) and keys[-1] == 16 - (12 - i)
    # BI = INV_CAUSAL and the bottom-right aligned causal triangle (equal to CAUSAL here: k_end = q_end)
    inv = _one_range(W.RANGE_INV_CAUSAL, 4, 15, 1, 15, L=15)
    ca = _one_range(W.RANGE_CAUSAL, 4, 15, 1, 15, L=15)
    assert np.array_equal(_one_range(W.RANGE_BI_CAUSAL, 4, 15, 1, 15, L=15), inv & ca)
    # a band is not prefix + chunk-local attention (the page's point)
    cc = OM.dense_mask(_ranges_spec([[(0, 20, 0, 20, W.RANGE_CHUNK_CAUSAL, 2)]]), 0, 20, 20)
    assert not np.array_equal(_one_range(W.RANGE_BI_CAUSAL, 0, 20, 0, 20), cc)


# ---- BLOCK_SPARSE ("Custom mask slows down attention.": the sparse API ≡ a custom mask) ----

def test_block_sparse_equals_custom_mask_of_its_blocks():
    rng = np.random.default_rng(12)
    lq, lk = np.array([200, 77, 300]), np.array([260, 77, 129])
    spec = W.random_mask_spec(rng, "BLOCK_SPARSE", lq, lk)
    bq, bk = spec.block_q, spec.block_k
    for b in range(3):
        m = OM.dense_mask(spec, b, int(lq[b]), int(lk[b]))
        # expand the listed blocks by hand (a separate statement of the same definition)
        exp = np.zeros_like(m)
        nbr = -(-int(lq[b]) // bq)
        for R in range(nbr):
            r = int(spec.bsr_seq_row0[b]) + R
            for c in spec.bsr_col_idx[spec.bsr_row_ptr[r]:spec.bsr_row_ptr[r + 1]]:
                exp[R * bq:(R + 1) * bq, c * bk:(c + 1) * bk] = True
        assert np.array_equal(m, exp)
        bits = W.pack_rows(m).reshape(-1)
        cu = W.MaskSpec("CUSTOM", bits=bits, word_offsets=np.array([0, bits.size], np.int64))
        assert np.array_equal(OM.dense_mask(cu, 0, int(lq[b]), int(lk[b])), m)


def test_block_sparse_all_blocks_is_full_and_none_is_empty():
    lq, lk, bq, bk = 130, 300, 64, 128
    nbr, nbc = 3, 3
    full = W.MaskSpec("BLOCK_SPARSE", block_q=bq, block_k=bk,
                      bsr_row_ptr=np.arange(0, nbc * nbr + 1, nbc, dtype=np.int32),
                      bsr_col_idx=np.tile(np.arange(nbc, dtype=np.int32), nbr), bsr_seq_row0=np.array([0]))
    assert OM.dense_mask(full, 0, lq, lk).all()
    none = W.MaskSpec("BLOCK_SPARSE", block_q=bq, block_k=bk, bsr_row_ptr=np.zeros(nbr + 1, np.int32),
                      bsr_col_idx=np.zeros(0, np.int32), bsr_seq_row0=np.array([0]))
    assert not OM.dense_mask(none, 0, lq, lk).any()
