"""CPU tests of the C ABI: exported symbols, host planner classification, validation.

The host planner's 128 x 128 tile classes must equal, bit for bit, the classes the
oracle derives from its dense boolean masks; its pair counts must equal the oracle's.
No call here touches a GPU (attn_classify_host makes no CUDA call).
"""
import os
import re
import subprocess

import numpy as np
import pytest

import workloads as W
from oracle import masks as OM

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = "".join(open(os.path.join(ROOT, "include", f)).read() for f in sorted(os.listdir(os.path.join(ROOT, "include"))))
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:attn_status_t|const char\*)\s+(attn_\w+)\s*\(", src, flags=re.M)))


def test_library_exports_every_declared_symbol(attn_lib):
    names = _declared_functions()
    assert len(names) >= 9
    lib = attn_lib.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(attn_lib.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", attn_lib._LIB_PATH], capture_output=True, text=True).stdout
    for n in names:
        assert re.search(rf"\bT {n}$", out, flags=re.M), n


def test_status_strings(attn_lib):
    for code in range(7):
        assert attn_lib.attn_status_string(code)


def _classify(M, wl, spec):
    kw = dict(hq=wl.hq, hkv=wl.hkv, head_dim=wl.d, cu_seqlens_q=wl.cu_seqlens_q, mask=spec)
    if wl.paged:
        kw.update(kv_lens=wl.kv_lens, page_size=wl.page_size, max_pages_per_seq=wl.page_table.shape[1],
                  num_pages=wl.k_cache.shape[0])
    else:
        kw.update(cu_seqlens_k=wl.cu_seqlens_k)
    return M.attn_classify_host(**kw)


def _lengths(wl):
    return [(wl.lq(b), wl.lk(b)) for b in range(wl.batch)]


@pytest.mark.parametrize("kind", ["FULL", "CAUSAL", "SLIDING_WINDOW", "PREFIX_LM", "CHUNK_CAUSAL", "RANGES", "BLOCK_SPARSE"])
@pytest.mark.parametrize("seed", range(6))
def test_host_classes_match_oracle_random(attn_lib, kind, seed):
    wl = W.random_small(seed=100 * seed + 7, kind=kind, batch=4, lmin=1, lmax=700, equal_qk=(seed % 2 == 0))
    cls, pairs = _classify(attn_lib, wl, wl.masks[0])
    ref = OM.tile_classes(wl.masks[0], _lengths(wl))
    assert np.array_equal(cls, ref)
    assert pairs == OM.unmasked_pairs(wl.masks[0], _lengths(wl))


def test_host_classes_paged_lengths(attn_lib):
    wl = W.random_small(seed=3, kind="SLIDING_WINDOW", batch=5, lmin=1, lmax=500, paged=True)
    cls, _ = _classify(attn_lib, wl, wl.masks[0])
    assert np.array_equal(cls, OM.tile_classes(wl.masks[0], _lengths(wl)))


def test_host_classes_workload_prefix_lm(attn_lib):
    wl = W.prefix_lm_small()
    cls, pairs = _classify(attn_lib, wl, wl.masks[0])
    assert list(cls) == [2, 0, 1, 2] and pairs == 34912


def test_host_classes_workload_gemma2(attn_lib):
    wl = W.gemma2_local_global()
    for spec in wl.masks:
        cls, pairs = _classify(attn_lib, wl, spec)
        assert np.array_equal(cls, OM.tile_classes(spec, _lengths(wl)))
        assert pairs == OM.unmasked_pairs(spec, _lengths(wl))


def test_host_classes_workload_chunk_causal_both_forms(attn_lib):
    L, p = 8192, 4096
    cq = W.cu_from_lengths([L] * 2)
    specs = [W.MaskSpec("CHUNK_CAUSAL", chunk=(p, L, 0, L, W.RANGE_CHUNK_CAUSAL, 2)),
             W.MaskSpec("RANGES", ranges=W.chunk_causal_ranges(2, L, p, 2))]
    res = []
    for spec in specs:
        cls, pairs = attn_lib.attn_classify_host(hq=16, hkv=16, head_dim=128, cu_seqlens_q=cq, cu_seqlens_k=cq,
                                                 mask=spec)
        assert pairs == 2 * 33560576
        n = np.bincount(cls, minlength=3)
        assert tuple(n) == (2 * 2016, 2 * 2016, 2 * 64)
        res.append(cls)
    assert np.array_equal(res[0], res[1])
    assert np.array_equal(res[0], OM.tile_classes(specs[0], [(L, L)] * 2))


def test_host_classes_workload_block_dense_ranges(attn_lib):
    L, dense, blk = 29576, 24576, 100
    ranges = [(0, dense, 0, dense, W.RANGE_FULL, 0)]
    for s in range(dense, L, blk):
        e = min(s + blk, L)
        ranges += [(s, e, 0, dense, W.RANGE_FULL, 0), (s, e, s, e, W.RANGE_CAUSAL, 0)]
    spec = W.MaskSpec("RANGES", ranges=[ranges])
    cq = W.cu_from_lengths([L])
    cls, pairs = attn_lib.attn_classify_host(hq=32, hkv=8, head_dim=128, cu_seqlens_q=cq, cu_seqlens_k=cq, mask=spec)
    assert tuple(np.bincount(cls, minlength=3)) == (9202, 44544, 78)
    assert pairs == 727112276
    assert np.array_equal(cls, OM.tile_classes(spec, [(L, L)]))


def _err(M, **kw):
    with pytest.raises(M.AttnError) as e:
        M.attn_classify_host(**kw)
    return e.value.status


def test_validation_errors(attn_lib):
    M = attn_lib
    cq = np.array([0, 10, 30], np.int32)
    base = dict(hq=4, hkv=2, head_dim=128, cu_seqlens_q=cq, cu_seqlens_k=cq)
    ok = M.attn_classify_host(mask=W.MaskSpec("CAUSAL"), **base)
    assert len(ok[0]) == 2
    assert _err(M, mask=W.MaskSpec("CAUSAL"), **{**base, "hkv": 3}) == 1           # hq % hkv
    assert _err(M, mask=W.MaskSpec("CAUSAL"), **{**base, "head_dim": 96}) == 2     # unsupported d
    assert _err(M, mask=W.MaskSpec("SLIDING_WINDOW", window=0), **base) == 1
    assert _err(M, mask=W.MaskSpec("PREFIX_LM", prefix_len=-1), **base) == 1
    assert _err(M, mask=W.MaskSpec("CHUNK_CAUSAL", chunk=(2, 10, 0, 10, W.RANGE_CHUNK_CAUSAL, 0)), **base) == 1
    bad = [[(0, 11, 0, 5, 0, 0)], []]                                              # q_end > L_q
    assert _err(M, mask=W.MaskSpec("RANGES", ranges=bad), **base) == 1
    bad = [[(0, 5, 3, 2, 0, 0)], []]                                               # k_end < k_start
    assert _err(M, mask=W.MaskSpec("RANGES", ranges=bad), **base) == 1
    bad = [[(0, 5, 0, 2, 7, 0)], []]                                               # unknown type
    assert _err(M, mask=W.MaskSpec("RANGES", ranges=bad), **base) == 1
    assert _err(M, mask=W.MaskSpec("CAUSAL"), **{**base, "cu_seqlens_q": np.array([0, 10, 5], np.int32)}) == 1
    # CUSTOM cannot be classified on the host (its bits live on the device)
    assert _err(M, mask=W.MaskSpec("CUSTOM", bits=np.zeros(4, np.uint32), word_offsets=np.array([0, 1, 2])),
                **base) in (2, 3)
    # paged: unsupported page size, and more keys than the page row holds
    assert _err(M, mask=W.MaskSpec("CAUSAL"), hq=4, hkv=2, head_dim=64, cu_seqlens_q=cq,
                kv_lens=np.array([10, 20], np.int32), page_size=8, max_pages_per_seq=4, num_pages=8) == 2
    assert _err(M, mask=W.MaskSpec("CAUSAL"), hq=4, hkv=2, head_dim=64, cu_seqlens_q=cq,
                kv_lens=np.array([10, 80], np.int32), page_size=16, max_pages_per_seq=4, num_pages=8) == 1


def test_empty_and_degenerate_lengths(attn_lib):
    M = attn_lib
    cq = np.array([0, 0, 5, 5], np.int32)
    ck = np.array([0, 3, 3, 9], np.int32)
    cls, pairs = M.attn_classify_host(hq=2, hkv=1, head_dim=64, cu_seqlens_q=cq, cu_seqlens_k=ck,
                                      mask=W.MaskSpec("CAUSAL"))
    # seq 0: no rows; seq 1: 5 rows x 0 keys (no tiles); seq 2: 0 rows
    assert len(cls) == 0 and pairs == 0
    cls, pairs = M.attn_classify_host(hq=2, hkv=1, head_dim=64, cu_seqlens_q=np.array([0], np.int32),
                                      cu_seqlens_k=np.array([0], np.int32), mask=W.MaskSpec("FULL"))
    assert len(cls) == 0


def test_dry_run_split_kv_decisions(attn_lib):
    """Split-KV planning on the host (attn_plan_dry_run): few long work items are cut into
    key ranges, the ranges cover each item's key tiles exactly once, and balanced
    workloads are left alone."""
    M = attn_lib
    lq, lk = [64] * 4, [23740, 25265, 24931, 22072]          # 4 requests x 8 KV heads = 32 items
    base = dict(hq=32, hkv=8, head_dim=128, cu_seqlens_q=W.cu_from_lengths(lq),
                cu_seqlens_k=W.cu_from_lengths(lk), mask=W.MaskSpec("CAUSAL"))
    never = M.attn_plan_dry_run(kv_splits=1, **base)
    assert never["work_items"] == 32 and never["kv_splits_max"] == 1 and never["merge_tiles"] == 0
    auto = M.attn_plan_dry_run(kv_splits=0, **base)
    assert auto["kv_splits_max"] >= 3 and auto["work_items"] >= 128
    assert auto["merge_tiles"] == 64                          # 32 items x 2 query tiles
    assert auto["jobs"] == never["jobs"] and auto["mask_tile_reads"] == never["mask_tile_reads"]
    assert auto["unmasked_pairs"] == never["unmasked_pairs"]
    for n in (2, 7):
        forced = M.attn_plan_dry_run(kv_splits=n, **base)
        assert forced["work_items"] == 32 * n and forced["kv_splits_max"] == n
        assert forced["jobs"] == never["jobs"]
    # fewer SMs than items: no split is worth it
    assert M.attn_plan_dry_run(kv_splits=0, num_sms=32, **base)["kv_splits_max"] == 1
    # the balanced benchmark workloads (analytic masks) are not split
    for c in (1, 2, 4, 5):
        wl = W.config(c)
        for spec in wl.masks:
            if spec.kind == "CUSTOM":
                continue
            st = M.attn_plan_dry_run(hq=wl.hq, hkv=wl.hkv, head_dim=wl.d, cu_seqlens_q=wl.cu_seqlens_q,
                                     cu_seqlens_k=wl.cu_seqlens_k, mask=spec)
            assert st["kv_splits_max"] == 1 and st["merge_tiles"] == 0, (c, spec.kind)
    assert _err_dry(M, kv_splits=-1, **base) == 1
    assert _err_dry(M, num_sms=0, **base) == 1


def _err_dry(M, **kw):
    with pytest.raises(M.AttnError) as e:
        M.attn_plan_dry_run(**kw)
    return e.value.status


def test_mask_tile_transposition(attn_lib):
    """The planner's tile transposition (what the dK/dV kernel reads) against a plain bit
    transpose of random, full, empty and single-bit tiles."""
    rng = np.random.default_rng(17)
    cases = [rng.integers(0, 2**32, size=512, dtype=np.uint64).astype(np.uint32),
             np.full(512, 0xFFFFFFFF, np.uint32), np.zeros(512, np.uint32)]
    one = np.zeros(512, np.uint32)
    one[4 * 5 + 2] = 1 << 7                      # row 5, key 64 + 7
    cases.append(one)
    for t in cases:
        bits = np.unpackbits(t.view(np.uint8), bitorder="little").reshape(128, 128)   # [row][key]
        want = np.packbits(bits.T.reshape(-1), bitorder="little").view(np.uint32)
        assert np.array_equal(attn_lib.attn_test_transpose_mask_tile(t), want)
