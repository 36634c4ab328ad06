"""The planner's device workspace checked against the oracle, bit for bit, on the CPU.

tests/c/plan_probe.cpp builds the host planner with host-memory stand-ins for the CUDA
runtime, so attn_plan() / attn_plan_bwd() run here and their workspace (what the kernels
would read) can be inspected. For random problems of every kind:
  * every (sequence, query head, query row) is covered by exactly one forward work item
    (or, split, by ranges of one), and an item's jobs are exactly the key tiles where the
    oracle's dense mask has a visible pair for that query tile;
  * a job marked full is fully visible in the oracle's mask, a job marked empty for one of
    the item's two tiles is fully hidden there, and every partial-tile mask (2 KiB, row r's
    128 bits at byte 16 r) equals the oracle's mask bits on the valid rows and keys and is
    zero elsewhere;
  * the backward lists (dQ items by query tile, dK/dV items by key tile) satisfy the same,
    with the key-major tiles the exact transposes of the query-major ones.
CUSTOM masks go through host versions of the two scan kernels written from their contracts
(tests/c/plan_probe.cpp), so their host-side planning is covered as well.
"""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

import workloads as W
from oracle import masks as OM

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "masked_flash_attention_attn_b200", "csrc")
FULL, NONE = -1, -2
KINDS = ["FULL", "CAUSAL", "SLIDING_WINDOW", "PREFIX_LM", "CHUNK_CAUSAL", "RANGES", "BLOCK_SPARSE", "CUSTOM"]


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    if shutil.which("g++") is None or not os.path.exists("/usr/local/cuda/include/cuda_runtime.h"):
        pytest.skip("needs g++ and the CUDA headers")
    so = str(tmp_path_factory.mktemp("probe") / "plan_probe.so")
    cmd = ["g++", "-O1", "-std=c++17", "-fPIC", "-shared", "-I/usr/local/cuda/include",
           "-I", os.path.join(ROOT, "include"), "-I", CSRC, os.path.join(ROOT, "tests", "c", "plan_probe.cpp"),
           "-o", so, "-Wl,-Bsymbolic"]   # bind the stand-ins locally even if a CUDA runtime is loaded
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    lib = ctypes.CDLL(so)
    vp = ctypes.c_void_p
    lib.attn_plan.argtypes = [vp, vp, vp, vp]
    lib.attn_plan_bwd.argtypes = [vp, vp, vp, vp]
    lib.attn_plan_destroy.argtypes = [vp]
    lib.probe_forward.argtypes = [vp] + [ctypes.POINTER(vp)] * 3 + [ctypes.POINTER(ctypes.c_int64)] * 2 + \
        [ctypes.POINTER(ctypes.c_int32)] * 3
    lib.probe_backward.argtypes = [vp] + [ctypes.POINTER(vp)] * 6 + [ctypes.POINTER(ctypes.c_int64)] * 2
    lib.probe_host_plan.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_int)] + [ctypes.POINTER(vp)] * 3 + \
        [ctypes.POINTER(ctypes.c_int64)] * 3
    lib.probe_host_plan.restype = vp
    lib.probe_host_plan_free.argtypes = [vp]
    lib.probe_merge.argtypes = [vp, ctypes.POINTER(vp), ctypes.POINTER(ctypes.c_int64)]
    lib.probe_fail_malloc_after.argtypes = [ctypes.c_int]
    lib.probe_live_allocations.restype = ctypes.c_int
    lib.probe_set_device.argtypes = [ctypes.c_int]
    lib.attn_masked_fwd.argtypes = [vp] * 7
    return lib


def _plan(probe, M, wl, spec, kv_splits=1, backward=False):
    m = M._Marshal()
    kw = dict(hq=wl.hq, hkv=wl.hkv, head_dim=wl.d, cu_seqlens_q=wl.cu_seqlens_q, kv_splits=kv_splits)
    if wl.paged:
        kw.update(kv_lens=wl.kv_lens, page_table=wl.page_table, page_size=wl.page_size,
                  num_pages=wl.k_cache.shape[0])
    else:
        kw.update(cu_seqlens_k=wl.cu_seqlens_k)
    pr = M._problem(m, **kw)
    bits = None
    if spec.kind == "CUSTOM":   # "device" words: host memory under the probe's stand-ins
        import torch
        bits = torch.from_numpy(np.ascontiguousarray(spec.bits.astype(np.uint32).view(np.int32)))
    d = M._mask_desc(m, spec, bits)
    h = ctypes.c_void_p()
    fn = probe.attn_plan_bwd if backward else probe.attn_plan
    st = fn(ctypes.addressof(pr), ctypes.addressof(d), None, ctypes.addressof(h))
    assert st == 0, M.STATUS.get(st, st)
    h.keep = bits
    return h


def _array(addr, n, cols):
    if n == 0:
        return np.zeros((0, cols), np.int32)
    return np.ctypeslib.as_array((ctypes.c_int32 * (n * cols)).from_address(addr)).reshape(n, cols).copy()


def _tile_bits(addr, n):
    """[n][128][4] words -> bool [n][128 rows][128 keys] (bit c of row r = key c)."""
    if n == 0:
        return np.zeros((0, 128, 128), bool)
    words = np.ctypeslib.as_array((ctypes.c_uint32 * (n * 512)).from_address(addr)).reshape(n, 128, 4).copy()
    by = words.astype("<u4").view(np.uint8).reshape(n, 128, 16)
    return np.unpackbits(by, axis=-1, bitorder="little").astype(bool)


def _dense(wl, spec):
    return [OM.dense_mask(spec, b, wl.lq(b), wl.lk(b)) for b in range(wl.batch)]


def _key_start(wl, b):
    return 0 if wl.paged else int(wl.cu_seqlens_k[b])


def _check_block(dense, r0, nrows, k0, lk, mask, what):
    """One (query rows, key tile) block of a job against the oracle's mask: an empty job
    sees nothing there, a full one everything. Returns whether the block has a visible pair."""
    blk = dense[r0:r0 + nrows, k0:min(lk, k0 + 128)]
    if mask == NONE:
        assert not blk.any(), what
    elif mask == FULL:
        assert blk.all() and k0 + 128 <= lk, what
    return bool(blk.any())


def _check_merge(items, merge, nq):
    """Split-KV bookkeeping: every partial slot is written by exactly one key range, and the
    merge list names, for each split query tile, exactly the slots of its ranges."""
    slots = {}
    for it in items:
        if it[13] < 0:
            continue
        for t in range(nq):
            if it[6 + t] > 0:
                slot = int(it[13]) + t
                assert slot not in slots, "a partial slot written twice"
                slots[slot] = (int(it[4 + t]), int(it[8 + t]), int(it[6 + t]))
    listed = set()
    for tok, head, rows, slot0, nsplit, stride, _, _ in merge:
        assert nsplit >= 2
        mine = {int(slot0) + c * int(stride) for c in range(nsplit)}
        assert all(slots.get(x) == (tok, head, rows) for x in mine), "merge tile and its ranges disagree"
        assert not (mine & listed)
        listed |= mine
    assert listed == set(slots), "every partial slot is merged once"


def _forward_check(probe, M, wl, spec, kv_splits):
    h = _plan(probe, M, wl, spec, kv_splits=kv_splits)
    try:
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
        pi, pj, pt, ni, nt, R, hp, nq = vp(), vp(), vp(), i64(), i64(), i32(), i32(), i32()
        assert probe.probe_forward(h, ctypes.byref(pi), ctypes.byref(pj), ctypes.byref(pt), ctypes.byref(ni),
                                   ctypes.byref(nt), ctypes.byref(R), ctypes.byref(hp), ctypes.byref(nq)) == 0
        items = _array(pi.value, ni.value, 16)
        n_jobs = int((items[:, 10] + items[:, 11]).max()) if len(items) else 0
        jobs = _array(pj.value, n_jobs, 4)
        tiles = _tile_bits(pt.value, nt.value)
        pm, nm = vp(), i64()
        assert probe.probe_merge(h, ctypes.byref(pm), ctypes.byref(nm)) == 0
        merge = _array(pm.value, nm.value, 8)
    finally:
        probe.attn_plan_destroy(h)
    R, hp, nq = R.value, hp.value, nq.value
    _check_merge(items, merge, nq)
    dense = _dense(wl, spec)
    cq = wl.cu_seqlens_q
    covered = np.zeros((int(cq[-1]), wl.hq), np.int32)
    # (seq, head, first row) -> key tiles with a visible pair, gathered over split ranges
    seen = {}
    used_tiles = np.zeros(len(tiles), bool)
    g = wl.hq // wl.hkv
    vt0 = np.concatenate([[0], np.cumsum([-(-wl.lk(b) // 128) * 128 for b in range(wl.batch)])])
    for it in items:
        seq, tok, rows, head = it[0], it[4:6], it[6:8], it[8:10]
        js = jobs[it[10]:it[10] + it[11]]
        lq, lk = wl.lq(seq), wl.lk(seq)
        # the fields the kernels address K / V with
        assert it[3] == lk and all(head[t] // g == it[1] for t in range(nq) if rows[t] > 0)
        if wl.paged:
            assert it[2] == seq * wl.page_table.shape[1] and it[12] == -(-lk // wl.page_size) and it[14] == 0
        else:
            assert it[2] == wl.cu_seqlens_k[seq] and it[12] == 0 and it[14] == vt0[seq]
        for t in range(nq):
            if rows[t] == 0:
                continue
            r0 = int(tok[t] - cq[seq])
            key = (seq, int(head[t]), r0)
            split = it[13] >= 0      # one key range of a split query tile
            if not split or key not in seen:
                for hh in range(hp):
                    covered[tok[t]:tok[t] + rows[t], head[t] + hh] += 1
            vis = seen.setdefault(key, set())
            for j in js:
                kt, mk = int(j[0]), int(j[1 + t])
                any_vis = _check_block(dense[seq], r0, rows[t], kt * 128, lk, mk, (spec.kind, key, kt))
                if any_vis:
                    assert mk != NONE
                    assert kt not in vis, (spec.kind, key, kt)   # in one key range only
                    vis.add(kt)
                if mk >= 0:
                    used_tiles[mk] = True
                    exp = np.zeros((128, 128), bool)
                    blk = dense[seq][r0:r0 + rows[t], kt * 128:min(lk, kt * 128 + 128)]
                    for hh in range(hp):
                        exp[hh * R:hh * R + rows[t], :blk.shape[1]] = blk
                    assert np.array_equal(tiles[mk], exp), (spec.kind, key, kt)
    assert (covered == 1).all(), spec.kind
    for (seq, head, r0), vis in seen.items():
        rows = min(R, wl.lq(seq) - r0)
        lk = wl.lk(seq)
        need = {kt for kt in range(-(-lk // 128)) if dense[seq][r0:r0 + rows, kt * 128:kt * 128 + 128].any()}
        assert vis == need, (spec.kind, seq, head, r0)
    assert used_tiles.all()
    return len(merge)


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("seed", range(3))
def test_forward_workspace_matches_oracle(attn_lib, probe, kind, seed):
    wl = W.random_small(seed=300 + seed, kind=kind, batch=3, hq=8, hkv=2, d=128, lmin=1, lmax=600,
                        equal_qk=(seed == 0))
    _forward_check(probe, attn_lib, wl, wl.masks[0], kv_splits=1)


@pytest.mark.parametrize("kind", ["CAUSAL", "PREFIX_LM", "RANGES", "BLOCK_SPARSE", "CUSTOM"])
def test_forward_workspace_short_queries_packed_heads(attn_lib, probe, kind):
    """Queries of at most 60 rows: several heads share one 128-row tile."""
    wl = W.random_small(seed=41, kind=kind, batch=4, hq=8, hkv=1, d=64, lmin=1, lmax=60)
    _forward_check(probe, attn_lib, wl, wl.masks[0], kv_splits=1)


@pytest.mark.parametrize("kind", ["CAUSAL", "SLIDING_WINDOW", "RANGES", "CUSTOM"])
def test_forward_workspace_split_and_paged(attn_lib, probe, kind):
    """Forced split-KV ranges still cover every visible key tile once; paged lengths."""
    wl = W.random_small(seed=57, kind=kind, batch=3, hq=4, hkv=2, d=128, lmin=200, lmax=900)
    assert _forward_check(probe, attn_lib, wl, wl.masks[0], kv_splits=3) > 0
    wp = W.random_small(seed=58, kind=kind, batch=3, hq=4, hkv=2, d=128, lmin=1, lmax=500, paged=True)
    _forward_check(probe, attn_lib, wp, wp.masks[0], kv_splits=1)


@pytest.mark.parametrize("kind", KINDS)
def test_backward_workspace_matches_oracle(attn_lib, probe, kind):
    wl = W.random_small(seed=77 + len(kind), kind=kind, batch=3, hq=4, hkv=2, d=64, lmin=1, lmax=500)
    spec = wl.masks[0]
    h = _plan(probe, attn_lib, wl, spec, backward=True)
    try:
        vp, i64 = ctypes.c_void_p, ctypes.c_int64
        a = [vp() for _ in range(6)]
        nqi, nki = i64(), i64()
        assert probe.probe_backward(h, *[ctypes.byref(x) for x in a], ctypes.byref(nqi), ctypes.byref(nki)) == 0
        qi = _array(a[0].value, nqi.value, 8)
        ki = _array(a[2].value, nki.value, 8)
        qj = _array(a[1].value, int((qi[:, 5] + qi[:, 6]).max()) if len(qi) else 0, 4)
        kj = _array(a[3].value, int((ki[:, 5] + ki[:, 6]).max()) if len(ki) else 0, 4)
        n_tiles = int(max([m for m in list(qj[:, 1]) + list(kj[:, 1])] + [-1])) + 1
        tq = _tile_bits(a[4].value, n_tiles)
        tk = _tile_bits(a[5].value, n_tiles)
    finally:
        probe.attn_plan_destroy(h)
    dense = _dense(wl, spec)
    cq = wl.cu_seqlens_q
    assert all(np.array_equal(tk[i], tq[i].T) for i in range(n_tiles)), "key-major tiles are the transposes"
    # dQ: one item per (query head, query tile); jobs = key tiles with a visible pair
    seen_q = set()
    for it in qi:
        seq, head, tok, rows = int(it[0]), int(it[2]), int(it[3]), int(it[4])
        r0, lk = tok - int(cq[seq]), wl.lk(seq)
        seen_q.add((seq, head, r0))
        kts = set()
        for j in qj[it[5]:it[5] + it[6]]:
            if j[1] == NONE:
                continue
            kt = (int(j[0]) - _key_start(wl, seq)) // 128
            kts.add(kt)
            _check_block(dense[seq], r0, rows, kt * 128, lk, int(j[1]), (kind, "dq", seq, head, r0, kt))
            if j[1] == FULL:
                assert rows == 128
            else:
                exp = np.zeros((128, 128), bool)
                blk = dense[seq][r0:r0 + rows, kt * 128:min(lk, kt * 128 + 128)]
                exp[:rows, :blk.shape[1]] = blk
                assert np.array_equal(tq[j[1]], exp), (kind, "dq tile", seq, r0, kt)
        need = {kt for kt in range(-(-lk // 128)) if dense[seq][r0:r0 + rows, kt * 128:kt * 128 + 128].any()}
        assert kts == need, (kind, "dq", seq, head, r0)
    assert seen_q == {(b, h, r0) for b in range(wl.batch) for h in range(wl.hq) for r0 in range(0, wl.lq(b), 128)}
    # dK/dV: one item per (KV head, key tile); jobs = (query head of the group, query tile)
    g = wl.hq // wl.hkv
    seen_k = set()
    for it in ki:
        seq, kvh, tok, krows = int(it[0]), int(it[1]), int(it[3]), int(it[4])
        k0 = tok - _key_start(wl, seq)
        seen_k.add((seq, kvh, k0))
        pairs = set()
        for j in kj[it[5]:it[5] + it[6]]:
            if j[1] == NONE:
                continue
            q0, head, rows = int(j[0]) - int(cq[seq]), int(j[2]), int(j[3])
            assert kvh * g <= head < (kvh + 1) * g
            pairs.add((head, q0))
            blk = dense[seq][q0:q0 + rows, k0:k0 + krows]
            if j[1] == FULL:
                assert blk.all() and rows == 128 and krows == 128
            else:
                exp = np.zeros((128, 128), bool)
                exp[:rows, :krows] = blk
                assert np.array_equal(tq[j[1]], exp), (kind, "dkv tile", seq, q0, k0)
        need = {(h, q0) for h in range(kvh * g, (kvh + 1) * g) for q0 in range(0, wl.lq(seq), 128)
                if dense[seq][q0:q0 + 128, k0:k0 + krows].any()}
        assert pairs == need, (kind, "dkv", seq, kvh, k0)
    assert seen_k == {(b, kh, k0) for b in range(wl.batch) for kh in range(wl.hkv) for k0 in range(0, wl.lk(b), 128)}


@pytest.mark.parametrize("kind", ["CAUSAL", "SLIDING_WINDOW", "CHUNK_CAUSAL", "RANGES", "BLOCK_SPARSE"])
def test_allocation_free_host_plan_equals_the_plan_workspace(attn_lib, probe, kind):
    """attn_masked_fwd_noalloc copies a host plan into its fixed array; that plan's items,
    jobs and mask tiles equal those attn_plan (never splitting) uploads."""
    M = attn_lib
    wl = W.random_small(seed=90 + len(kind), kind=kind, batch=3, hq=8, hkv=2, d=128, lmin=1, lmax=700)
    spec = wl.masks[0]
    h = _plan(probe, M, wl, spec, kv_splits=1)
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    try:
        pi, pj, pt, ni, nt, R, hp, nq = vp(), vp(), vp(), i64(), i64(), i32(), i32(), i32()
        assert probe.probe_forward(h, ctypes.byref(pi), ctypes.byref(pj), ctypes.byref(pt), ctypes.byref(ni),
                                   ctypes.byref(nt), ctypes.byref(R), ctypes.byref(hp), ctypes.byref(nq)) == 0
        items = _array(pi.value, ni.value, 16)
        n_jobs = int((items[:, 10] + items[:, 11]).max())
        jobs = _array(pj.value, n_jobs, 4)
        tiles = _tile_bits(pt.value, nt.value)
    finally:
        probe.attn_plan_destroy(h)
    m = M._Marshal()
    pr = M._problem(m, hq=wl.hq, hkv=wl.hkv, head_dim=wl.d, cu_seqlens_q=wl.cu_seqlens_q,
                    cu_seqlens_k=wl.cu_seqlens_k)
    d = M._mask_desc(m, spec)
    st = ctypes.c_int()
    hi, hj, ht, hni, hnt, nbytes = vp(), vp(), vp(), i64(), i64(), i64()
    hplan = probe.probe_host_plan(ctypes.addressof(pr), ctypes.addressof(d), ctypes.byref(st), ctypes.byref(hi),
                                  ctypes.byref(hj), ctypes.byref(ht), ctypes.byref(hni), ctypes.byref(hnt),
                                  ctypes.byref(nbytes))
    assert st.value == 0 and hplan
    try:
        h_items = _array(hi.value, hni.value, 16)
        h_jobs = _array(hj.value, n_jobs, 4)
        h_tiles = _tile_bits(ht.value, hnt.value)
    finally:
        probe.probe_host_plan_free(hplan)
    assert np.array_equal(h_items, items) and np.array_equal(h_jobs, jobs) and np.array_equal(h_tiles, tiles)
    assert nbytes.value <= M.NOALLOC_SCRATCH_BYTES


@pytest.mark.parametrize("kind", ["CAUSAL", "CUSTOM"])
def test_failed_device_allocations_are_reported_and_cleaned_up(attn_lib, probe, kind):
    """Every device allocation of a backward plan failing in turn: attn_plan_bwd reports
    ATTN_ERR_OOM, returns no plan and frees every device allocation it had made (counted by
    the probe; a double free would abort this process); afterwards planning works again."""
    M = attn_lib
    wl = W.random_small(seed=5, kind=kind, batch=2, hq=4, hkv=2, d=64, lmin=100, lmax=400)
    spec = wl.masks[0]
    m = M._Marshal()
    pr = M._problem(m, hq=wl.hq, hkv=wl.hkv, head_dim=wl.d, cu_seqlens_q=wl.cu_seqlens_q,
                    cu_seqlens_k=wl.cu_seqlens_k)
    bits = None
    if kind == "CUSTOM":
        import torch
        bits = torch.from_numpy(np.ascontiguousarray(spec.bits.astype(np.uint32).view(np.int32)))
    d = M._mask_desc(m, spec, bits)
    live = probe.probe_live_allocations()
    try:
        for n in range(12):
            probe.probe_fail_malloc_after(n)
            h = ctypes.c_void_p()
            st = probe.attn_plan_bwd(ctypes.addressof(pr), ctypes.addressof(d), None, ctypes.addressof(h))
            if st == 0:
                probe.attn_plan_destroy(h)
                assert probe.probe_live_allocations() == live
                break
            assert st == 4 and not h.value, (n, st)   # ATTN_ERR_OOM
            assert probe.probe_live_allocations() == live, f"allocation {n} failed: device memory leaked"
        else:
            pytest.fail("a backward plan needs more than 11 allocations")
        assert n >= 2   # forward workspace and backward workspace at least
    finally:
        probe.probe_fail_malloc_after(-1)


@pytest.mark.parametrize("kind", KINDS)
def test_plan_tile_classes_and_stats_match_the_oracle(attn_lib, probe, kind):
    """attn_plan_get_tile_classes / attn_plan_get_stats of a plan built by attn_plan (CUSTOM
    through the scan's host versions) against the oracle's classes and pair count."""
    M = attn_lib
    wl = W.random_small(seed=120 + len(kind), kind=kind, batch=3, hq=4, hkv=2, d=128, lmin=1, lmax=700)
    spec = wl.masks[0]
    h = _plan(probe, M, wl, spec)
    try:
        n = ctypes.c_size_t()
        probe.attn_plan_get_tile_classes.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                                     ctypes.c_void_p]
        assert probe.attn_plan_get_tile_classes(h, None, 0, ctypes.addressof(n)) == 0
        cls = np.zeros(n.value, np.uint8)
        assert probe.attn_plan_get_tile_classes(h, cls.ctypes.data, n.value, None) == 0
        st = M.attn_plan_stats_t()
        probe.attn_plan_get_stats.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
        assert probe.attn_plan_get_stats(h, ctypes.addressof(st)) == 0
    finally:
        probe.attn_plan_destroy(h)
    lengths = [(wl.lq(b), wl.lk(b)) for b in range(wl.batch)]
    ref = OM.tile_classes(spec, lengths)
    assert np.array_equal(cls, ref)
    assert st.unmasked_pairs == OM.unmasked_pairs(spec, lengths)
    assert (st.tiles_empty, st.tiles_full, st.tiles_partial) == tuple(int((ref == c).sum()) for c in (0, 1, 2))


def test_calls_on_another_device_than_the_plans_are_refused(attn_lib, probe):
    """A plan's workspace lives on the device it was made on: attn_masked_fwd with another
    current device returns INVALID_ARG before any launch (the probe's launcher stub answers
    UNSUPPORTED when the call gets that far)."""
    wl = W.random_small(seed=4, kind="CAUSAL", batch=2, hq=2, hkv=1, d=128, lmin=10, lmax=100)
    h = _plan(probe, attn_lib, wl, wl.masks[0])
    try:
        fake = [4096, 8192, 12288, 16384, 20480]   # aligned addresses, never dereferenced here
        assert probe.attn_masked_fwd(h, *fake, None) == 2
        probe.probe_set_device(1)
        assert probe.attn_masked_fwd(h, *fake, None) == 1
    finally:
        probe.probe_set_device(0)
        probe.attn_plan_destroy(h)
