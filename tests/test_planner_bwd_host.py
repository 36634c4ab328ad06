"""Host-side pins of the backward planner through attn_plan_bwd_dry_run (no GPU): the dQ and
dK/dV work lists that attn_plan_bwd() builds have exactly the items and jobs the oracle's
dense masks imply (one dQ item per query tile and query head, running every key tile that
holds a visible pair, or one job that writes zeros; one dK/dV item per key tile and KV head,
running every (query head of the group, query tile) that sees it, or one zero job), mask
tiles for exactly the partial tiles and the full tiles cut by the end of the keys or queries,
the same lists for a paged cache as for contiguous keys, and CTA loads within the bound of
the longest-first assignment."""
import numpy as np
import pytest

import oracle
import workloads as W

KINDS = ["FULL", "CAUSAL", "SLIDING_WINDOW", "PREFIX_LM", "CHUNK_CAUSAL", "RANGES", "BLOCK_SPARSE"]
T = 128


def _expected(wl, spec):
    """Counts from the dense masks (plain definitions), per the rules in the module docstring."""
    g = wl.hq // wl.hkv
    e = dict(dq_items=0, dq_jobs=0, dkv_items=0, dkv_jobs=0, mask_tiles=0)
    for b in range(wl.batch):
        lq, lk = wl.lq(b), wl.lk(b)
        n_qt, n_kt = -(-lq // T), -(-lk // T)
        m = oracle.dense_mask(spec, b, lq, lk)
        nonempty = np.zeros((n_qt, n_kt), bool)
        for qt in range(n_qt):
            for kt in range(n_kt):
                blk = m[qt * T:(qt + 1) * T, kt * T:(kt + 1) * T]
                nonempty[qt, kt] = blk.any()
                interior = (qt + 1) * T <= lq and (kt + 1) * T <= lk
                if blk.any() and not (blk.all() and interior):
                    e["mask_tiles"] += 1
        e["dq_items"] += n_qt * wl.hq
        e["dq_jobs"] += wl.hq * int(np.maximum(nonempty.sum(axis=1), 1).sum())
        e["dkv_items"] += n_kt * wl.hkv
        col = nonempty.sum(axis=0)
        e["dkv_jobs"] += wl.hkv * int(np.where(col > 0, g * col, 1).sum())
    return e


def _kw(wl, spec, num_sms):
    kw = dict(hq=wl.hq, hkv=wl.hkv, head_dim=wl.d, cu_seqlens_q=wl.cu_seqlens_q, mask=spec, num_sms=num_sms)
    if wl.paged:
        kw.update(kv_lens=wl.kv_lens, page_size=wl.page_size, max_pages_per_seq=wl.page_table.shape[1],
                  num_pages=int(wl.k_cache.shape[0]))
    else:
        kw.update(cu_seqlens_k=wl.cu_seqlens_k)
    return kw


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("kind", KINDS)
def test_backward_lists_match_the_dense_masks(attn_lib, kind, d):
    wl = W.random_small(seed=31 + d + len(kind), kind=kind, batch=3, hq=4, hkv=2, d=d, lmin=1, lmax=700)
    spec = wl.masks[0]
    st = attn_lib.attn_plan_bwd_dry_run(**_kw(wl, spec, 148))
    exp = _expected(wl, spec)
    assert {k: st[k] for k in exp} == exp, (kind, d)
    assert st["dq_cost"] == st["dq_jobs"] + 2 * st["dq_items"]
    assert st["dkv_cost"] == st["dkv_jobs"] + 2 * st["dkv_items"]


@pytest.mark.parametrize("kind", ["CAUSAL", "SLIDING_WINDOW", "CHUNK_CAUSAL", "FULL"])
@pytest.mark.parametrize("ps", [16, 64])
def test_paged_lists_equal_contiguous_ones(attn_lib, kind, ps):
    # the same lengths and mask over a paged cache: the lists differ only in how keys are
    # addressed, not in their items, jobs, mask tiles or balance
    wl = W.random_small(seed=7 + ps, kind=kind, batch=3, hq=4, hkv=2, d=128, lmin=1, lmax=600, paged=True,
                        page_size=ps)
    spec = wl.masks[0]
    paged = attn_lib.attn_plan_bwd_dry_run(**_kw(wl, spec, 148))
    cu_k = np.concatenate([[0], np.cumsum([wl.lk(b) for b in range(wl.batch)])]).astype(np.int32)
    contig = attn_lib.attn_plan_bwd_dry_run(hq=wl.hq, hkv=wl.hkv, head_dim=wl.d, cu_seqlens_q=wl.cu_seqlens_q,
                                            cu_seqlens_k=cu_k, mask=spec, num_sms=148)
    assert paged == contig
    assert {k: paged[k] for k in _expected(wl, spec)} == _expected(wl, spec)


@pytest.mark.parametrize("num_sms", [1, 7, 148])
def test_cta_loads_within_the_longest_first_bound(attn_lib, num_sms):
    # a greedy assignment of items (longest first, to the least loaded CTA) ends with no CTA
    # above the mean load plus one item
    wl = W.random_small(seed=9, kind="CAUSAL", batch=4, hq=8, hkv=2, d=128, lmin=200, lmax=3000)
    st = attn_lib.attn_plan_bwd_dry_run(**_kw(wl, wl.masks[0], num_sms))
    for side in ("dq", "dkv"):
        ctas = st[f"{side}_ctas"]
        assert 1 <= ctas <= num_sms
        assert st[f"{side}_max_cta_cost"] <= st[f"{side}_cost"] / ctas + st[f"{side}_max_item_cost"], side
        assert st[f"{side}_max_cta_cost"] >= -(-st[f"{side}_cost"] // ctas)


def test_custom_and_bad_arguments_are_refused(attn_lib):
    M = attn_lib
    wl = W.random_small(seed=3, kind="CUSTOM", batch=2, hq=2, hkv=1, d=64, lmin=10, lmax=50)
    with pytest.raises(M.AttnError) as e:
        M.attn_plan_bwd_dry_run(**_kw(wl, wl.masks[0], 148))
    assert e.value.status == 2
    wl = W.random_small(seed=3, kind="CAUSAL", batch=2, hq=2, hkv=1, d=64, lmin=10, lmax=50)
    with pytest.raises(M.AttnError) as e:
        M.attn_plan_bwd_dry_run(**_kw(wl, wl.masks[0], 0))
    assert e.value.status == 1


def test_chunk_causal_workload_closed_form(attn_lib):
    # 8 sequences of 8192 = 64 x 128 rows, causal over [0, 4096) then chunk-causal (chunk 2)
    # over [4096, 8192): per sequence and head 2016 full + 64 partial non-empty tiles (the
    # forward's tile classes), no tile cut by a sequence end, every query tile sees a key and
    # every key tile is seen -- so both kernels run 16 x 8 x 2080 jobs and 8 x 64 tiles carry a mask
    wl = W.config(4)
    for spec in wl.masks:   # both descriptor forms
        st = attn_lib.attn_plan_bwd_dry_run(**_kw(wl, spec, 148))
        assert st["dq_items"] == st["dkv_items"] == 16 * 8 * 64
        assert st["dq_jobs"] == st["dkv_jobs"] == 16 * 8 * 2080
        assert st["mask_tiles"] == 8 * 64
