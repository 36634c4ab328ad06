"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Small problems are compared element by element on every output row (several
128-row tiles, ragged tails, every mask kind, every head dim, contiguous and
paged K/V, short-query head packing); tile classes from the GPU plan (including
the device scan of CUSTOM bits) must equal the oracle's bit for bit.
"""
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


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("kind", KINDS)
def test_small_ragged_all_kinds(kind, d):
    wl = W.random_small(seed=d + 17 * KINDS.index(kind), kind=kind, batch=3, hq=4, hkv=2, d=d,
                        lmin=1, lmax=400)
    G.check_full(wl, wl.masks[0], f"{kind} d={d}")


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("kind", ["CAUSAL", "SLIDING_WINDOW", "CUSTOM"])
def test_small_paged(kind, d):
    wl = W.random_small(seed=5 + d, kind=kind, batch=3, hq=4, hkv=2, d=d, lmin=1, lmax=300, paged=True)
    G.check_full(wl, wl.masks[0], f"paged {kind} d={d}")


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("ps", [16, 32, 64, 128])
def test_page_sizes(ps, d):
    # every page size against every head_dim: the producer issues one lane per page (one per
    # box in the 2-SM kernel), so the lane count changes with both
    wl = W.random_small(seed=ps + d, kind="CAUSAL", batch=3, hq=2, hkv=1, d=d, lmin=1, lmax=300, paged=True,
                        page_size=ps)
    G.check_full(wl, wl.masks[0], f"page size {ps} d={d}")


@pytest.mark.parametrize("g,lmax", [(2, 64), (4, 32), (8, 16), (4, 64)])
def test_short_queries_pack_heads(g, lmax):
    # decode / verify shapes: L_q <= 128 / heads_per_tile packs several query heads per tile
    rng = np.random.default_rng(g * 100 + lmax)
    lq = rng.integers(1, lmax + 1, size=5)
    lk = lq + rng.integers(0, 500, size=5)
    gen = torch.Generator().manual_seed(g)
    cq, ck = W.cu_from_lengths(lq), W.cu_from_lengths(lk)
    hkv = 2
    wl = W.Workload(name="short", hq=hkv * g, hkv=hkv, d=128, scale=0.1, cu_seqlens_q=cq,
                    q=W.randn_bf16(gen, int(cq[-1]), hkv * g, 128), masks=[W.MaskSpec("CAUSAL")],
                    cu_seqlens_k=ck, k=W.randn_bf16(gen, int(ck[-1]), hkv, 128),
                    v=W.randn_bf16(gen, int(ck[-1]), hkv, 128))
    out, lse, plan = G.run(wl, wl.masks[0])
    assert plan.stats["heads_per_tile"] > 1
    ref_o, ref_l = oracle.masked_attention(wl, wl.masks[0])
    G.compare(out, lse, ref_o, ref_l, f"g={g}")


def test_fully_masked_rows_and_empty_sequences():
    # rows outside every range see nothing: out = 0, lse = -inf; empty sequences are skipped
    cq = np.array([0, 0, 200, 201, 201, 457], np.int32)
    ck = np.array([0, 5, 205, 205, 300, 700], np.int32)   # seq 2 has L_k = 0
    ranges = [[], [(10, 50, 0, 100, W.RANGE_FULL, 0), (150, 200, 20, 200, W.RANGE_CAUSAL, 0)], [], [],
              [(0, 256, 300, 400, W.RANGE_FULL, 0)]]
    gen = torch.Generator().manual_seed(0)
    wl = W.Workload(name="edge", hq=4, hkv=2, d=128, scale=0.125, cu_seqlens_q=cq,
                    q=W.randn_bf16(gen, int(cq[-1]), 4, 128), masks=[W.MaskSpec("RANGES", ranges=ranges)],
                    cu_seqlens_k=ck, k=W.randn_bf16(gen, int(ck[-1]), 2, 128),
                    v=W.randn_bf16(gen, int(ck[-1]), 2, 128))
    G.check_full(wl, wl.masks[0], "masked rows")


def test_no_keys_at_all():
    cq = np.array([0, 3, 7], np.int32)
    ck = np.array([0, 0, 0], np.int32)
    gen = torch.Generator().manual_seed(1)
    wl = W.Workload(name="nokeys", hq=2, hkv=1, d=64, scale=0.125, cu_seqlens_q=cq,
                    q=W.randn_bf16(gen, 7, 2, 64), masks=[W.MaskSpec("FULL")], cu_seqlens_k=ck,
                    k=torch.zeros(1, 1, 64, dtype=torch.bfloat16), v=torch.zeros(1, 1, 64, dtype=torch.bfloat16))
    out, lse, _ = G.run(wl, wl.masks[0])
    assert torch.all(out == 0) and torch.all(lse == -float("inf"))


def test_canary_rows_untouched_and_outputs_deterministic():
    wl = W.random_small(seed=9, kind="CAUSAL", batch=3, hq=4, hkv=2, d=128, lmin=50, lmax=300)
    tq = int(wl.cu_seqlens_q[-1])
    out, lse, _ = G.run(wl, wl.masks[0], extra_rows=64, canary=7.0)
    assert torch.all(out[tq:] == 7.0) and torch.all(lse[tq:] == 7.0)
    out2, lse2, _ = G.run(wl, wl.masks[0])
    assert torch.equal(out[:tq], out2) and torch.equal(lse[:tq], lse2)


@pytest.mark.parametrize("poison", ["finite", "nan", "inf"])
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("kind", ["CUSTOM", "CAUSAL"])
def test_paged_poison_in_unused_slots(kind, d, poison):
    # Cache slots no sequence owns -- keys past kv_len in a sequence's last page and pages
    # no page table names -- hold whatever a serving cache left there: a large finite value,
    # NaN or Inf. The output must be bit-identical to the one with clean slots.
    wl = W.random_small(seed=21 + d, kind=kind, batch=4, hq=4, hkv=2, d=d, lmin=20, lmax=400, paged=True)
    ref = G.run(wl, wl.masks[0])
    kc, vc = wl.k_cache.clone(), wl.v_cache.clone()
    used = np.zeros((kc.shape[0], wl.page_size), bool)
    for b in range(wl.batch):
        n = wl.lk(b)
        for j in range(n):
            used[wl.page_table[b, j // wl.page_size], j % wl.page_size] = True
    mask = torch.from_numpy(~used)
    assert mask.any() and bool(mask[np.unique(wl.page_table[wl.page_table >= 0])].any()), \
        "some last page must be partly unused"
    kv = {"finite": (3.0e4, -3.0e4), "nan": (float("nan"), float("nan")), "inf": (float("inf"), -float("inf"))}
    kc[mask], vc[mask] = kv[poison]
    wl.k_cache, wl.v_cache = kc, vc
    out, lse, _ = G.run(wl, wl.masks[0])
    assert torch.equal(out, ref[0]) and torch.equal(lse, ref[1])


def test_paged_equals_contiguous():
    wl = W.random_small(seed=33, kind="SLIDING_WINDOW", batch=3, hq=4, hkv=2, d=128, lmin=30, lmax=500, paged=True)
    out_p, lse_p, _ = G.run(wl, wl.masks[0])
    ks, vs = zip(*[wl.kv_of_seq(b) for b in range(wl.batch)])
    wc = W.Workload(name="contig", hq=wl.hq, hkv=wl.hkv, d=wl.d, scale=wl.scale, cu_seqlens_q=wl.cu_seqlens_q,
                    q=wl.q, masks=wl.masks, cu_seqlens_k=W.cu_from_lengths(wl.kv_lens), k=torch.cat(ks),
                    v=torch.cat(vs))
    out_c, lse_c, _ = G.run(wc, wc.masks[0])
    assert torch.equal(out_p, out_c) and torch.equal(lse_p, lse_c)


def test_custom_mask_too_small_is_rejected():
    import masked_flash_attention_attn_b200 as M
    wl = W.random_small(seed=2, kind="CUSTOM", batch=2, lmin=40, lmax=80)
    spec = wl.masks[0]
    short = W.MaskSpec("CUSTOM", bits=spec.bits[:-1], word_offsets=spec.word_offsets.copy())
    short.word_offsets[-1] -= 1
    with pytest.raises(M.AttnError) as e:
        G.make_plan(wl, short)
    assert e.value.status == 3


def test_bounded_wait_timeout_reports_and_context_survives():
    """A forced missing arrival makes a bounded wait expire: the kernel returns through its
    abort path, the status word reports ATTN_ERR_TIMEOUT, and the next forward is correct."""
    import masked_flash_attention_attn_b200 as M
    wl = W.random_small(seed=4, kind="CAUSAL", batch=2, hq=4, hkv=2, d=128, lmin=100, lmax=300)
    q, k, v = G.device_inputs(wl)
    plan = G.make_plan(wl, wl.masks[0])
    tq = int(wl.cu_seqlens_q[-1])
    out = torch.empty(tq, wl.hq, wl.d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(tq, wl.hq, dtype=torch.float32, device="cuda")
    M.attn_plan_set_debug(plan, 1, 50_000_000)   # 50 ms per wait
    M.attn_masked_fwd(plan, q, k, v, out, lse)
    assert M.attn_plan_check_status(plan) == 6
    M.attn_plan_set_debug(plan, 0, 0)
    M.attn_masked_fwd(plan, q, k, v, out, lse)
    assert M.attn_plan_check_status(plan) == 0
    ref_o, ref_l = oracle.masked_attention(wl, wl.masks[0])
    G.compare(out.float().cpu(), lse.cpu(), ref_o, ref_l, "after timeout")


def test_exp2_polynomial_error_bound():
    """The FMA-pipe exp2 used for part of the softmax: relative error <= 7.5e-5 (the Remez fit's
    bound, plus fp32 evaluation rounding) against fp64 2^x on the range the softmax feeds it,
    tiny and exact-zero behaviour below it."""
    import masked_flash_attention_attn_b200 as M
    x = torch.cat([torch.linspace(-120.0, 8.0, 2_000_001), torch.tensor([-125.0, -1e4, -float("inf"), 0.0, 1.0])])
    xd = x.cuda()
    y = torch.empty_like(xd)
    M.attn_test_exp2_poly(xd, y)
    y = y.cpu().double()
    ref = torch.exp2(x.double())
    body = x >= -120
    rel = ((y[body] - ref[body]).abs() / ref[body]).max().item()
    assert rel <= 8e-5, rel
    assert torch.all(y[~body] <= 2.0 ** -120) and torch.all(y[~body] >= 0)
    assert y[-2].item() == pytest.approx(1.0, rel=8e-5) and y[-1].item() == pytest.approx(2.0, rel=8e-5)


@pytest.mark.parametrize("d", [128, 256])
def test_inv_and_bi_causal_ranges(d):
    """The INV_CAUSAL / BI_CAUSAL range types on non-square, overlapping ranges."""
    rng = np.random.default_rng(d)
    lq = np.array([300, 517, 129])
    lk = np.array([420, 517, 700])
    ranges = []
    for b in range(3):
        rs = []
        for t in (W.RANGE_INV_CAUSAL, W.RANGE_BI_CAUSAL, W.RANGE_BI_CAUSAL, W.RANGE_FULL):
            a, c = sorted(rng.integers(0, lq[b] + 1, size=2).tolist())
            e, f = sorted(rng.integers(0, lk[b] + 1, size=2).tolist())
            rs.append((a, c, e, f, t, 0))
        ranges.append(rs)
    gen = torch.Generator().manual_seed(d)
    cq, ck = W.cu_from_lengths(lq), W.cu_from_lengths(lk)
    wl = W.Workload(name="invbi", hq=4, hkv=2, d=d, scale=1.0 / np.sqrt(d), cu_seqlens_q=cq,
                    q=W.randn_bf16(gen, int(cq[-1]), 4, d), masks=[W.MaskSpec("RANGES", ranges=ranges)],
                    cu_seqlens_k=ck, k=W.randn_bf16(gen, int(ck[-1]), 2, d), v=W.randn_bf16(gen, int(ck[-1]), 2, d))
    G.check_full(wl, wl.masks[0], f"inv/bi d={d}")


def test_block_sparse_equals_custom_of_its_blocks():
    """The sparse (BSR) descriptor and the packed custom mask of the same blocks plan the same
    tiles and give bit-identical outputs ("Custom mask slows down attention.": equivalence)."""
    wl = W.random_small(seed=77, kind="BLOCK_SPARSE", batch=3, hq=4, hkv=2, d=128, lmin=50, lmax=500)
    spec = wl.masks[0]
    out_b, lse_b, plan_b = G.run(wl, spec)
    words, offs = [], [0]
    for b in range(wl.batch):
        m = oracle.dense_mask(spec, b, wl.lq(b), wl.lk(b))
        w = W.pack_rows(m).reshape(-1)
        words.append(w)
        offs.append(offs[-1] + w.size)
    cu = W.MaskSpec("CUSTOM", bits=np.concatenate(words).astype(np.uint32), word_offsets=np.asarray(offs, np.int64))
    out_c, lse_c, plan_c = G.run(wl, cu)
    import masked_flash_attention_attn_b200 as M
    assert np.array_equal(M.attn_plan_get_tile_classes(plan_b), M.attn_plan_get_tile_classes(plan_c))
    assert torch.equal(out_b, out_c) and torch.equal(lse_b, lse_c)
