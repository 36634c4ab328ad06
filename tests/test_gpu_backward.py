"""GPU parity of the backward pass (dQ, dK, dV) through the C ABI against the fp64 oracle
gradients (oracle/backward.py), on ragged batches of every mask kind, head dims 64, 128 and
256, contiguous K/V and paged caches (dk / dv in the cache layout; unused slots poisoned),
grouped-query heads, rows that see no key and keys no query sees; and three benchmark
workloads at full size on sampled rows and keys.

Tolerance: P and dS enter the tensor cores as bf16 (relative rounding 2^-9 each) with fp32
accumulation, and the gradients are stored as bf16 (relative rounding 2^-9, i.e. a mean
error of about 2e-3 of the mean magnitude from the storage alone); with the forward's bf16
out in delta = dout . out the expected error is a few 1e-3 of the gradient scale. Measured
over every case of this file on B200: worst max |err| / max |ref| = 7.2e-3 (dq), worst
mean |err| / mean |ref| = 3.0e-3. The bound used, per tensor: max |err| <= 1.2e-2 * max |ref|
and mean |err| <= 5e-3 * mean |ref|."""
import numpy as np
import pytest
import torch

import workloads as W
import oracle
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu

KINDS = ["FULL", "CAUSAL", "SLIDING_WINDOW", "PREFIX_LM", "CHUNK_CAUSAL", "RANGES", "CUSTOM", "BLOCK_SPARSE"]
REL_MAX, REL_MEAN = 1.2e-2, 5e-3


@pytest.fixture(scope="module", autouse=True)
def _lib(attn_lib):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return attn_lib


def _close(got, ref, what):
    got = got.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite"
    err = np.abs(got - ref)
    scale_max, scale_mean = max(np.abs(ref).max(), 1e-6), max(np.abs(ref).mean(), 1e-6)
    assert err.max() <= REL_MAX * scale_max, f"{what}: max err {err.max():.3e} vs scale {scale_max:.3e}"
    assert err.mean() <= REL_MEAN * scale_mean, f"{what}: mean err {err.mean():.3e} vs scale {scale_mean:.3e}"


def _bwd_plan(wl, spec):
    kw = dict(hq=wl.hq, hkv=wl.hkv, head_dim=wl.d, cu_seqlens_q=wl.cu_seqlens_q, mask=spec, scale=wl.scale,
              backward=True)
    if wl.paged:
        kw.update(kv_lens=wl.kv_lens, page_table=torch.from_numpy(wl.page_table).cuda(), page_size=wl.page_size,
                  num_pages=wl.k_cache.shape[0])
    else:
        kw.update(cu_seqlens_k=wl.cu_seqlens_k)
    return G.M.attn_plan(**kw)


def check_backward(wl, spec, what, seed=0, with_dlse=False, inputs=None):
    q, k, v = inputs if inputs is not None else G.device_inputs(wl)
    plan = _bwd_plan(wl, spec)
    out, lse = G.M.forward(plan, q, k, v)
    gen = torch.Generator().manual_seed(1000 + seed)
    dout_h = W.randn_bf16(gen, q.shape[0], wl.hq, wl.d)
    dlse_h = torch.randn(q.shape[0], wl.hq, generator=gen) if with_dlse else None
    dq, dk, dv = G.M.backward(plan, q, k, v, out, lse, dout_h.cuda(),
                              dlse=None if dlse_h is None else dlse_h.cuda())
    assert G.M.attn_plan_check_status(plan) == 0
    rq, rk, rv = oracle.masked_attention_backward(wl, spec, dout_h, dlse_h)
    _close(dq, rq, f"{what} dq")
    _close(dk, rk, f"{what} dk")
    _close(dv, rv, f"{what} dv")


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("kind", KINDS)
def test_backward_all_kinds(kind, d):
    wl = W.random_small(seed=500 + d + 3 * KINDS.index(kind), kind=kind, batch=3, hq=4, hkv=2, d=d,
                        lmin=1, lmax=330)
    check_backward(wl, wl.masks[0], f"bwd {kind} d={d}")


@pytest.mark.parametrize("kind", ["CAUSAL", "CUSTOM"])
def test_backward_with_lse_gradient(kind):
    # a loss on lse as well: ds picks up p dlse (delta becomes dout . out - dlse)
    wl = W.random_small(seed=60 + len(kind), kind=kind, batch=2, hq=4, hkv=2, d=128, lmin=50, lmax=400)
    check_backward(wl, wl.masks[0], f"bwd dlse {kind}", seed=3, with_dlse=True)


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("g", [1, 4])
def test_backward_gqa_long(g, d):
    # several items per CTA and several jobs per item (the head_dim 256 kernels stream
    # their operands in half-tiles through a three-slot ring and run dK / dV in two passes)
    wl = W.random_small(seed=70 + g + d, kind="CAUSAL", batch=2, hq=2 * g, hkv=2, d=d, lmin=200, lmax=700)
    check_backward(wl, wl.masks[0], f"bwd gqa g={g} d={d}")


def test_backward_gemma2_shape_sliding_window():
    # the Gemma2 workload's shape at reduced length: head_dim 256, 2 query heads per KV head,
    # a sliding window narrower than the sequences
    wl = W.random_small(seed=77, kind="SLIDING_WINDOW", batch=2, hq=4, hkv=2, d=256, lmin=300, lmax=900)
    check_backward(wl, wl.masks[0], "bwd d=256 sliding window")


def test_backward_rows_without_keys_and_unseen_keys():
    # rows 0..9 see nothing (dq = 0); keys 600.. are seen by no query (dk = dv = 0)
    rng = np.random.default_rng(12)
    lq, lk = [190, 260], [700, 300]
    dense = []
    for a, b in zip(lq, lk):
        m = rng.random((a, b)) < 0.4
        m[:10] = False
        m[:, 600:] = False
        dense.append(m)
    words, offs = [], [0]
    for m in dense:
        w = W.pack_rows(m)
        words.append(w.reshape(-1))
        offs.append(offs[-1] + w.size)
    spec = W.MaskSpec("CUSTOM", bits=np.concatenate(words).astype(np.uint32), word_offsets=np.asarray(offs, np.int64))
    gen = torch.Generator().manual_seed(5)
    cq, ck = W.cu_from_lengths(lq), W.cu_from_lengths(lk)
    wl = W.Workload(name="bwd_masked", hq=4, hkv=2, d=128, scale=0.09, cu_seqlens_q=cq,
                    q=W.randn_bf16(gen, int(cq[-1]), 4, 128), masks=[spec], cu_seqlens_k=ck,
                    k=W.randn_bf16(gen, int(ck[-1]), 2, 128), v=W.randn_bf16(gen, int(ck[-1]), 2, 128), seed=5)
    check_backward(wl, spec, "bwd masked rows")


def test_backward_plan_required_and_unsupported():
    wl = W.random_small(seed=3, kind="CAUSAL", batch=2, hq=2, hkv=1, d=128, lmin=10, lmax=50)
    q, k, v = G.device_inputs(wl)
    plan = G.make_plan(wl, wl.masks[0])          # forward-only plan
    out, lse = G.M.forward(plan, q, k, v)
    with pytest.raises(G.M.AttnError) as e:
        G.M.backward(plan, q, k, v, out, lse, torch.zeros_like(out))
    assert e.value.status == 1
    # paged backward: not when two sequences read the same page (its gradient would be the sum
    # of both)
    wl = W.random_small(seed=4, kind="CAUSAL", batch=2, hq=2, hkv=1, d=128, lmin=40, lmax=60, paged=True)
    wl.page_table[1, 0] = wl.page_table[0, 0]
    with pytest.raises(G.M.AttnError) as e:
        _bwd_plan(wl, wl.masks[0])
    assert e.value.status == 2


def test_backward_full_size_chunk_causal_sampled():
    """The chunk-causal workload at full size (8 x 8192 tokens, 16 heads, d=128), both
    descriptor forms: dq on sampled rows (first / middle / last rows of every sequence and
    random ones) and dk, dv on sampled keys of two (sequence, head) pairs, against the oracle
    evaluated at those places; the two descriptor forms give identical gradients."""
    wl = W.config(4)
    q, k, v = G.device_inputs(wl)
    gen = torch.Generator().manual_seed(44)
    dout_h = W.randn_bf16(gen, q.shape[0], wl.hq, wl.d)
    dout = dout_h.cuda()
    rng = np.random.default_rng(44)
    qs = G.sample_rows(wl, 40, seed=44)
    ks = [(b, int(rng.integers(0, wl.hkv)), int(j)) for b in (0, 5) for j in
          list(rng.integers(0, wl.lk(b), size=6)) + [0, wl.lk(b) - 1, 4095, 4096]]
    grads = []
    for spec in wl.masks:
        plan = G.M.attn_plan(hq=wl.hq, hkv=wl.hkv, head_dim=wl.d, cu_seqlens_q=wl.cu_seqlens_q,
                             cu_seqlens_k=wl.cu_seqlens_k, mask=spec, scale=wl.scale, backward=True)
        out, lse = G.M.forward(plan, q, k, v)
        dq, dk, dv = G.M.backward(plan, q, k, v, out, lse, dout)
        assert G.M.attn_plan_check_status(plan) == 0
        grads.append((dq.cpu(), dk.cpu(), dv.cpu()))
    for a, b in zip(grads[0], grads[1]):
        assert torch.equal(a, b)
    dq, dk, dv = grads[0]
    rq, rk, rv = oracle.sampled_backward(wl, wl.masks[0], dout_h, qs, ks)
    got_q = torch.stack([dq[int(wl.cu_seqlens_q[b]) + i, h] for b, h, i in qs])
    got_k = torch.stack([dk[int(wl.cu_seqlens_k[b]) + j, kh] for b, kh, j in ks])
    got_v = torch.stack([dv[int(wl.cu_seqlens_k[b]) + j, kh] for b, kh, j in ks])
    _close(got_q, rq, "full-size dq")
    _close(got_k, rk, "full-size dk")
    _close(got_v, rv, "full-size dv")


def _full_size_sampled(cfg, seed, n_rows, key_pairs, n_keys, compare_forms):
    """Backward of a benchmark workload at full size, every mask of it, in the launch the
    benchmark times: dq on sampled rows (first / middle / last rows of every sequence and
    random ones), dk and dv on sampled keys of the given (sequence, KV head) pairs, against
    the oracle evaluated at those places; with `compare_forms`, the masks are two descriptor
    forms of one mask and must give identical gradients."""
    wl = W.config(cfg)
    q, k, v = G.device_inputs(wl)
    gen = torch.Generator().manual_seed(seed)
    dout_h = W.randn_bf16(gen, q.shape[0], wl.hq, wl.d)
    dout = dout_h.cuda()
    rng = np.random.default_rng(seed)
    qs = G.sample_rows(wl, n_rows, seed=seed)
    ks = [(b, kh, int(j)) for b, kh in key_pairs
          for j in list(rng.integers(0, wl.lk(b), size=n_keys)) + [0, wl.lk(b) - 1]]
    grads = []
    for spec in wl.masks:
        plan = G.M.attn_plan(hq=wl.hq, hkv=wl.hkv, head_dim=wl.d, cu_seqlens_q=wl.cu_seqlens_q,
                             cu_seqlens_k=wl.cu_seqlens_k, mask=spec, scale=wl.scale, backward=True)
        out, lse = G.M.forward(plan, q, k, v)
        dq, dk, dv = G.M.backward(plan, q, k, v, out, lse, dout)
        assert G.M.attn_plan_check_status(plan) == 0
        grads.append((spec, dq.cpu(), dk.cpu(), dv.cpu()))
    if compare_forms:
        for a, b in zip(grads[0][1:], grads[1][1:]):
            assert torch.equal(a, b)
        grads = grads[:1]
    for spec, dq, dk, dv in grads:
        rq, rk, rv = oracle.sampled_backward(wl, spec, dout_h, qs, ks)
        got_q = torch.stack([dq[int(wl.cu_seqlens_q[b]) + i, h] for b, h, i in qs])
        got_k = torch.stack([dk[int(wl.cu_seqlens_k[b]) + j, kh] for b, kh, j in ks])
        got_v = torch.stack([dv[int(wl.cu_seqlens_k[b]) + j, kh] for b, kh, j in ks])
        _close(got_q, rq, f"workload {cfg} {spec.kind} dq")
        _close(got_k, rk, f"workload {cfg} {spec.kind} dk")
        _close(got_v, rv, f"workload {cfg} {spec.kind} dv")


def test_backward_full_size_gemma2_sampled():
    """The Gemma2 workload (4 sequences up to 7028 tokens, 16 / 8 heads, d = 256), its
    sliding-window and causal masks, through the head_dim 256 kernels."""
    _full_size_sampled(2, seed=45, n_rows=24, key_pairs=[(0, 3), (2, 6)], n_keys=6, compare_forms=False)


def test_backward_full_size_block_dense_sampled():
    """The block-dense workload (one sequence of 29576 tokens, 32 / 8 heads, d = 128), as
    packed bits and as ranges (identical gradients), on sampled rows and on keys of one
    KV head, among them keys of the causal blocks past 24576."""
    _full_size_sampled(5, seed=46, n_rows=24, key_pairs=[(0, 5)], n_keys=6, compare_forms=True)


@pytest.mark.parametrize("d", [128, 256])
def test_backward_timeout_reports_and_context_survives(d):
    """The forced missing arrival of the debug hook in both backward kernels: a bounded wait
    expires, the status word reports ATTN_ERR_TIMEOUT, the kernels return through their abort
    paths, and the next backward on the same plan is correct."""
    wl = W.random_small(seed=6, kind="CAUSAL", batch=2, hq=4, hkv=2, d=d, lmin=100, lmax=300)
    q, k, v = G.device_inputs(wl)
    plan = G.M.attn_plan(hq=wl.hq, hkv=wl.hkv, head_dim=wl.d, cu_seqlens_q=wl.cu_seqlens_q,
                         cu_seqlens_k=wl.cu_seqlens_k, mask=wl.masks[0], scale=wl.scale, backward=True)
    out, lse = G.M.forward(plan, q, k, v)
    gen = torch.Generator().manual_seed(6)
    dout_h = W.randn_bf16(gen, q.shape[0], wl.hq, wl.d)
    G.M.attn_plan_set_debug(plan, 1, 50_000_000)   # 50 ms per wait
    G.M.backward(plan, q, k, v, out, lse, dout_h.cuda())
    assert G.M.attn_plan_check_status(plan) == 6
    G.M.attn_plan_set_debug(plan, 0, 0)
    dq, dk, dv = G.M.backward(plan, q, k, v, out, lse, dout_h.cuda())
    assert G.M.attn_plan_check_status(plan) == 0
    rq, rk, rv = oracle.masked_attention_backward(wl, wl.masks[0], dout_h)
    _close(dq, rq, "after timeout dq")
    _close(dk, rk, "after timeout dk")
    _close(dv, rv, "after timeout dv")


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("ps", [16, 64])
@pytest.mark.parametrize("kind", ["CAUSAL", "SLIDING_WINDOW", "CUSTOM"])
def test_backward_paged(kind, ps, d):
    # K / V from a paged cache (pages permuted, spare pages no sequence reads); dk / dv come
    # back in the cache layout, zero on every row no sequence reads
    wl = W.random_small(seed=80 + ps + d + len(kind), kind=kind, batch=3, hq=4, hkv=2, d=d, lmin=1, lmax=330,
                        paged=True, page_size=ps)
    check_backward(wl, wl.masks[0], f"bwd paged {kind} ps={ps} d={d}")


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("poison", [1e30, float("nan")])
def test_backward_paged_poison_in_unused_slots(poison, d):
    # the slots past each sequence's last key in its last page hold garbage; the dQ kernel
    # zeroes those K / V rows in shared memory, so the gradients are those of clean caches
    wl = W.random_small(seed=88, kind="CAUSAL", batch=3, hq=4, hkv=2, d=d, lmin=20, lmax=300, paged=True,
                        page_size=64)
    kc, vc = wl.k_cache.clone(), wl.v_cache.clone()
    for b in range(wl.batch):
        n = wl.lk(b)
        if n % wl.page_size:
            last = int(wl.page_table[b, n // wl.page_size])
            kc[last, n % wl.page_size:] = poison
            vc[last, n % wl.page_size:] = poison
    check_backward(wl, wl.masks[0], f"bwd paged poison {poison} d={d}", inputs=(wl.q.cuda(), kc.cuda(), vc.cuda()))
