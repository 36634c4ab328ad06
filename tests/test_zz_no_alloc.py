"""GPU tests of attn_masked_fwd_noalloc, the forward for callers that cannot allocate device
memory (for example a serving runtime that hands out every device buffer from its own pool,
or code that may not call cudaMalloc / cudaFree while it runs). The call keeps its plan in a
fixed array inside the library. These tests call it through the C ABI:

  * twice in a row on one stream, on different problems, with no host synchronisation in
    between, and check both outputs against the fp64 oracle and against the regular
    attn_plan + attn_masked_fwd path, with the tolerances of the other parity tests; the
    torch allocator's counters and the device's free memory must not move across the calls;
  * with a bounded wait forced to expire inside the kernel: the rows it did not compute keep
    lse = NaN, and the next call (debug settings restored) is correct again;
  * beyond the array's size, and with a CUSTOM mask: rejected before any device work.

The file is collected last, so a run that stops at the first failure has run every other
test before these."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
import masked_flash_attention_attn_b200 as M
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


def _buffers(wl):
    tq = int(wl.cu_seqlens_q[-1])
    out = torch.full((tq, wl.hq, wl.d), 5.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((tq, wl.hq), 5.0, dtype=torch.float32, device="cuda")
    return out, lse


def _enqueue(wl, spec, inputs, out, lse, page_table=None):
    """One attn_masked_fwd_noalloc call on the current stream (no synchronisation)."""
    q, k, v = inputs
    kw = dict(hq=wl.hq, hkv=wl.hkv, head_dim=wl.d, cu_seqlens_q=wl.cu_seqlens_q, mask=spec, scale=wl.scale,
              q=q, k=k, v=v, out=out, lse=lse)
    if wl.paged:
        kw.update(kv_lens=wl.kv_lens, page_table=page_table, page_size=wl.page_size, num_pages=wl.k_cache.shape[0])
    else:
        kw.update(cu_seqlens_k=wl.cu_seqlens_k)
    M.attn_masked_fwd_noalloc(**kw)


def _cases():
    return [W.random_small(seed=61, kind="CHUNK_CAUSAL", batch=3, hq=4, hkv=2, d=128, lmin=100, lmax=600),
            W.random_small(seed=62, kind="SLIDING_WINDOW", batch=4, hq=8, hkv=2, d=256, lmin=1, lmax=500,
                           paged=True)]


def test_noalloc_two_calls_in_a_row_match_oracle_and_allocate_nothing(attn_lib):
    assert torch.cuda.is_available()
    cases = _cases()
    inputs = [G.device_inputs(wl) for wl in cases]
    pts = [torch.from_numpy(wl.page_table).cuda() if wl.paged else None for wl in cases]
    bufs = [_buffers(wl) for wl in cases]
    # the first call on a device looks up the array's address (and may load the module):
    # make it before taking the memory figures
    _enqueue(cases[0], cases[0].masks[0], inputs[0], *bufs[0], page_table=pts[0])
    torch.cuda.synchronize()
    before = (torch.cuda.memory_allocated(), torch.cuda.memory_reserved(), torch.cuda.mem_get_info()[0])
    for wl, inp, (out, lse), pt in zip(cases, inputs, bufs, pts):
        _enqueue(wl, wl.masks[0], inp, out, lse, page_table=pt)   # back to back, one stream
    torch.cuda.synchronize()
    after = (torch.cuda.memory_allocated(), torch.cuda.memory_reserved(), torch.cuda.mem_get_info()[0])
    assert after == before, f"device memory moved across the calls: {before} -> {after}"
    for wl, inp, (out, lse) in zip(cases, inputs, bufs):
        ref_o, ref_l = oracle.masked_attention(wl, wl.masks[0])
        G.compare(out.float().cpu(), lse.cpu(), ref_o, ref_l, f"noalloc vs oracle {wl.name}")
        reg_o, reg_l, _ = G.run(wl, wl.masks[0], inp)
        G.compare(out.float().cpu(), lse.cpu(), reg_o.numpy().astype(np.float64),
                  reg_l.numpy().astype(np.float64), f"noalloc vs attn_masked_fwd {wl.name}")


def test_noalloc_expired_wait_leaves_nan_lse(attn_lib):
    wl = _cases()[0]
    inputs = G.device_inputs(wl)
    out, lse = _buffers(wl)
    try:
        # every CTA skips its first item's query load: its wait expires after 50 ms and the
        # CTA stops, so the rows of its items are never written
        M.attn_test_noalloc_debug(1, 50_000_000)
        _enqueue(wl, wl.masks[0], inputs, out, lse)
        torch.cuda.synchronize()
    finally:
        M.attn_test_noalloc_debug(0, 2_000_000_000)
    assert torch.isnan(lse).any(), "rows left uncomputed by an expired wait must read lse = NaN"
    # the context is intact and the next call computes every row
    out, lse = _buffers(wl)
    _enqueue(wl, wl.masks[0], inputs, out, lse)
    torch.cuda.synchronize()
    assert not torch.isnan(lse).any()
    ref_o, ref_l = oracle.masked_attention(wl, wl.masks[0])
    G.compare(out.float().cpu(), lse.cpu(), ref_o, ref_l, "noalloc after an expired wait")


def test_noalloc_rejects_plans_beyond_its_scratch(attn_lib):
    # 16384 sequences of 128 tokens x 64 heads: about a million 64-byte work items (68 MiB,
    # see the CPU test of this premise), rejected before any device work (no tensors are touched)
    cq, kw = G.noalloc_too_large_problem()
    with pytest.raises(M.AttnError) as e:
        M.attn_masked_fwd_noalloc(cu_seqlens_q=cq, cu_seqlens_k=cq, mask=W.MaskSpec("FULL"), q=None, k=None,
                                  v=None, out=None, **kw)
    assert e.value.status == 7
    with pytest.raises(M.AttnError) as e:
        wl = W.random_small(seed=3, kind="CUSTOM", batch=2)
        out, lse = _buffers(wl)
        _enqueue(wl, wl.masks[0], G.device_inputs(wl), out, lse)
    assert e.value.status == 2
