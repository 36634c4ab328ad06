"""GPU parity of the e4m3 (fp8) forward against the fp64 oracle on the dequantised inputs.

Inputs: the bf16 workloads quantised per tensor to e4m3 (workloads.quantize_e4m3); the
oracle decodes the same bytes (oracle.decode_e4m3) and runs the plain fp64 attention.

Bound (per row, rigorous): the scores q8 . k8 are exact in fp32 (products of two e4m3
values are exact, and the sums stay well inside fp32 precision), so the error comes from
rounding P to e4m3 for the P V product: with p_ij = exp(s_ij - lse_i) (rows sum to one)
and the kernel's l >= 1 (its reference maximum never exceeds the row maximum), each
rounded P is off by at most max(2^-4 p_ij, 2^-10) in units of l (half an e4m3 ulp:
2^-4 relative for normal values, 2^-10 absolute for subnormals), plus the error of the
exponential before rounding: a quarter of the columns use the FMA-pipe polynomial, whose
relative error (7.5e-5, pinned by its own test) is below 2^-13, so
    |out_i - ref_i| <= v_scale sum_j (max(2^-4 p_ij, 2^-10) + 2^-13 p_ij) |v8_j| + 2^-8 |ref_i| + 1e-5,
the second term covering the bf16 rounding of out. lse uses P before rounding: 1e-3."""
import numpy as np
import pytest
import torch

import workloads as W
import oracle
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(attn_lib):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return attn_lib


def _run_fp8(wl, spec, kv_splits=0):
    q8, qs = W.quantize_e4m3(wl.q)
    k8, ks = W.quantize_e4m3(wl.k)
    v8, vs = W.quantize_e4m3(wl.v)
    plan = G.make_plan(wl, spec, kv_splits=kv_splits)
    ldv = (plan.stats["vt_keys"] + 15) // 16 * 16
    vt = torch.empty(wl.hkv, wl.d, max(ldv, 16), dtype=torch.uint8, device="cuda")
    G.M.attn_fp8_transpose_v(plan, v8.cuda(), vt, ldv)
    tq = int(wl.cu_seqlens_q[-1])
    out = torch.empty(tq, wl.hq, wl.d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(tq, wl.hq, dtype=torch.float32, device="cuda")
    G.M.attn_masked_fwd_fp8(plan, q8.cuda(), k8.cuda(), vt, ldv, qs, ks, vs, out, lse)
    assert G.M.attn_plan_check_status(plan) == 0
    deq = lambda t8, sc: torch.from_numpy(oracle.decode_e4m3(t8.numpy()) * sc)
    wl_deq = W.Workload(name=wl.name + "_e4m3", hq=wl.hq, hkv=wl.hkv, d=wl.d, scale=wl.scale,
                        cu_seqlens_q=wl.cu_seqlens_q, q=deq(q8, qs), masks=wl.masks, cu_seqlens_k=wl.cu_seqlens_k,
                        k=deq(k8, ks), v=deq(v8, vs), seed=wl.seed)
    return out.float().cpu().numpy(), lse.cpu().numpy(), wl_deq, plan


def _bound(wl_deq, spec):
    """Per-row bound of the module docstring, from the dequantised inputs."""
    g = wl_deq.hq // wl_deq.hkv
    tq = int(wl_deq.cu_seqlens_q[-1])
    bound = np.zeros((tq, wl_deq.hq))
    for b in range(wl_deq.batch):
        lq, lk = wl_deq.lq(b), wl_deq.lk(b)
        q0, k0 = int(wl_deq.cu_seqlens_q[b]), int(wl_deq.cu_seqlens_k[b])
        if lq == 0 or lk == 0:
            continue
        m = oracle.dense_mask(spec, b, lq, lk)
        for h in range(wl_deq.hq):
            q = wl_deq.q[q0:q0 + lq, h].numpy()
            k = wl_deq.k[k0:k0 + lk, h // g].numpy()
            v = wl_deq.v[k0:k0 + lk, h // g].numpy()
            _, lse = oracle.attention_one_head(q, k, v, m, wl_deq.scale)
            s = wl_deq.scale * q @ k.T
            has = np.isfinite(lse)
            p = np.where(m & has[:, None], np.exp(np.where(m, s, 0) - np.where(has, lse, 0)[:, None]), 0)
            w = np.where(m & has[:, None], np.maximum(2.0 ** -4 * p, 2.0 ** -10) + 2.0 ** -13 * p, 0)
            bound[q0:q0 + lq, h] = w @ np.abs(v).max(axis=1)
    return bound


def check_fp8(wl, spec, what, kv_splits=0):
    out, lse, wl_deq, plan = _run_fp8(wl, spec, kv_splits)
    ref_o, ref_l = oracle.masked_attention(wl_deq, spec)
    bound = _bound(wl_deq, spec)[..., None] + 2.0 ** -8 * np.abs(ref_o) + 1e-5
    err = np.abs(out - ref_o)
    assert np.isfinite(out).all(), f"{what}: non-finite"
    worst = (err / bound).max()
    assert worst <= 1.0, f"{what}: error {err.max():.3e} exceeds the e4m3 bound (ratio {worst:.2f})"
    fin = np.isfinite(ref_l)
    assert np.array_equal(fin, np.isfinite(lse)), f"{what}: -inf rows differ"
    if fin.any():
        assert np.abs(lse[fin] - ref_l[fin]).max() <= 1e-3, f"{what}: lse"
    return float(err.max()), float(worst)


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("kind", ["FULL", "CAUSAL", "SLIDING_WINDOW", "PREFIX_LM", "CHUNK_CAUSAL", "RANGES",
                                  "CUSTOM", "BLOCK_SPARSE"])
def test_fp8_all_kinds(kind, d):
    wl = W.random_small(seed=900 + len(kind) + d, kind=kind, batch=3, hq=4, hkv=2, d=d, lmin=1, lmax=400)
    check_fp8(wl, wl.masks[0], f"fp8 {kind} d={d}")


@pytest.mark.parametrize("d", [128, 256])
def test_fp8_short_queries_and_split(d):
    # head packing (short queries) and split-KV partials go through the same e4m3 kernels
    rng = np.random.default_rng(8)
    lq = rng.integers(1, 33, size=4)
    lk = lq + rng.integers(500, 1500, size=4)
    gen = torch.Generator().manual_seed(8)
    cq, ck = W.cu_from_lengths(lq), W.cu_from_lengths(lk)
    wl = W.Workload(name="fp8_short", hq=8, hkv=2, d=d, scale=d ** -0.5, cu_seqlens_q=cq,
                    q=W.randn_bf16(gen, int(cq[-1]), 8, d), masks=[W.MaskSpec("CAUSAL")], cu_seqlens_k=ck,
                    k=W.randn_bf16(gen, int(ck[-1]), 2, d), v=W.randn_bf16(gen, int(ck[-1]), 2, d), seed=8)
    check_fp8(wl, wl.masks[0], "fp8 short q")
    check_fp8(wl, wl.masks[0], "fp8 short q split", kv_splits=4)


def test_fp8_transpose_layout():
    # the transposed V: sequence b at 128-aligned columns, zeros in the gaps
    wl = W.random_small(seed=77, kind="CAUSAL", batch=3, hq=2, hkv=2, d=128, lmin=1, lmax=300)
    v8, _ = W.quantize_e4m3(wl.v)
    plan = G.make_plan(wl, wl.masks[0])
    ldv = (plan.stats["vt_keys"] + 15) // 16 * 16
    vt = torch.full((wl.hkv, wl.d, ldv), 0xAB, dtype=torch.uint8, device="cuda")
    G.M.attn_fp8_transpose_v(plan, v8.cuda(), vt, ldv)
    got = vt.cpu().numpy()
    col = 0
    for b in range(wl.batch):
        lk, k0 = wl.lk(b), int(wl.cu_seqlens_k[b])
        want = v8[k0:k0 + lk].numpy().transpose(1, 2, 0)          # [hkv][d][lk]
        assert np.array_equal(got[:, :, col:col + lk], want)
        pad = (lk + 127) // 128 * 128
        assert np.all(got[:, :, col + lk:col + pad] == 0)
        col += pad
    assert col == plan.stats["vt_keys"]


def test_fp8_unsupported_and_invalid():
    wl = W.random_small(seed=1, kind="CAUSAL", batch=2, hq=2, hkv=1, d=64, lmin=10, lmax=50)
    plan = G.make_plan(wl, wl.masks[0])
    z = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    out = torch.zeros(int(wl.cu_seqlens_q[-1]), 2, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(G.M.AttnError) as e:
        G.M.attn_masked_fwd_fp8(plan, z, z, z, 128, 1.0, 1.0, 1.0, out)
    assert e.value.status == 2
    wl = W.random_small(seed=1, kind="CAUSAL", batch=2, hq=2, hkv=1, d=128, lmin=10, lmax=50)
    plan = G.make_plan(wl, wl.masks[0])
    with pytest.raises(G.M.AttnError) as e:   # ldv not a multiple of 16
        G.M.attn_masked_fwd_fp8(plan, z, z, z, plan.stats["vt_keys"] + 1, 1.0, 1.0, 1.0, out)
    assert e.value.status == 1
