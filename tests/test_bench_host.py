"""Host-side pieces of bench.py's measurement (no GPU): the roofline peak it picks from the
sampled clocks, the algorithmic FLOPs of a workload (4 d per unmasked pair and head, from
the planner's pair count) and the kernel it names for a workload and pass."""
import bench
import workloads as W


def test_choose_peak_burst_sustained_and_e4m3(monkeypatch):
    fake = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6500.0}
    monkeypatch.setattr(bench, "peaks", lambda: (dict(fake), "test"))
    at_max = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0}
    capped = {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0}
    assert bench.choose_peak(at_max)[0] == 1600.0                 # a short run at full clock: burst
    assert bench.choose_peak(capped)[0] == 1400.0                 # below 90 % of the max clock: sustained
    assert bench.choose_peak({"error": "no NVML"})[0] == 1600.0   # no samples: burst
    assert bench.choose_peak(at_max, fp8=True, e4m3_tflops=3030.0)[0] == 3030.0   # measured e4m3 rate
    assert bench.choose_peak(at_max, fp8=True)[0] == 3200.0       # else bf16 x the nominal 2
    assert bench.choose_peak(at_max)[2] == 6500.0


def test_flops_of_the_chunk_causal_workload(attn_lib):
    # 8 sequences x 16 heads x 33,560,576 visible pairs (causal half + chunk-causal half, the
    # closed form of the oracle's pins), 4 d FLOPs each at d = 128: 2.199 TFLOP per forward
    wl = W.config(4)
    for spec in wl.masks:
        st = attn_lib.attn_plan_dry_run(hq=wl.hq, hkv=wl.hkv, head_dim=wl.d, cu_seqlens_q=wl.cu_seqlens_q,
                                        cu_seqlens_k=wl.cu_seqlens_k, mask=spec)
        assert bench.flops_of(st, wl) == 4.0 * 128 * 16 * 8 * 33_560_576


def test_kernel_names():
    assert bench.kernel_name(W.config(5)) == "masked_attn_fwd_kernel d=128"
    assert bench.kernel_name(W.config(2)) == "masked_attn_fwd_pair_kernel (2-SM) d=256"
    assert bench.kernel_name(W.config(3)) == "masked_attn_fwd_kernel d=128 paged"
    assert bench.kernel_name(W.config(2), fp8=True) == "masked_attn_fwd_pair_kernel (2-SM) e4m3 d=256"
    assert bench.kernel_name(W.config(4), bwd=True) == "masked_attn_bwd_dq_kernel + masked_attn_bwd_dkv_kernel d=128"
    assert bench.kernel_name(W.config(2), bwd=True) == \
        "masked_attn_bwd256_dq_kernel + masked_attn_bwd256_dkv_kernel d=256"
