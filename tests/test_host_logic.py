"""CPU checks of host-side helpers: FP8 cache preparation, the dispatch report
(gqa_decode_plan) and traffic-record keying, workspace sizes."""
import os
import sys

import pytest
import torch

import gqa_decode_attention_attn_b200 as gq
import workloads
from workloads import fp8_caches, make_problem

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def test_fp8_caches_range_scale_and_poison():
    p = make_problem("fp8h", 2, 8, 2, 64, [37, 5], seed=3, block_size=8, spare_blocks=2,
                     key_outlier_frac=0.05)
    k8, v8, ks, vs = fp8_caches(p)
    assert k8.dtype == torch.uint8 and k8.shape == p.k_cache.shape
    assert ks > 0 and vs > 0
    kf = k8.view(torch.float8_e4m3fn).to(torch.float32)
    fin = torch.isfinite(p.k_cache.float())
    assert torch.all(torch.isnan(kf[~fin]))          # poison stays NaN
    assert torch.all(kf[fin].abs() <= 448)          # every finite value representable
    assert kf[fin].abs().max() == 448               # the largest maps to E4M3's maximum
    # dequantised values track the bf16 originals within E4M3 precision (3 mantissa bits)
    err = (kf[fin] * ks - p.k_cache.float()[fin]).abs()
    assert torch.all(err <= p.k_cache.float()[fin].abs() * 2 ** -4 + ks * 2 ** -9)


def _plan(B, Hq, Hkv, D, bs=None, paged=False, nb=0, **kw):
    return gq.decode_plan(B, Hq, Hkv, D, bs if bs is not None else 4096, paged, nb, device=-1,
                          **kw)


def test_plan_reports_the_dispatch():
    """gqa_decode_plan (no device query) reports the kernel the launch path takes."""
    tc, cc = gq.KERNEL_TENSOR_CORE, gq.KERNEL_CUDA_CORE
    p = _plan(16, 32, 8, 128, seq_lens_host=[8192] * 16)
    assert p["kernel"] == tc and p["heads_per_pass"] == 4 and p["head_chunks"] == 1
    assert p["kernel_name"] == "gqa_decode_tc_kernel<NV=4,MQ=0,D=128,F8=0>"
    assert p["cooperative"] == 1 and p["tile_tokens"] == 128 and p["tiles"] == 16 * 8 * 64
    assert _plan(1, 32, 32, 128)["kernel"] == cc                      # G = 1
    d64 = _plan(1, 32, 8, 64)
    assert d64["kernel"] == tc and d64["ring_stages"] == 5            # D = 64, deep ring
    d256 = _plan(1, 32, 8, 256)                                       # D = 256: two slots per tile
    assert d256["kernel"] == tc and d256["kernel_name"] == "gqa_decode_tc_kernel<NV=4,MQ=0,D=256,F8=0>"
    assert d256["ring_stages"] == 3
    assert _plan(1, 32, 16, 256)["kernel"] == cc                      # D = 256, G = 2
    assert _plan(1, 32, 8, 128, bs=48, paged=True, nb=10)["kernel"] == cc  # page size
    assert _plan(1, 32, 8, 128, bs=64, paged=True, nb=10)["box_rows"] == 64
    f8 = _plan(1, 32, 8, 128, kv_fp8=True, seq_lens_host=[1000])
    assert f8["kernel"] == tc and f8["kernel_name"].endswith("F8=1>")
    assert f8["tile_tokens"] == 256 and f8["ring_stages"] == 3 and f8["tiles"] == 8 * 4  # 256-token tiles
    assert _plan(1, 32, 8, 64, kv_fp8=True)["kernel"] == cc           # FP8 at D = 64
    mqa = _plan(8, 64, 1, 128, seq_lens_host=[100] * 8)   # G = 64: one 64-head pass per tile
    assert mqa["heads_per_pass"] == 64 and mqa["head_chunks"] == 1 and mqa["tiles"] == 8
    assert mqa["kernel_name"] == "gqa_decode_tc_wide_kernel<NV=64,D=128>" and mqa["ring_stages"] == 3
    assert _plan(2, 128, 1, 128)["head_chunks"] == 2                  # G = 128: two passes of 64
    assert _plan(2, 32, 1, 128)["heads_per_pass"] == 64               # G = 32 on the wide kernel
    assert _plan(2, 32, 2, 128)["heads_per_pass"] == 16               # G = 16 stays at 16
    assert _plan(2, 64, 1, 64)["heads_per_pass"] == 16                # D = 64: 16-head passes
    wfx = _plan(2, 64, 1, 128, num_splits=4)                          # fixed split: 16-head kernel
    assert wfx["heads_per_pass"] == 16 and wfx["grid"] == 2 * 4 * 4
    assert _plan(2, 64, 1, 128, num_splits=1)["heads_per_pass"] == 64
    assert _plan(2, 32, 8, 128, qlen=4)["kernel_name"].startswith("gqa_decode_tc_kernel<NV=16,MQ=1")
    fx = _plan(2, 32, 8, 128, num_splits=4)
    assert fx["num_splits"] == 4 and fx["grid"] == 2 * 8 * 4 and fx["merge_launch"] == 1
    assert _plan(0, 32, 8, 128)["kernel"] == 0                        # nothing launched
    # a traffic record is keyed to the sources of the kernel the plan names
    import bench
    assert bench.kernel_source_hash(p["kernel_name"]) != \
        bench.kernel_source_hash(_plan(1, 32, 32, 128)["kernel_name"])


def test_plan_errors():
    with pytest.raises(gq.GqaError) as e:
        _plan(2, 32, 16, 256, num_splits=2)       # fixed split needs the tensor-core kernel
    assert e.value.code == 2
    with pytest.raises(gq.GqaError) as e:
        _plan(2, 32, 8, 256, qlen=2)              # several query tokens at D = 256: not built
    assert e.value.code == 2
    with pytest.raises(gq.GqaError) as e:
        _plan(2, 32, 8, 128, num_splits=-1)       # auto needs lengths and a device
    assert e.value.code == 1
    with pytest.raises(gq.GqaError) as e:
        _plan(2, 32, 8, 128, qlen=2, kv_fp8=True)
    assert e.value.code == 2
    with pytest.raises(gq.GqaError) as e:
        _plan(2, 30, 8, 128)                      # Hq % Hkv != 0
    assert e.value.code == 1
    with pytest.raises(gq.GqaError):
        _plan(1, 32, 8, 128, seq_lens_host=[-1])


def test_fixed_split_workspace_grows_with_splits():
    sizes = [gq.fixed_split_workspace_size(16, 32, 8, 128, s, 0) for s in (1, 2, 8, 32)]
    assert sizes == sorted(sizes) and sizes[0] < sizes[-1]


def test_timeline_summary():
    import numpy as np
    # Three CTAs over a 10 us span: busy 10 + 8 + 2 = 20 of 30 us; the idle one has no tiles.
    tl = np.array([[1000, 11000, 0, 5, 1500, 3000, 9000, 10500],
                   [2000, 10000, 1, 4, 2500, 4000, 9500, 9900],
                   [1000, 3000, 2, 0, 0, 0, 0, 0]])
    s = gq.timeline_summary(tl)
    assert s["ctas"] == 3 and s["ctas_with_work"] == 2 and s["sms"] == 3 and s["tiles"] == 9
    assert abs(s["span_us"] - 10.0) < 1e-12
    assert abs(s["busy_frac"] - 20.0 / 30.0) < 1e-12
    assert abs(s["tail_idle"] - 10.0 / 30.0) < 1e-12
    assert s["start_us_max"] == 1.0
    assert s["end_us_min"] == 9.0 and s["end_us_max"] == 10.0   # CTAs with tiles only
    ph = s["phases_us"]                 # after each CTA's own start, recorded rows only
    assert ph["first_tma"] == {"median": 0.5, "max": 0.5}
    assert ph["first_scores"] == {"median": 2.0, "max": 2.0}
    assert ph["streamed"] == {"median": 7.75, "max": 8.0}
    assert ph["merged"] == {"median": 8.7, "max": 9.5}
    assert gq.timeline_summary(np.array([[0, 5, 0, 1] + [0] * 4]))["phases_us"] == {}
    with pytest.raises(ValueError):
        gq.timeline_summary(np.array([[5, 4, 0, 1] + [0] * 4]))   # ends before it starts
    with pytest.raises(ValueError):
        gq.timeline_summary(np.zeros((0, 8)))
    with pytest.raises(ValueError):
        gq.timeline_summary(np.zeros((2, 4)))                     # rows of the wrong width


def test_cpu_baseline_reports_parity_of_its_sample():
    import bench
    import oracle
    p = make_problem("cb", 3, 8, 2, 128, [300, 5, 900], seed=5, block_size=16)
    ref = oracle.gqa_decode(p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, p.scale)
    exact = torch.from_numpy(ref).to(torch.bfloat16)    # the correctly rounded result
    r = bench.cpu_oracle_sample(p, 0.2, gpu_out=exact)
    par = r["parity_of_sample"]
    assert par["rows"] == 3 * 8                         # every request compared once
    assert par["max_abs"] <= 1e-2 and par["rel_rms"] <= 2e-3
    wrong = exact.clone()
    wrong[1, 3, 7] += 1.0                               # one wrong element is seen
    assert bench.cpu_oracle_sample(p, 0.2, gpu_out=wrong)["parity_of_sample"]["max_abs"] > 0.9
    assert "parity_of_sample" not in bench.cpu_oracle_sample(p, 0.05)


def test_bf16_scaled_bound_is_the_binade_half_ulp():
    """The stress-case tolerance: half a bf16 ulp of |ref|'s binade plus slack, and
    exactly MAX_ABS below |ref| = 4; every correctly rounded value meets it."""
    import numpy as np
    from gpu_util import MAX_ABS, bf16_scaled_bound, half_ulp_bf16
    assert half_ulp_bf16(np.array([1.0, 1.99, 2.0, 4.0, 4.5, 7.99]))[[0, 1, 2, 3, 4, 5]].tolist() == \
        [2 ** -8, 2 ** -8, 2 ** -7, 2 ** -6, 2 ** -6, 2 ** -6]
    below = np.linspace(-3.999, 3.999, 10001)
    assert np.all(bf16_scaled_bound(below) == MAX_ABS)
    assert bf16_scaled_bound(np.array([4.5]))[0] < 2 ** -6 + 2e-3
    x = torch.randn(200000, dtype=torch.float64) * 8
    rounded = x.to(torch.bfloat16).double()
    assert np.all((rounded - x).abs().numpy() <= bf16_scaled_bound(x.numpy()))
    # a one-ulp miss above 4 is caught
    assert not np.all(2 * half_ulp_bf16(np.array([4.5])) <= bf16_scaled_bound(np.array([4.5])))
