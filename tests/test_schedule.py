"""Host-side schedule selector (gqa_select_schedule): runs on the CPU.

The selector follows the runtime selection policy of the LeanAttention decode
tiles digest (section "Runtime selection policy"): inputs are the context-length
distribution, heads per device, head dimension and SM count.
"""
import pytest

import gqa_decode_attention_attn_b200 as gq


def test_selector_follows_the_policy():
    import workloads
    # Large uniform batch (128 segments for 148 SMs): one CTA per segment, no
    # reduction (stream-K over 128 of the 148 CTAs does the same work: a tie, which
    # goes to the schedule that needs neither a cooperative launch nor merges).
    n, (sk, fs) = gq.select_schedule([8192] * 16, 32, 8, 128, 148)
    assert n == 1 and fs <= sk
    # Long context, few KV heads; uneven continuous batch: stream-K.
    for lens, hq, hkv in (([262144], 32, 2), ([1, 5, 100000, 300], 32, 8),
                          (workloads.varlen_lengths(64, 1003), 32, 8)):
        n, (sk, fs) = gq.select_schedule(lens, hq, hkv, 128, 148)
        assert n == 0 and 0 < sk <= fs


def test_selector_estimates_scale_with_work():
    _, (a, _) = gq.select_schedule([8192] * 16, 32, 8, 128, 148)
    _, (b, _) = gq.select_schedule([16384] * 16, 32, 8, 128, 148)
    assert 1.8 < b / a < 2.2


def test_selector_fixed_split_not_applicable_off_the_tensor_core_shapes():
    n, (sk, fs) = gq.select_schedule([4096] * 4, 32, 16, 256, 148)  # D = 256, G = 2
    assert n == 0 and fs == -1.0 and sk > 0
    n, (_, fs) = gq.select_schedule([4096] * 4, 32, 32, 128, 148)  # G = 1
    assert n == 0 and fs == -1.0
    # D = 256 with G >= 4 runs on the tensor cores (two ring slots per tile).
    _, (sk, fs) = gq.select_schedule([4096] * 4, 32, 8, 256, 148)
    assert sk > 0 and fs > 0


def test_selector_covers_head_dim_64_on_the_tensor_cores():
    # D = 64 runs on the tensor-core kernel, so the fixed split is a candidate too,
    # and a tile costs half the bytes of D = 128.
    n, (sk, fs) = gq.select_schedule([8192] * 16, 32, 8, 64, 148)
    assert n == 1 and 0 < fs <= sk
    _, (sk128, _) = gq.select_schedule([8192] * 16, 32, 8, 128, 148)
    assert 0.4 < sk / sk128 < 0.6


def test_selector_empty_and_bad_arguments():
    n, (sk, _) = gq.select_schedule([], 32, 8, 128, 148)
    assert n == 0 and sk >= 0
    with pytest.raises(gq.GqaError):
        gq.select_schedule([10, -1], 32, 8, 128, 148)
    with pytest.raises(gq.GqaError):
        gq.select_schedule([10], 32, 8, 128, 0)
    with pytest.raises(gq.GqaError):
        gq.select_schedule([10], 30, 8, 128, 148)
