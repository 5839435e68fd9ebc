"""GPU: the streaming-floor measurement kernel (gqa_stream_floor) runs to the end
on every grid size it accepts, leaves the status word clean, and streams at an
HBM-like rate on a buffer larger than L2."""
import pytest
import torch

import gqa_decode_attention_attn_b200 as gq

pytestmark = pytest.mark.gpu


def test_floor_runs_on_any_grid():
    dev = torch.device("cuda", 0)
    k = torch.randn(4096, 128, device=dev).to(torch.bfloat16)
    v = torch.randn(4096, 128, device=dev).to(torch.bfloat16)
    ws = gq.Workspace(dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    for ctas in (1, 3, 32, sms):                       # fewer and more CTAs than tiles
        for nbytes in (gq.FLOOR_TILE_BYTES, 5 * gq.FLOOR_TILE_BYTES, k.numel() * 2):
            gq.stream_floor(k, v, nbytes, ctas, ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    with pytest.raises(gq.GqaError):
        gq.stream_floor(k, v, gq.FLOOR_TILE_BYTES, sms + 1, ws)   # above the resident CTAs
    with pytest.raises(ValueError):
        gq.stream_floor(k, v, gq.FLOOR_TILE_BYTES + 256, 4, ws)
    with pytest.raises(ValueError):
        gq.stream_floor(k, v, k.numel() * 2 + gq.FLOOR_TILE_BYTES, 4, ws)


def test_floor_streams_at_hbm_rate():
    dev = torch.device("cuda", 0)
    n = 256 << 20                                       # 256 MiB each of K and V
    k = torch.empty(n, dtype=torch.uint8, device=dev)
    v = torch.empty(n, dtype=torch.uint8, device=dev)
    ws = gq.Workspace(dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    for _ in range(3):
        gq.stream_floor(k, v, n, sms, ws)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(10):
        gq.stream_floor(k, v, n, sms, ws)
    b.record()
    torch.cuda.synchronize()
    assert ws.status() == 0
    gbs = 10 * 2 * n / (a.elapsed_time(b) / 1e3) / 1e9
    assert gbs > 2000.0, gbs                            # a loose bound: the B200 streams ~6.5 TB/s
