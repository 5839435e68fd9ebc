"""GPU parity of the FP8 E4M3 cache path (gqa_decode_fp8, gqa_decode_fp8_auto)
against the fp64 oracle on the same E4M3 bytes and scales: the tensor-core kernel
(D = 128, G >= 4) and the CUDA-core kernel (the other shapes)."""
import pytest
import torch

import gqa_decode_attention_attn_b200 as gq
import oracle
import workloads
from gpu_util import parity
from workloads import fp8_caches, make_problem

pytestmark = pytest.mark.gpu

CASES = [
    # B, Hq, Hkv, D, lens, block_size
    (3, 8, 2, 128, [1, 63, 700], None),
    (2, 32, 8, 128, [3000, 129], 16),       # G = 4
    (2, 8, 8, 128, [500, 64], 32),          # MHA
    (2, 16, 1, 128, [1000, 7], 64),         # G = 16: two head chunks
    (3, 4, 2, 64, [128, 127, 900], 8),
    (2, 16, 4, 256, [777, 2], 16),
    (1, 4, 1, 128, [60000], None),          # one long segment over every CTA
    (2, 16, 2, 128, [5000, 300], 32),       # G = 8
    (1, 32, 2, 128, [40000], 64),           # G = 16, long: split segments merged
    # 256-token LeanTiles on the tensor cores: lengths around tile and half-tile
    # edges, 8-token pages (32 TMA boxes per tile, a full warp of them), pages of a
    # whole tile, a contiguous cache
    (4, 16, 4, 128, [255, 256, 257, 129], 8),
    (3, 8, 2, 128, [511, 513, 128], 256),
    (2, 32, 8, 128, [384, 1], None),
    (2, 64, 4, 128, [3000, 700], 32),       # G = 16: two head chunks per KV head
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}_Hq{c[1]}_Hkv{c[2]}_D{c[3]}_bs{c[5]}")
def test_fp8_matches_oracle(case):
    B, Hq, Hkv, D, lens, bs = case
    p = make_problem("fp8", B, Hq, Hkv, D, lens, seed=500 + sum(lens) + D, block_size=bs,
                     spare_blocks=2 if bs else 0, key_outlier_frac=0.01)
    k8, v8, ks, vs = fp8_caches(p)
    d = p.to("cuda")
    ws = gq.Workspace(d.q.device)
    out = gq.gqa_decode_fp8(d.q, k8.cuda(), v8.cuda(), ks, vs, d.block_table, d.seq_lens,
                            scale=p.scale, workspace=ws)
    assert ws.status() == 0
    ref = oracle.gqa_decode_fp8(p.q, k8, v8, ks, vs, p.block_table, p.seq_lens, p.scale)
    parity(out.cpu(), ref, str(case), bf16_scaled=True)


def test_fp8_llama3_shape_full():
    """The full-size FP8 step (Llama-3-8B shape, 1% of keys x8): all 512 query rows."""
    p = workloads.workload("llama3_8b_fp8")
    k8, v8, ks, vs = fp8_caches(p)
    d = p.to("cuda")
    out = gq.gqa_decode_fp8(d.q, k8.cuda(), v8.cuda(), ks, vs, d.block_table, d.seq_lens,
                            scale=p.scale).cpu()
    ref = oracle.gqa_decode_fp8(p.q, k8, v8, ks, vs, p.block_table, p.seq_lens, p.scale)
    parity(out, ref, "llama3_8b_fp8", bf16_scaled=True)


AUTO_CASES = [
    # B, Hq, Hkv, D, lens, block_size
    (4, 32, 8, 128, [3000, 129, 2048, 7], 16),  # G = 4, uneven lengths
    (1, 32, 2, 128, [40000], 64),           # one long request: stream-K, segments merged
    (2, 64, 1, 128, [30000, 500], 64),      # G = 64: four 16-head passes (no wide kernel)
    (3, 4, 2, 64, [128, 127, 900], 8),      # D = 64: the CUDA-core kernel, stream-K
]


@pytest.mark.parametrize("case", AUTO_CASES, ids=lambda c: f"B{c[0]}_Hq{c[1]}_Hkv{c[2]}_D{c[3]}")
def test_fp8_auto_matches_oracle_and_its_plan(case):
    """gqa_decode_fp8_auto: the schedule gqa_decode_plan reports for the FP8 cache
    (kv_fp8, num_splits = -1) and the oracle's result on the same E4M3 bytes."""
    B, Hq, Hkv, D, lens, bs = case
    p = make_problem("fp8a", B, Hq, Hkv, D, lens, seed=900 + sum(lens) % 97 + D, block_size=bs,
                     spare_blocks=2, key_outlier_frac=0.01)
    k8, v8, ks, vs = fp8_caches(p)
    d = p.to("cuda")
    host = p.seq_lens.to(torch.int32).contiguous()
    plan = gq.decode_plan(B, Hq, Hkv, D, bs, True, p.num_blocks, kv_fp8=True, num_splits=-1,
                          seq_lens_host=host, device=0)
    if D == 128:
        assert plan["kernel"] == gq.KERNEL_TENSOR_CORE and plan["heads_per_pass"] == min(16, Hq // Hkv)
        # 256-token LeanTiles: tiles = head passes x KV heads x sum of ceil(L / 256)
        assert plan["tile_tokens"] == 256
        assert plan["tiles"] == plan["head_chunks"] * Hkv * sum(-(-L // 256) for L in lens)
    else:
        assert plan["kernel"] == gq.KERNEL_CUDA_CORE and plan["num_splits"] == 0
    if B == 1:  # two segments on 148 SMs: stream-K
        assert plan["num_splits"] == 0
    ws = gq.Workspace(d.q.device)
    out = gq.gqa_decode_fp8_auto(d.q, k8.cuda(), v8.cuda(), ks, vs, d.block_table, d.seq_lens,
                                 host, scale=p.scale, workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    ref = oracle.gqa_decode_fp8(p.q, k8, v8, ks, vs, p.block_table, p.seq_lens, p.scale)
    parity(out.cpu(), ref, f"auto {case}", bf16_scaled=True)


def test_fp8_auto_llama3_shape_full():
    """The full-size FP8 step through gqa_decode_fp8_auto (one CTA per (request, KV
    head), the schedule the bench times): all 512 query rows against the oracle."""
    p = workloads.workload("llama3_8b_fp8")
    k8, v8, ks, vs = fp8_caches(p)
    d = p.to("cuda")
    host = p.seq_lens.to(torch.int32).contiguous()
    plan = gq.decode_plan(p.B, p.Hq, p.Hkv, p.D, p.block_size, p.paged, p.num_blocks,
                          kv_fp8=True, num_splits=-1, seq_lens_host=host, device=0)
    assert plan["num_splits"] == 1 and plan["kernel_name"].endswith("F8=1>")
    out = gq.gqa_decode_fp8_auto(d.q, k8.cuda(), v8.cuda(), ks, vs, d.block_table, d.seq_lens,
                                 host, scale=p.scale).cpu()
    ref = oracle.gqa_decode_fp8(p.q, k8, v8, ks, vs, p.block_table, p.seq_lens, p.scale)
    parity(out, ref, "llama3_8b_fp8 auto", bf16_scaled=True)
