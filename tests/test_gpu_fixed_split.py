"""GPU parity of the fixed-split comparator (gqa_decode_fixed_split) against the
fp64 oracle, and its agreement with the stream-K gqa_decode."""
import pytest
import torch

import gqa_decode_attention_attn_b200 as gq
import oracle
from gpu_util import parity
from workloads import make_problem

pytestmark = pytest.mark.gpu

CASES = [
    # B, Hq, Hkv, lens, block_size, splits
    (4, 32, 8, [3000, 1, 700, 129], None, 1),
    (4, 32, 8, [3000, 1, 700, 129], None, 3),
    (2, 32, 2, [20000, 5000], 64, 7),
    (3, 16, 1, [100, 5000, 1280], 16, 64),     # more chunks than tiles: empty chunks
    (2, 64, 2, [4000, 999], 32, 4),             # G = 32: two head chunks
    (5, 8, 1, [0, 17, 0, 2500, 64], 16, 5),     # empty requests
    (2, 32, 4, [9000, 130], 16, 5, 64),         # D = 64
    (2, 64, 1, [6000, 999], 32, 1),             # G = 64, one CTA per segment: the 64-head kernel
    (2, 64, 1, [6000, 999], 32, 4),             # G = 64 split in 4: 16-head passes
    (2, 16, 4, [9000, 130], 16, 5, 256),        # D = 256
    (3, 16, 4, [2000, 1, 4100], None, 1, 256),  # D = 256, one CTA per segment
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}_Hq{c[1]}_Hkv{c[2]}_bs{c[4]}_s{c[5]}")
def test_fixed_split_matches_oracle_and_stream_k(case):
    B, Hq, Hkv, lens, bs, splits, *rest = case
    D = rest[0] if rest else 128
    p = make_problem("fixed", B, Hq, Hkv, D, lens, seed=700 + sum(lens) + splits, block_size=bs,
                     key_outlier_frac=0.01)
    d = p.to("cuda")
    ws = gq.Workspace(d.q.device)
    out = gq.gqa_decode_fixed_split(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens, splits,
                                    scale=p.scale, workspace=ws)
    assert ws.status() == 0
    ref = oracle.gqa_decode(p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, p.scale)
    parity(out.cpu(), ref, str(case), bf16_scaled=True)
    sk = gq.gqa_decode(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens, scale=p.scale)
    diff = (out.float() - sk.float()).abs().max().item()
    assert diff <= 2e-2


def test_fixed_split_rejects_cuda_core_shapes():
    p = make_problem("fixedg1", 2, 8, 8, 128, [100, 50], seed=3)    # G = 1
    d = p.to("cuda")
    with pytest.raises(gq.GqaError):
        gq.gqa_decode_fixed_split(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens, 2,
                                  scale=p.scale)


@pytest.mark.parametrize("lens,hq,hkv,bs,D", [
    ([3000] * 16, 32, 8, None, 128),     # uniform, many segments: one CTA per segment
    ([40000], 32, 2, 64, 128),           # long context: stream-K
    ([100, 7000, 1, 2500], 32, 8, 16, 128),  # uneven: stream-K
    ([9000, 3000], 64, 1, 32, 128),      # MQA: the 64-head kernel
    ([3000] * 40, 64, 2, 16, 128),       # MQA, many segments: one CTA per segment
    ([20000, 1, 5000], 16, 4, 16, 256),  # D = 256
])
def test_auto_matches_oracle(lens, hq, hkv, bs, D):
    p = make_problem("auto", len(lens), hq, hkv, D, lens, seed=900 + sum(lens), block_size=bs)
    d = p.to("cuda")
    ws = gq.Workspace(d.q.device)
    out = gq.gqa_decode_auto(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens,
                             p.seq_lens.to(torch.int32).contiguous(), scale=p.scale, workspace=ws)
    assert ws.status() == 0
    ref = oracle.gqa_decode(p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, p.scale)
    parity(out.cpu(), ref, str(lens[:4]))
