"""GPU parity of several query tokens per request (gqa_decode_multi, the
speculative-verification pass) against the fp64 oracle."""
import pytest
import torch

import gqa_decode_attention_attn_b200 as gq
import oracle
from gpu_util import parity
from workloads import make_problem

pytestmark = pytest.mark.gpu

CASES = [
    # B, Q, Hq, Hkv, lens, block_size
    (3, 2, 32, 8, [1000, 2, 300], None),        # G = 4: 8 query rows per KV head
    (2, 4, 32, 8, [5000, 129], 16),             # 16 rows: one full MMA chunk
    (2, 3, 16, 16, [700, 3], 32),               # MHA: 3 rows (R = 3 < 4: not supported)
    (2, 4, 8, 8, [900, 4], 64),                 # MHA with 4 tokens: R = 4
    (2, 2, 32, 2, [40000, 777], 64),            # G = 16: 32 rows, two chunks; long: split segments
    (1, 5, 24, 8, [100000], None),              # G = 3, 15 rows; one long segment over every CTA
    (4, 3, 16, 4, [3, 130, 128, 1], 8),         # a request shorter than Q -> error row
    (2, 2, 16, 2, [6000, 301], 16, 64),         # D = 64: 16 rows per KV head
]


def _problem(B, Q, Hq, Hkv, lens, bs, seed, D=128):
    p = make_problem("multi", B, Q * Hq, Hkv, D, lens, seed=seed, block_size=bs,
                     key_outlier_frac=0.01)
    return p, p.q.reshape(B, Q, Hq, D).contiguous()


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}_Q{c[1]}_Hq{c[2]}_Hkv{c[3]}_bs{c[5]}")
def test_multi_matches_oracle(case):
    B, Q, Hq, Hkv, lens, bs, *rest = case
    D = rest[0] if rest else 128
    p, q = _problem(B, Q, Hq, Hkv, lens, bs, 1200 + sum(lens) + Q, D)
    d = p.to("cuda")
    qd = q.cuda()
    ws = gq.Workspace(qd.device)
    if Q * Hq // Hkv < 4:
        with pytest.raises(gq.GqaError):
            gq.gqa_decode_multi(qd, d.k_cache, d.v_cache, d.block_table, d.seq_lens,
                                scale=p.scale, workspace=ws)
        return
    out = gq.gqa_decode_multi(qd, d.k_cache, d.v_cache, d.block_table, d.seq_lens, scale=p.scale,
                              workspace=ws)
    status = ws.status()
    short = [b for b in range(B) if lens[b] < Q]
    if short:
        assert status & gq.DEV_BAD_LENGTH
        o = out.float().cpu()
        for b in short:
            assert torch.isnan(o[b]).all()
        keep = [b for b in range(B) if lens[b] >= Q]
        sub = make_problem("multi", B, Q * Hq, Hkv, D, lens, seed=1200 + sum(lens) + Q,
                           block_size=bs, key_outlier_frac=0.01)
        lens_ok = sub.seq_lens.clone()
        for b in short:
            lens_ok[b] = Q  # any valid length: only the other rows are compared
        ref = oracle.gqa_decode_multi(q, p.k_cache, p.v_cache, p.block_table, lens_ok, p.scale)
        parity(o[keep], ref[keep], str(case), bf16_scaled=True)
        return
    assert status == 0
    ref = oracle.gqa_decode_multi(q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, p.scale)
    parity(out.cpu(), ref, str(case), bf16_scaled=True)


def test_multi_with_one_token_is_decode():
    p = make_problem("multi1", 3, 32, 8, 128, [700, 1, 2000], seed=77, block_size=16)
    d = p.to("cuda")
    a = gq.gqa_decode_multi(d.q.unsqueeze(1).contiguous(), d.k_cache, d.v_cache, d.block_table,
                            d.seq_lens, scale=p.scale)
    b = gq.gqa_decode(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens, scale=p.scale)
    assert torch.equal(a[:, 0], b)
