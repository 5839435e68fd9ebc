"""Checks that pin the fp64 oracle to facts fixed outside itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError when
the oracle disagrees with:
  * a closed form (one key, two keys, identical keys, zero query, a dominant key),
  * a library routine (torch's scaled_dot_product_attention in float64, numpy in
    extended precision),
  * an algebraic invariant (paging permutation, power-of-two rescaling, exact
    split-and-merge in any order, head mapping),
  * or a worked example printed on the pages (tests/golden/).
They are plain functions so that the mutation test can run the same checks on
deliberately broken copies of the oracle.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F
from scipy.special import logsumexp

from workloads import make_problem

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a bf16 tensor."""
    return t.to(torch.float64).numpy()


def _decode(o, p, **kw):
    return o.gqa_decode(p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, p.scale, **kw)


def _kv_rows(p, b, kvh):
    """Logical K and V rows [L, D] of (b, kvh), gathered through the block table."""
    L = int(p.seq_lens[b])
    if p.block_table is None:
        return p.k_cache[b, kvh, :L], p.v_cache[b, kvh, :L]
    t = torch.arange(L)
    blk = p.block_table[b, t // p.block_size].long()
    return p.k_cache[blk, kvh, t % p.block_size], p.v_cache[blk, kvh, t % p.block_size]


# --------------------------------------------------------------------------- closed forms

def pin_single_key(o):
    """softmax of one score is 1: the output is that key's value row, exactly."""
    p = make_problem("one_key", 2, 4, 2, 16, [1, 1], seed=11)
    out = _decode(o, p)
    for b in range(2):
        for h in range(4):
            assert np.array_equal(out[b, h], f64(p.v_cache[b, h // 2, 0]))


def pin_identical_keys_mean(o):
    """All scores equal: uniform weights, so the output is the mean value row."""
    p = make_problem("same_keys", 1, 2, 1, 8, [13], seed=12)
    p.k_cache[0, 0, :13] = p.k_cache[0, 0, 0]
    out = _decode(o, p)
    mean = f64(p.v_cache[0, 0, :13]).mean(axis=0)
    for h in range(2):
        assert np.allclose(out[0, h], mean, rtol=0, atol=1e-12)


def pin_zero_query_mean(o):
    """q = 0 gives all-zero scores, hence the mean value row."""
    p = make_problem("zero_q", 2, 2, 2, 8, [7, 20], seed=13)
    p.q.zero_()
    out = _decode(o, p)
    for b, L in enumerate([7, 20]):
        for h in range(2):
            mean = f64(p.v_cache[b, h, :L]).mean(axis=0)
            assert np.allclose(out[b, h], mean, rtol=0, atol=1e-12)


def pin_two_keys_logistic(o):
    """Two keys: weights are the logistic function of the score difference."""
    p = make_problem("two_keys", 1, 1, 1, 8, [2], seed=14, scale=0.5)
    p.q.zero_()
    p.q[0, 0, 0] = 2.0                       # s_t = 0.5 * 2 * k_t[0] = k_t[0]
    p.k_cache[0, 0, 0, 0] = 1.25
    p.k_cache[0, 0, 1, 0] = -0.75            # s0 - s1 = 2
    out = _decode(o, p)
    v0, v1 = f64(p.v_cache[0, 0, 0]), f64(p.v_cache[0, 0, 1])
    w0 = 1.0 / (1.0 + math.exp(-2.0))
    w1 = 1.0 / (1.0 + math.exp(2.0))
    assert np.allclose(out[0, 0], w0 * v0 + w1 * v1, rtol=0, atol=1e-14)


def pin_dominant_key(o):
    """A key whose score exceeds all others by ~1000 takes all the weight, with no
    overflow: the output is exactly its value row."""
    p = make_problem("dominant", 1, 2, 1, 8, [50], seed=15, scale=1.0)
    p.q.zero_()
    p.q[0, :, 0] = 1.0
    p.k_cache[0, 0, :50, 0] = p.k_cache[0, 0, :50, 0].clamp(-4, 4)
    p.k_cache[0, 0, 17, 0] = 1024.0
    out = _decode(o, p)
    for h in range(2):
        assert np.array_equal(out[0, h], f64(p.v_cache[0, 0, 17]))


def pin_zero_length(o):
    """Empty context: the convention is a zero row (the pages define no output)."""
    p = make_problem("empty", 2, 2, 1, 8, [0, 3], seed=16)
    out = _decode(o, p)
    assert np.array_equal(out[0], np.zeros((2, 8)))
    assert np.all(np.isfinite(out[1])) and np.any(out[1] != 0)


# --------------------------------------------------------------------------- library routines

def pin_brute_force_extended(o):
    """Tiny shapes against a full score matrix, softmax and matmul in numpy
    extended precision (np.longdouble)."""
    for (B, Hq, Hkv, D, lens, bs) in [(2, 4, 2, 8, [5, 3], None), (1, 3, 1, 4, [4], 2),
                                      (2, 2, 2, 6, [1, 5], 2)]:
        p = make_problem("brute", B, Hq, Hkv, D, lens, seed=17 + D, block_size=bs)
        out = _decode(o, p)
        G = Hq // Hkv
        for b in range(B):
            for h in range(Hq):
                K, V = _kv_rows(p, b, h // G)
                qv = f64(p.q[b, h]).astype(np.longdouble)
                S = (f64(K).astype(np.longdouble) @ qv) * np.longdouble(p.scale)
                P = np.exp(S - S.max())
                P = P / P.sum()
                ref = P @ f64(V).astype(np.longdouble)
                assert np.allclose(out[b, h], ref.astype(np.float64), rtol=1e-13, atol=1e-15)


def pin_torch_sdpa(o):
    """Against torch.nn.functional.scaled_dot_product_attention in float64, with KV
    heads repeated G times (query head h reads KV head h // G)."""
    lens = [37, 1, 64]
    p = make_problem("sdpa", 3, 8, 2, 32, lens, seed=18, block_size=8, spare_blocks=3)
    out = _decode(o, p)
    G = p.G
    for b, L in enumerate(lens):
        K = torch.stack([_kv_rows(p, b, j)[0] for j in range(p.Hkv)]).double()   # [Hkv, L, D]
        V = torch.stack([_kv_rows(p, b, j)[1] for j in range(p.Hkv)]).double()
        K = K.repeat_interleave(G, dim=0)[None]
        V = V.repeat_interleave(G, dim=0)[None]
        qd = p.q[b].double()[None, :, None, :]                                # [1, Hq, 1, D]
        ref = F.scaled_dot_product_attention(qd, K, V, scale=p.scale)[0, :, 0].numpy()
        assert np.allclose(out[b], ref, rtol=1e-12, atol=1e-13)


def pin_logsumexp(o):
    """The merged log-normaliser equals scipy's logsumexp of the scores."""
    p = make_problem("lse", 1, 2, 1, 16, [40], seed=19)
    acc, m, l = o.gqa_decode_states(p.q, p.k_cache, p.v_cache, None, [0], [40], p.scale)
    _, lse = o.merge_states(acc.reshape(1, 2, 16), m.reshape(1, 2), l.reshape(1, 2))
    K = f64(p.k_cache[0, 0, :40])
    for h in range(2):
        s = (K @ f64(p.q[0, h])) * p.scale
        assert abs(lse[h] - logsumexp(s)) < 1e-12


# --------------------------------------------------------------------------- invariants

def pin_head_mapping(o):
    """Query head h reads KV head h // G: with every value row of KV head j equal to
    j + 1, head h returns exactly h // G + 1."""
    Hq, Hkv = 8, 2
    p = make_problem("heads", 1, Hq, Hkv, 8, [9], seed=20)
    for j in range(Hkv):
        p.v_cache[0, j, :9] = float(j + 1)
    out = _decode(o, p)
    for h in range(Hq):
        assert np.array_equal(out[0, h], np.full(8, float(h // (Hq // Hkv) + 1)))


def pin_mha_and_mqa(o):
    """G = 1 (MHA) and Hkv = 1 (MQA) reduce to single-head attention per head."""
    for Hq, Hkv in [(4, 4), (4, 1)]:
        p = make_problem("mha_mqa", 1, Hq, Hkv, 8, [11], seed=21 + Hkv)
        out = _decode(o, p)
        for h in range(Hq):
            K, V = _kv_rows(p, 0, h if Hkv == Hq else 0)
            s = (f64(K) @ f64(p.q[0, h])) * p.scale
            w = np.exp(s - s.max())
            ref = (w / w.sum()) @ f64(V)
            assert np.allclose(out[0, h], ref, rtol=1e-12, atol=1e-14)


def pin_scale_invariance(o):
    """K * 2 with scale / 2 gives bit-identical scores, hence identical output."""
    p = make_problem("scale", 2, 4, 2, 16, [9, 30], seed=23)
    a = _decode(o, p)
    p.k_cache.mul_(2.0)
    p.scale = p.scale / 2.0
    b = _decode(o, p)
    assert np.array_equal(a, b)


def pin_paging_invariance(o):
    """Renaming physical blocks (permuting the pool and the table together) leaves the
    result bit-identical; a contiguous copy of the same rows agrees too."""
    lens = [21, 8, 3]
    p = make_problem("paged", 3, 4, 2, 8, lens, seed=24, block_size=4, spare_blocks=2)
    a = _decode(o, p)
    perm = torch.randperm(p.num_blocks, generator=torch.Generator().manual_seed(5))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(p.num_blocks)
    p2 = make_problem("paged", 3, 4, 2, 8, lens, seed=24, block_size=4, spare_blocks=2)
    p2.k_cache = p.k_cache[inv].clone()          # new block i holds old block inv[i]
    p2.v_cache = p.v_cache[inv].clone()
    bt = p.block_table.clone()
    valid = bt >= 0
    bt[valid] = perm[bt[valid].long()].to(torch.int32)
    p2.block_table = bt
    b = _decode(o, p2)
    assert np.array_equal(a, b)
    # Contiguous layout with the same logical rows.
    cap = max(lens)
    kc = torch.full((3, 2, cap, 8), float("nan"), dtype=torch.bfloat16)
    vc = kc.clone()
    for bi, L in enumerate(lens):
        for j in range(2):
            K, V = _kv_rows(p, bi, j)
            kc[bi, j, :L], vc[bi, j, :L] = K, V
    c = o.gqa_decode(p.q, kc, vc, None, p.seq_lens, p.scale)
    assert np.array_equal(a, c)


def pin_split_merge(o):
    """Splitting the key range anywhere and merging the partial states in any order
    reproduces the unsplit output (2-way, N-way, uneven, empty pieces, reversed)."""
    L = 97
    p = make_problem("split", 1, 4, 2, 16, [L], seed=25, block_size=8)
    full = _decode(o, p)[0]
    for cuts in ([48], [10, 20, 30, 40, 50, 60, 70, 80], [1, 2, 39], [0, 0, 50, 97]):
        edges = [0] + cuts + [L]
        pieces = [o.gqa_decode_states(p.q, p.k_cache, p.v_cache, p.block_table, [a], [b], p.scale)
                  for a, b in zip(edges[:-1], edges[1:])]
        for order in (list(range(len(pieces))), list(reversed(range(len(pieces))))):
            acc = np.stack([pieces[i][0][0] for i in order])
            m = np.stack([pieces[i][1][0] for i in order])
            l = np.stack([pieces[i][2][0] for i in order])
            merged, _ = o.merge_states(acc, m, l)
            assert np.allclose(merged, full, rtol=1e-12, atol=1e-14)


def pin_merge_empty(o):
    """An empty piece (m = -inf, l = 0) has weight zero; all-empty gives 0, lse -inf."""
    rng = np.random.default_rng(0)
    acc = rng.standard_normal((1, 3, 4))
    m = rng.standard_normal((1, 3))
    l = rng.random((1, 3)) + 0.5
    one, lse1 = o.merge_states(acc, m, l)
    acc2 = np.concatenate([acc, np.zeros((1, 3, 4))])
    m2 = np.concatenate([m, np.full((1, 3), -np.inf)])
    l2 = np.concatenate([l, np.zeros((1, 3))])
    two, lse2 = o.merge_states(acc2, m2, l2)
    assert np.array_equal(one, two) and np.array_equal(lse1, lse2)
    assert np.allclose(one, acc[0] / l[0][:, None], rtol=1e-15, atol=0)
    z, lz = o.merge_states(np.zeros((2, 1, 4)), np.full((2, 1), -np.inf), np.zeros((2, 1)))
    assert np.array_equal(z, np.zeros((1, 4))) and lz[0] == -np.inf


# --------------------------------------------------------------------------- worked examples

def pin_fig_6_13(o):
    """The PagedAttention figure: blocks 7, 1, 3 of 4 tokens, the last holding 2.
    Every other block of the pool is poisoned with NaN; the result is finite and
    bit-identical to the same rows stored contiguously."""
    g = json.load(open(os.path.join(GOLDEN, "paged_fig6_13.json")))
    bs, table, L = g["block_size"], g["block_table"], g["seq_len"]
    assert sum(g["tokens_per_block"]) == L and len(table) == math.ceil(L / bs)
    pool = max(table) + 1
    D, Hq, Hkv = 8, 2, 1
    gen = torch.Generator().manual_seed(26)
    q = torch.randn((1, Hq, D), generator=gen).to(torch.bfloat16)
    kc = torch.full((pool, Hkv, bs, D), float("nan"), dtype=torch.bfloat16)
    vc = kc.clone()
    krows = torch.randn((L, D), generator=gen).to(torch.bfloat16)
    vrows = torch.randn((L, D), generator=gen).to(torch.bfloat16)
    for t in range(L):
        kc[table[t // bs], 0, t % bs] = krows[t]
        vc[table[t // bs], 0, t % bs] = vrows[t]
    bt = torch.tensor([table], dtype=torch.int32)
    lens = torch.tensor([L], dtype=torch.int32)
    scale = 1.0 / math.sqrt(D)
    paged = o.gqa_decode(q, kc, vc, bt, lens, scale)
    contig = o.gqa_decode(q, krows[None, None], vrows[None, None], None, lens, scale)
    assert np.all(np.isfinite(paged))
    assert np.array_equal(paged, contig)


def pin_bad_block_rejected(o):
    """A block id outside the pool is an error, never a read."""
    p = make_problem("bad", 1, 2, 1, 8, [9], seed=27, block_size=4)
    p.block_table[0, 1] = p.num_blocks
    try:
        _decode(o, p)
    except RuntimeError:
        return
    raise AssertionError("out-of-pool block id was accepted")


# --------------------------------------------------------------------------- several query tokens

def _multi_problem(B, Q, Hq, Hkv, D, lens, seed, bs):
    """A problem with Q query tokens per request: q [B, Q, Hq, D]."""
    p = make_problem("multi", B, Q * Hq, Hkv, D, lens, seed=seed, block_size=bs)
    return p, p.q.reshape(B, Q, Hq, D).contiguous()


MULTI_CASES = [(2, 3, 4, 2, 8, [9, 5], 4), (1, 4, 2, 1, 6, [4], None), (2, 2, 6, 3, 4, [3, 7], 2)]


def pin_multi_brute_force(o):
    """Speculative verification (Inference optimization ..., section 5): query token
    i of Q sits at position L - Q + i and sees keys t <= L - Q + i.  Checked against
    the full score matrix with an explicit causal mask, softmax and matmul in numpy
    extended precision."""
    for (B, Q, Hq, Hkv, D, lens, bs) in MULTI_CASES:
        p, q = _multi_problem(B, Q, Hq, Hkv, D, lens, 31 + D, bs)
        out = o.gqa_decode_multi(q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, p.scale)
        G = Hq // Hkv
        for b in range(B):
            L = int(p.seq_lens[b])
            for h in range(Hq):
                K, V = _kv_rows(p, b, h // G)
                Kl, Vl = f64(K).astype(np.longdouble), f64(V).astype(np.longdouble)
                for i in range(Q):
                    S = (Kl @ f64(q[b, i, h]).astype(np.longdouble)) * np.longdouble(p.scale)
                    S[np.arange(L) > L - Q + i] = -np.inf
                    P = np.exp(S - S.max())
                    ref = (P / P.sum()) @ Vl
                    assert np.allclose(out[b, i, h], ref.astype(np.float64), rtol=1e-13, atol=1e-15)


def pin_multi_query_prefix(o):
    """Query token i sees exactly what a single-query decode of the request cut to
    L - Q + i + 1 tokens sees; the last token sees the whole request."""
    for (B, Q, Hq, Hkv, D, lens, bs) in MULTI_CASES:
        p, q = _multi_problem(B, Q, Hq, Hkv, D, lens, 57 + D, bs)
        out = o.gqa_decode_multi(q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, p.scale)
        for i in range(Q):
            lens_i = (p.seq_lens - Q + i + 1).to(torch.int32)
            ref = o.gqa_decode(q[:, i].contiguous(), p.k_cache, p.v_cache, p.block_table, lens_i,
                               p.scale)
            assert np.allclose(out[:, i], ref, rtol=1e-13, atol=1e-15)


def pin_multi_too_short_rejected(o):
    """A request shorter than its Q query tokens is an error, not a guess."""
    p, q = _multi_problem(1, 3, 2, 1, 4, [2], 5, None)
    try:
        o.gqa_decode_multi(q, p.k_cache, p.v_cache, None, p.seq_lens, p.scale)
    except RuntimeError:
        return
    raise AssertionError("L < Q accepted")


# --------------------------------------------------------------------------- FP8 E4M3 cache

def pin_e4m3_widening(o):
    """All 256 FP8 E4M3 codes widen exactly as torch's float8_e4m3fn does."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([o.e4m3_to_double(c) for c in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(got[fin], ref[fin])


def pin_fp8_equals_dequantized_bf16(o):
    """An FP8 cache with power-of-two scales gives exactly the result of the bf16
    oracle on the dequantized cache (every e4m3 value times 2^k is a bf16 value)."""
    for (B, Hq, Hkv, D, lens, bs, ks, vs) in [(2, 8, 2, 16, [37, 5], 4, 0.25, 2.0),
                                              (1, 4, 1, 8, [20], None, 1.0, 0.5)]:
        p = make_problem("fp8", B, Hq, Hkv, D, lens, seed=41 + D, block_size=bs)
        gen = torch.Generator().manual_seed(99 + D)
        k8 = torch.randint(0, 256, p.k_cache.shape, generator=gen, dtype=torch.int32).to(torch.uint8)
        v8 = torch.randint(0, 256, p.v_cache.shape, generator=gen, dtype=torch.int32).to(torch.uint8)
        k8[(k8 & 0x7F) == 0x7F] -= 1   # no NaN codes
        v8[(v8 & 0x7F) == 0x7F] -= 1
        kd = (k8.view(torch.float8_e4m3fn).to(torch.float64) * ks).to(torch.bfloat16)
        vd = (v8.view(torch.float8_e4m3fn).to(torch.float64) * vs).to(torch.bfloat16)
        assert torch.equal(kd.to(torch.float64), k8.view(torch.float8_e4m3fn).to(torch.float64) * ks)
        got = o.gqa_decode_fp8(p.q, k8, v8, ks, vs, p.block_table, p.seq_lens, p.scale)
        ref = o.gqa_decode(p.q, kd, vd, p.block_table, p.seq_lens, p.scale)
        assert np.array_equal(got, ref)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
