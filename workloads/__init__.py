"""Seeded synthetic decode-attention inputs, shared by the tests, the bench and
the smoke check.

This module holds input generation only -- shapes, random values, block-table
structure, poisoning of slots that must never be read -- and none of the
attention arithmetic.  Both the fp64 oracle and the CUDA path receive the
tensors built here.

Recipe (all on the host, with ``torch.Generator`` seeded per problem):

* values: q, then the K pool, then the V pool, each i.i.d. N(0, 1) drawn in
  float32 and rounded to bf16 (round to nearest even);
* structure (lengths, key outliers, block shuffle) from a second generator
  seeded with ``seed + 7919``;
* key outliers (the Llama-3-8B-shaped step): each (request, kv head, token) key
  row is multiplied by 8 with probability 1% -- a power of two, so exact in bf16;
* paged caches: each request needs ceil(L_b / block_size) blocks; all needed
  blocks (plus optional spares) get a seeded random permutation of physical ids;
  unused block-table entries hold -1;
* poisoning: slots past a request's length inside its last block, and every
  spare block, hold bf16 NaN (0x7FC0), so any read of them shows up as NaN.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Sequence

import torch

BF16_NAN_BITS = 0x7FC0
_STRUCT_SALT = 7919


@dataclass
class Problem:
    """One decode-attention call: q [B, Hq, D]; caches [num_blocks, Hkv, block_size, D]."""
    name: str
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    block_table: Optional[torch.Tensor]
    seq_lens: torch.Tensor
    scale: float
    meta: dict = field(default_factory=dict)

    @property
    def B(self) -> int:
        return self.q.shape[0]

    @property
    def Hq(self) -> int:
        return self.q.shape[1]

    @property
    def D(self) -> int:
        return self.q.shape[2]

    @property
    def Hkv(self) -> int:
        return self.k_cache.shape[1]

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def block_size(self) -> int:
        return self.k_cache.shape[2]

    @property
    def num_blocks(self) -> int:
        return self.k_cache.shape[0]

    @property
    def max_blocks(self) -> int:
        return 0 if self.block_table is None else self.block_table.shape[1]

    @property
    def paged(self) -> bool:
        return self.block_table is not None

    def total_tokens(self) -> int:
        return int(self.seq_lens.to(torch.int64).sum())

    def algorithmic_bytes(self) -> int:
        """K + V rows of valid tokens (bf16, or one byte per element for an FP8 cache),
        plus q read and out written (bf16)."""
        eb = int(self.meta.get("kv_elem_bytes", 2))
        return kv_bytes(self.seq_lens, self.Hkv, self.D, eb) + 2 * 2 * self.B * self.Hq * self.D

    def block_table_bytes(self) -> int:
        if self.block_table is None:
            return 0
        return 4 * sum(math.ceil(int(L) / self.block_size) for L in self.seq_lens.tolist())

    def to(self, device) -> "Problem":
        bt = None if self.block_table is None else self.block_table.to(device)
        return Problem(self.name, self.q.to(device), self.k_cache.to(device),
                       self.v_cache.to(device), bt, self.seq_lens.to(device), self.scale,
                       dict(self.meta))


def kv_bytes(seq_lens, Hkv: int, D: int, elem_bytes: int = 2) -> int:
    """Bytes of K and V read for one layer: 2 (K, V) * Hkv * D * elem_bytes per token."""
    total = int(torch.as_tensor(seq_lens).to(torch.int64).sum())
    return 2 * Hkv * D * elem_bytes * total


def kv_cache_bytes_per_token(layers: int, kv_heads: int, head_dim: int, elem_bytes: int) -> int:
    """Whole-model KV-cache bytes per token: 2 (K and V) * layers * kv_heads * head_dim * bytes."""
    return 2 * layers * kv_heads * head_dim * elem_bytes


def _normal_bf16(gen: torch.Generator, shape, chunk_rows: int = 1 << 14) -> torch.Tensor:
    """i.i.d. N(0,1) rounded to bf16, drawn in chunks along dim 0 to bound host memory."""
    out = torch.empty(shape, dtype=torch.bfloat16)
    if out.numel() == 0:
        return out
    n0 = shape[0]
    per_row = out[0].numel() if n0 else 0
    step = max(1, (chunk_rows * 4096) // max(per_row, 1))
    for i in range(0, n0, step):
        j = min(n0, i + step)
        out[i:j] = torch.randn((j - i,) + tuple(shape[1:]), generator=gen,
                               dtype=torch.float32).to(torch.bfloat16)
    return out


def _poison_(t: torch.Tensor) -> None:
    t.view(torch.int16).fill_(BF16_NAN_BITS)


def make_problem(name: str, B: int, Hq: int, Hkv: int, D: int, seq_lens: Sequence[int],
                 seed: int, block_size: Optional[int] = None, capacity: Optional[int] = None,
                 key_outlier_frac: float = 0.0, key_outlier_scale: float = 8.0,
                 spare_blocks: int = 0, max_blocks: Optional[int] = None,
                 shuffle: bool = True, scale: Optional[float] = None) -> Problem:
    """Build one seeded problem on the host.

    block_size=None gives a contiguous cache [B, Hkv, capacity, D] (capacity
    defaults to max(seq_lens)); otherwise a paged pool of block_size-token blocks.
    """
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    lens = [int(x) for x in seq_lens]
    if len(lens) != B:
        raise ValueError("need one length per request")
    gen = torch.Generator().manual_seed(seed)
    sgen = torch.Generator().manual_seed(seed + _STRUCT_SALT)
    q = _normal_bf16(gen, (B, Hq, D))

    if block_size is None:
        cap = max(lens + [1]) if capacity is None else capacity
        if max(lens + [0]) > cap:
            raise ValueError("a length exceeds the capacity")
        k = _normal_bf16(gen, (B, Hkv, cap, D))
        v = _normal_bf16(gen, (B, Hkv, cap, D))
        for b, L in enumerate(lens):
            if L < cap:
                _poison_(k[b, :, L:])
                _poison_(v[b, :, L:])
        table = None
        bs = cap
    else:
        bs = block_size
        need = [math.ceil(L / bs) for L in lens]
        total = sum(need) + spare_blocks
        mb = max(need + [1]) if max_blocks is None else max_blocks
        if max(need + [0]) > mb:
            raise ValueError("max_blocks too small for a length")
        k = _normal_bf16(gen, (total, Hkv, bs, D))
        v = _normal_bf16(gen, (total, Hkv, bs, D))
        ids = torch.randperm(total, generator=sgen) if shuffle else torch.arange(total)
        table = torch.full((B, mb), -1, dtype=torch.int32)
        used = torch.zeros(total, dtype=torch.bool)
        pos = 0
        for b, (L, n) in enumerate(zip(lens, need)):
            blocks = ids[pos:pos + n]
            pos += n
            table[b, :n] = blocks.to(torch.int32)
            used[blocks] = True
            if n and L % bs:
                last = int(blocks[-1])
                _poison_(k[last, :, L % bs:])
                _poison_(v[last, :, L % bs:])
        for blk in torch.nonzero(~used).flatten().tolist():
            _poison_(k[blk])
            _poison_(v[blk])

    if key_outlier_frac > 0:
        # One Bernoulli draw per (request, kv head, token) key row.
        for b, L in enumerate(lens):
            hit = torch.rand((Hkv, L), generator=sgen) < key_outlier_frac
            kvh_idx, t_idx = torch.nonzero(hit, as_tuple=True)
            if table is None:
                blk, off = torch.full_like(t_idx, b), t_idx
            else:
                blk, off = table[b, t_idx // bs].long(), t_idx % bs
            rows = k[blk, kvh_idx, off].float() * key_outlier_scale
            k[blk, kvh_idx, off] = rows.to(torch.bfloat16)

    sc = float(torch.tensor(1.0 / math.sqrt(D), dtype=torch.float32)) if scale is None else scale
    meta = dict(seed=seed, key_outlier_frac=key_outlier_frac, spare_blocks=spare_blocks)
    return Problem(name, q, k, v, table, torch.tensor(lens, dtype=torch.int32), sc, meta)


# ---------------------------------------------------------------------------
# The five workloads (shapes and structure as stated for this hot path).
# ---------------------------------------------------------------------------

SWEEP = [(32, 32, 128), (32, 8, 128), (64, 4, 128), (64, 1, 128), (32, 8, 64), (16, 4, 256)]


def varlen_lengths(B: int, seed: int, lo: int = 1024, hi: int = 131072):
    """Per-request lengths floor(exp(U[ln lo, ln hi])), clamped to [lo, hi]."""
    sgen = torch.Generator().manual_seed(seed + _STRUCT_SALT)
    u = torch.rand(B, generator=sgen, dtype=torch.float64)
    L = torch.floor(torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo))))
    return [int(x) for x in L.clamp(lo, hi).tolist()]


def fp8_caches(p: Problem):
    """The problem's caches stored as FP8 E4M3 with one scale per tensor (the largest
    finite magnitude maps to 448, E4M3's largest finite value): returns (k8, v8,
    k_scale, v_scale), k8/v8 uint8 in the bf16 caches' layouts.  Poisoned slots
    stay NaN (E4M3 0x7F)."""
    out = []
    for c in (p.k_cache, p.v_cache):
        f = c.to(torch.float32)
        fin = f[torch.isfinite(f)]
        amax = float(fin.abs().max()) if fin.numel() else 1.0
        sc = amax / 448.0 if amax > 0 else 1.0
        out.append(((f / sc).to(torch.float8_e4m3fn).view(torch.uint8), sc))
    return out[0][0], out[1][0], out[0][1], out[1][1]


WORKLOADS = {
    "tiny": "B=1, Hq=4, Hkv=1, D=128, L=512, contiguous",
    "llama3_8b": "B=16, Hq=32, Hkv=8, D=128, L=8192, contiguous, 1% of keys x8",
    "long_256k": "B=1, Hq=32, Hkv=2, D=128, L=262144, 64-token pages, permuted table",
    "varlen_paged": "B=64, Hq=32, Hkv=8, D=128, L log-uniform [1024, 131072], 16-token pages",
}
WORKLOADS["llama3_8b_fp8"] = "llama3_8b's shape and values, K/V stored as FP8 E4M3"
for _i, (_hq, _hkv, _d) in enumerate(SWEEP):
    WORKLOADS[f"sweep_{_hq}_{_hkv}_{_d}"] = f"B=8, Hq={_hq}, Hkv={_hkv}, D={_d}, L=32768, contiguous"


def workload(name: str) -> Problem:
    """The named full-size workload (host tensors)."""
    if name == "tiny":
        return make_problem(name, 1, 4, 1, 128, [512], seed=1000)
    if name == "llama3_8b":
        return make_problem(name, 16, 32, 8, 128, [8192] * 16, seed=1001, key_outlier_frac=0.01)
    if name == "llama3_8b_fp8":
        p = make_problem(name, 16, 32, 8, 128, [8192] * 16, seed=1001, key_outlier_frac=0.01)
        p.meta["kv_elem_bytes"] = 1
        return p
    if name == "long_256k":
        return make_problem(name, 1, 32, 2, 128, [262144], seed=1002, block_size=64)
    if name == "varlen_paged":
        return make_problem(name, 64, 32, 8, 128, varlen_lengths(64, 1003), seed=1003,
                            block_size=16)
    if name.startswith("sweep_"):
        hq, hkv, d = (int(x) for x in name.split("_")[1:])
        if (hq, hkv, d) not in SWEEP:
            raise KeyError(name)
        return make_problem(name, 8, hq, hkv, d, [32768] * 8, seed=1004 + SWEEP.index((hq, hkv, d)))
    raise KeyError(name)
