"""Seeded synthetic inputs for block-diffusion attention workloads.

This module is shared by the tests, the benchmark, the oracle checks and the
CUDA path's callers.  It only draws random numbers and lays them out; it holds
none of the attention arithmetic.

Recipe (all draws from one ``torch.Generator('cpu').manual_seed(seed)``):
  training/prefill form: q, k, v in that order, ``randn`` fp32 in
  [B, H, 2L, d] layout, keys multiplied by ``k_scale`` before the cast to
  bf16 (round to nearest even).
  block-decode form: cache lengths first (verify workload: ``randint(lo,
  hi + 1)``), then q_blk, then per batch element its K cache and V cache
  slices.  Each cache row beyond cache_len + b is zero; the block's own K/V
  sit at positions cache_len .. cache_len + b - 1 like every other row.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class FwdShape:
    name: str
    B: int
    Hq: int
    Hkv: int
    L: int
    b: int
    d: int
    k_scale: float = 1.0
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


@dataclass(frozen=True)
class DecodeShape:
    name: str
    B: int
    Hq: int
    Hkv: int
    b: int
    d: int
    mode: int  # 0 bidirectional inside the block, 1 causal
    len_lo: int
    len_hi: int  # cache lengths uniform in [len_lo, len_hi]
    seed: int = 0

    @property
    def S_cap(self) -> int:
        return self.len_hi + self.b

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


# The workloads: a tiny one the oracle finishes at once, the training shape,
# the long-context block-size sweep, and the two block-decode workloads.
FWD_TINY = FwdShape("fwd_tiny", 1, 2, 2, 64, 8, 32)
FWD_TRAIN = FwdShape("fwd_train", 4, 32, 8, 2048, 32, 128, k_scale=0.5)
FWD_LONG = {bb: FwdShape("fwd_long_b%d" % bb, 1, 32, 8, 8192, bb, 128)
            for bb in (4, 16, 64, 256)}
DEC_DENOISE = DecodeShape("decode_denoise", 16, 32, 8, 32, 128, 0, 8192, 8192)
DEC_VERIFY = DecodeShape("decode_verify", 64, 32, 8, 28, 128, 1, 512, 8192)


def fwd_inputs(B, Hq, Hkv, L, d, seed=0, k_scale=1.0):
    """q [B,Hq,2L,d], k, v [B,Hkv,2L,d] bf16 on the CPU."""
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn((B, Hq, 2 * L, d), generator=g, dtype=torch.float32)
    k = torch.randn((B, Hkv, 2 * L, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, Hkv, 2 * L, d), generator=g, dtype=torch.float32)
    if k_scale != 1.0:
        k = k * k_scale
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def fwd_inputs_for(s: FwdShape):
    return fwd_inputs(s.B, s.Hq, s.Hkv, s.L, s.d, seed=s.seed, k_scale=s.k_scale)


def decode_inputs(B, Hq, Hkv, b, d, S_cap, cache_len=None, len_range=None,
                  seed=0):
    """Returns (q_blk [B,Hq,b,d], k_cache, v_cache [B,Hkv,S_cap,d] bf16,
    cache_len int32 [B]) on the CPU.  Give either explicit ``cache_len`` or a
    ``len_range`` (lo, hi) to draw them uniformly (inclusive)."""
    g = torch.Generator("cpu").manual_seed(seed)
    if cache_len is None:
        lo, hi = len_range
        if lo == hi:
            lens = torch.full((B,), lo, dtype=torch.int32)
        else:
            lens = torch.randint(lo, hi + 1, (B,), generator=g,
                                 dtype=torch.int64).to(torch.int32)
    else:
        lens = torch.as_tensor(cache_len, dtype=torch.int32).reshape(B)
    assert int(lens.max()) + b <= S_cap
    q = torch.randn((B, Hq, b, d), generator=g, dtype=torch.float32)
    kc = torch.zeros((B, Hkv, S_cap, d), dtype=torch.bfloat16)
    vc = torch.zeros((B, Hkv, S_cap, d), dtype=torch.bfloat16)
    for i in range(B):
        n = int(lens[i]) + b
        kc[i, :, :n] = torch.randn((Hkv, n, d), generator=g,
                                   dtype=torch.float32).to(torch.bfloat16)
        vc[i, :, :n] = torch.randn((Hkv, n, d), generator=g,
                                   dtype=torch.float32).to(torch.bfloat16)
    return q.to(torch.bfloat16), kc, vc, lens


def decode_inputs_for(s: DecodeShape):
    return decode_inputs(s.B, s.Hq, s.Hkv, s.b, s.d, s.S_cap,
                         len_range=(s.len_lo, s.len_hi), seed=s.seed)


def fwd_sample_rows(B: int, H: int, L: int, b: int, n: int, heads: int = 8,
                    per_block: int = 16, seed: int = 1):
    """Flat row ids of a [B, H, 2L] forward output for a sampled parity check
    (sorted, unique): in ``heads`` seeded (batch, head) pairs -- the first and
    the last always among them -- rows of the first and the last block of
    each half (the whole block when b <= per_block, else ``per_block`` rows
    spread over it, its first and last row included), plus ``n`` uniform
    picks over the whole tensor."""
    g = torch.Generator("cpu").manual_seed(seed)
    nh = B * H
    if nh <= heads:
        hsel = torch.arange(nh)
    else:
        mid = torch.randperm(nh - 2, generator=g)[:heads - 2] + 1
        hsel = torch.cat([torch.tensor([0, nh - 1]), mid])
    if b <= per_block:
        inblk = torch.arange(b)
    else:
        inblk = torch.linspace(0, b - 1, per_block).round().long().unique()
    starts = torch.tensor([0, L - b, L, 2 * L - b])
    local = (starts[:, None] + inblk[None, :]).reshape(-1)
    forced = (hsel[:, None] * (2 * L) + local[None, :]).reshape(-1)
    pick = torch.randint(0, nh * 2 * L, (n,), generator=g)
    return torch.unique(torch.cat([pick, forced])).tolist()


def sample_rows(total_rows: int, block: int, n: int, seed: int = 1):
    """A seeded sample of flat row ids that always includes the first and
    last ``block`` rows plus ``n`` uniform picks (sorted, unique)."""
    g = torch.Generator("cpu").manual_seed(seed)
    pick = torch.randint(0, total_rows, (n,), generator=g)
    edge = torch.cat([torch.arange(0, min(block, total_rows)),
                      torch.arange(max(0, total_rows - block), total_rows)])
    return torch.unique(torch.cat([pick, edge])).tolist()
