"""KV-cache bookkeeping of block decoding: plain numpy definitions.

TEST INFRASTRUCTURE ONLY: the tests and ``__graft_entry__.smoke()`` are its
users.  The CUDA library never imports or calls it; the two share no code.

Linear speculative decoding ("Nemotron-Labs-Diffusion-8B-Base 3x decoding
speed-up", section 2 "Linear Speculative Decoding") drafts a block with
bidirectional attention, verifies it with causal attention over the same KV
cache ("Nemotron-Labs-Diffusion-3B", section "What it is"), accepts the
longest matching prefix and then updates the KV cache before generating on;
the same article's section "KV cache strategy" crops the cache to a maximum
length.  The three steps, on a cache laid out [B, Hkv, S_cap, d] whose
prefix length per sequence is cache_len[i]:

  accept_len  n[i] = length of the longest prefix of block positions j on
              which the draft token equals the verifier's token;
  append      rows 0 .. n[i]-1 of the block's K/V go to cache positions
              cache_len[i] .. cache_len[i] + n[i] - 1, then
              cache_len[i] += n[i];
  crop        cache_len[i] = min(cache_len[i], max_len).

Integer and byte work only: the results are exact.
"""
from __future__ import annotations

import numpy as np


def _arr(t):
    if isinstance(t, np.ndarray):
        return t
    return t.detach().cpu().numpy()


def accept_len(draft, target) -> np.ndarray:
    """draft, target: [B, b] integer tokens.  Returns int32 [B]."""
    draft, target = _arr(draft), _arr(target)
    B, b = draft.shape
    n = np.zeros(B, np.int32)
    for i in range(B):
        j = 0
        while j < b and draft[i, j] == target[i, j]:
            j += 1
        n[i] = j
    return n


def append(k_cache, v_cache, cache_len, k_new, v_new, n_new):
    """Returns (k_cache', v_cache', cache_len') after appending rows
    0 .. n_new[i]-1 of k_new / v_new [B, Hkv, b, d] to each sequence.
    Arrays may hold bf16 bit patterns (uint16/int16) or any dtype: rows are
    copied bit for bit.  Raises ValueError if a sequence would overflow."""
    kc = _arr(k_cache).copy()
    vc = _arr(v_cache).copy()
    lens = _arr(cache_len).astype(np.int64).copy()
    kn, vn, nn = _arr(k_new), _arr(v_new), _arr(n_new)
    B, Hkv, S_cap, d = kc.shape
    b = kn.shape[2]
    for i in range(B):
        n = int(nn[i])
        if n < 0 or n > b or lens[i] + n > S_cap:
            raise ValueError("append out of range for sequence %d" % i)
        kc[i, :, lens[i]:lens[i] + n] = kn[i, :, :n]
        vc[i, :, lens[i]:lens[i] + n] = vn[i, :, :n]
        lens[i] += n
    return kc, vc, lens.astype(np.int32)


def crop(cache_len, max_len: int) -> np.ndarray:
    lens = _arr(cache_len).astype(np.int64)
    return np.minimum(lens, int(max_len)).astype(np.int32)


def compact(k_cache, v_cache, kept, new_len):
    """Stable compaction for sparse prefix retention: the kept positions
    kept[i, :new_len[i]] (in increasing order) become positions
    0 .. new_len[i]-1 of the result; rows from new_len[i] on are zero."""
    kc, vc = _arr(k_cache), _arr(v_cache)
    ko = np.zeros_like(kc)
    vo = np.zeros_like(vc)
    for i in range(kc.shape[0]):
        n = int(new_len[i])
        idx = np.asarray(kept[i, :n], dtype=np.int64)
        ko[i, :, :n] = kc[i][:, idx]
        vo[i, :, :n] = vc[i][:, idx]
    return ko, vo
