"""Pins of the fp64 oracle to facts fixed outside the oracle itself.

Each ``pin_*`` function takes an oracle library handle (``oracle.load()`` or a
deliberately mutated copy) and raises AssertionError if the oracle disagrees
with: the hand-written mask fixtures in ``tests/golden/``, closed forms of the
definition, textbook attention computed by a library routine
(``torch.nn.functional.scaled_dot_product_attention`` / ``torch.logsumexp``
in fp64) in the special cases that reduce to it, or invariants of the
definition.  ``tests/test_oracle_pins.py`` runs them on the real oracle;
``tests/test_oracle_mutants.py`` checks that planted mistakes fail at least
one of them.
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch
import torch.nn.functional as F

import bd_inputs
import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
TIGHT = 1e-11


def read_mask_fixture(name):
    """Parse a golden mask file into a list of (header dict, 0/1 matrix)."""
    blocks = []
    cur = None
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if "=" in line:
                hdr = dict(kv.split("=") for kv in line.split())
                cur = ({k: int(v) for k, v in hdr.items()}, [])
                blocks.append(cur)
            else:
                cur[1].append([int(ch) for ch in line])
    return [(h, np.array(m, dtype=np.int64)) for h, m in blocks]


def _bf(x):
    return x.to(torch.bfloat16)


def _f64(t):
    return t.to(torch.float64)


def sdpa_out_lse(q, k, v, scale):
    """Textbook unmasked attention of q [n,d] over k, v [m,d] (fp64)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    out = F.scaled_dot_product_attention(q[None], k[None], v[None],
                                         scale=scale)[0]
    lse = torch.logsumexp(scale * (q @ k.T), dim=-1)
    return out, lse


# ----------------------------------------------------------------------------
# mask fixtures (hand-written from the pages)


def pin_fwd_mask_fixtures(lib):
    for name in ("fwd_mask_L4_b2.txt", "fwd_mask_L6_b3.txt",
                 "fwd_mask_L4_b1.txt", "fwd_mask_L4_b4.txt"):
        for hdr, m in read_mask_fixture(name):
            L, b = hdr["L"], hdr["b"]
            got = np.array([[lib.bdo_fwd_sees(L, b, r, c) for c in range(2 * L)]
                            for r in range(2 * L)])
            assert (got == m).all(), (name, got)


def pin_decode_mask_fixture(lib):
    for hdr, m in read_mask_fixture("decode_mask_len3_b2.txt"):
        n, b, S, mode = hdr["cache_len"], hdr["b"], hdr["S_cap"], hdr["mode"]
        got = np.array([[lib.bdo_decode_sees(n, b, mode, j, c)
                         for c in range(S)] for j in range(b)])
        assert (got == m).all(), (hdr, got)


def pin_visible_pair_count(lib):
    """Closed form: a (batch, head) slice has L^2 + L*b visible pairs
    (noisy row in block k: b + k*b keys; clean row: (k+1)*b keys)."""
    for L, b in ((64, 8), (12, 3), (16, 16), (10, 1), (30, 5)):
        n = sum(lib.bdo_fwd_sees(L, b, r, c)
                for r in range(2 * L) for c in range(2 * L))
        assert n == L * L + L * b, (L, b, n)
    assert sum(lib.bdo_fwd_sees(64, 8, r, c)
               for r in range(128) for c in range(128)) == 4608


# ----------------------------------------------------------------------------
# special cases that reduce to textbook attention (library routine)


def pin_b1_clean_half_is_causal(lib):
    L, d = 24, 16
    q, k, v = bd_inputs.fwd_inputs(1, 2, 2, L, d, seed=3)
    s = 1 / math.sqrt(d)
    out, lse = oracle.fwd(q, k, v, L, 1, s, lib=lib)
    for h in range(2):
        qq, kk, vv = _f64(q[0, h, L:]), _f64(k[0, h, L:]), _f64(v[0, h, L:])
        ref = F.scaled_dot_product_attention(qq[None], kk[None], vv[None],
                                             is_causal=True, scale=s)[0]
        np.testing.assert_allclose(out[0, h, L:], ref.numpy(), rtol=0,
                                   atol=TIGHT)
        sc = s * (qq @ kk.T)
        sc = sc.masked_fill(torch.ones(L, L).triu(1).bool(), -math.inf)
        np.testing.assert_allclose(lse[0, h, L:],
                                   torch.logsumexp(sc, -1).numpy(), rtol=0,
                                   atol=TIGHT)


def pin_b1_noisy_row_is_self_plus_earlier_clean(lib):
    L, d = 12, 8
    q, k, v = bd_inputs.fwd_inputs(1, 1, 1, L, d, seed=4)
    s = 1 / math.sqrt(d)
    out, lse = oracle.fwd(q, k, v, L, 1, s, lib=lib)
    for r in range(L):
        keys = torch.cat([k[0, 0, L:L + r], k[0, 0, r:r + 1]])
        vals = torch.cat([v[0, 0, L:L + r], v[0, 0, r:r + 1]])
        o, l_ = sdpa_out_lse(q[0, 0, r:r + 1], keys, vals, s)
        np.testing.assert_allclose(out[0, 0, r], o[0].numpy(), rtol=0,
                                   atol=TIGHT)
        np.testing.assert_allclose(lse[0, 0, r], l_[0].item(), rtol=0,
                                   atol=TIGHT)


def pin_bL_halves_are_bidirectional(lib):
    L, d = 16, 32
    q, k, v = bd_inputs.fwd_inputs(2, 2, 1, L, d, seed=5)
    s = 0.3
    out, lse = oracle.fwd(q, k, v, L, L, s, lib=lib)
    for bi in range(2):
        for h in range(2):
            for lo, hi in ((0, L), (L, 2 * L)):
                o, l_ = sdpa_out_lse(q[bi, h, lo:hi], k[bi, 0, lo:hi],
                                     v[bi, 0, lo:hi], s)
                np.testing.assert_allclose(out[bi, h, lo:hi], o.numpy(),
                                           rtol=0, atol=TIGHT)
                np.testing.assert_allclose(lse[bi, h, lo:hi], l_.numpy(),
                                           rtol=0, atol=TIGHT)


def pin_decode_causal_is_prefix_attention(lib):
    """Mode 1: block row j attends exactly to cache positions
    0 .. cache_len + j (textbook attention over that prefix)."""
    B, Hq, Hkv, b, d, S = 2, 4, 2, 5, 16, 40
    q, kc, vc, lens = bd_inputs.decode_inputs(B, Hq, Hkv, b, d, S,
                                              cache_len=[7, 30], seed=6)
    s = 1 / math.sqrt(d)
    out, lse = oracle.decode(q, kc, vc, lens, 1, s, lib=lib)
    for i in range(B):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            for j in range(b):
                n = int(lens[i]) + j + 1
                o, l_ = sdpa_out_lse(q[i, h, j:j + 1], kc[i, g, :n],
                                     vc[i, g, :n], s)
                np.testing.assert_allclose(out[i, h, j], o[0].numpy(),
                                           rtol=0, atol=TIGHT)
                np.testing.assert_allclose(lse[i, h, j], l_[0].item(),
                                           rtol=0, atol=TIGHT)


def pin_decode_bidirectional_is_full_attention(lib):
    """Mode 0: every block row attends to cache positions
    0 .. cache_len + b - 1; with cache_len = 0 this is full attention inside
    the block, and mode 1 then is textbook causal attention."""
    B, Hq, Hkv, b, d, S = 3, 2, 1, 6, 32, 24
    q, kc, vc, lens = bd_inputs.decode_inputs(B, Hq, Hkv, b, d, S,
                                              cache_len=[0, 1, 18], seed=7)
    s = 1 / math.sqrt(d)
    out, lse = oracle.decode(q, kc, vc, lens, 0, s, lib=lib)
    for i in range(B):
        n = int(lens[i]) + b
        for h in range(Hq):
            o, l_ = sdpa_out_lse(q[i, h], kc[i, 0, :n], vc[i, 0, :n], s)
            np.testing.assert_allclose(out[i, h], o.numpy(), rtol=0,
                                       atol=TIGHT)
            np.testing.assert_allclose(lse[i, h], l_.numpy(), rtol=0,
                                       atol=TIGHT)
    out1, _ = oracle.decode(q, kc, vc, lens, 1, s, lib=lib)
    for h in range(Hq):
        ref = F.scaled_dot_product_attention(
            _f64(q[0, h])[None], _f64(kc[0, 0, :b])[None],
            _f64(vc[0, 0, :b])[None], is_causal=True, scale=s)[0]
        np.testing.assert_allclose(out1[0, h], ref.numpy(), rtol=0,
                                   atol=TIGHT)


# ----------------------------------------------------------------------------
# closed forms


def pin_zero_query_closed_form(lib):
    """q = 0 makes every visible score equal: lse = ln(#visible) =
    ln((k+1) b) for a row of block k in either half, and out is the plain mean
    of the visible values (own noisy block + earlier clean blocks for a noisy
    row; clean blocks up to its own for a clean row)."""
    L, b, d = 24, 4, 8
    _, k, v = bd_inputs.fwd_inputs(1, 2, 1, L, d, seed=8)
    q = torch.zeros((1, 2, 2 * L, d), dtype=torch.bfloat16)
    out, lse = oracle.fwd(q, k, v, L, b, 0.7, lib=lib)
    vv = _f64(v[0, 0])
    for h in range(2):
        for r in range(2 * L):
            kb = (r if r < L else r - L) // b
            assert abs(lse[0, h, r] - math.log((kb + 1) * b)) < TIGHT, (h, r)
            if r < L:
                rows = torch.cat([vv[kb * b:(kb + 1) * b], vv[L:L + kb * b]])
            else:
                rows = vv[L:L + (kb + 1) * b]
            np.testing.assert_allclose(out[0, h, r], rows.mean(0).numpy(),
                                       rtol=0, atol=TIGHT)


def pin_unit_values_and_probs(lib):
    """Rows of the attention matrix sum to 1: v = 1 gives out = 1 exactly
    (to rounding), and the probability hook sums to 1 with zeros outside the
    visible set."""
    L, b, d = 16, 4, 16
    q, k, _ = bd_inputs.fwd_inputs(1, 2, 2, L, d, seed=9)
    ones = torch.ones((1, 2, 2 * L, d), dtype=torch.bfloat16)
    out, _ = oracle.fwd(q, k, ones, L, b, 0.25, lib=lib)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-13)
    for row in (0, 5, 17, 2 * L - 1, 2 * L + 3, 4 * L - 1):
        p = oracle.fwd_row_probs(q, k, L, b, 0.25, row, lib=lib)
        assert abs(p.sum() - 1.0) < 1e-13
        r = row % (2 * L)
        mask = np.array([lib.bdo_fwd_sees(L, b, r, c) for c in range(2 * L)])
        assert (p[mask == 0] == 0).all() and (p[mask == 1] > 0).all()


def pin_brute_force_tiny(lib):
    """The whole tiny workload against a dense masked softmax over the
    full 2L x 2L score matrix, with the mask taken from the hand-checked
    predicate (fixtures above) evaluated cell by cell in Python."""
    s = bd_inputs.FWD_TINY
    q, k, v = bd_inputs.fwd_inputs_for(s)
    out, lse = oracle.fwd(q, k, v, s.L, s.b, s.scale, lib=lib)
    N = 2 * s.L
    vis = np.zeros((N, N), bool)
    for r in range(N):
        for c in range(N):
            hr, hc = r >= s.L, c >= s.L
            br, bc = (r - hr * s.L) // s.b, (c - hc * s.L) // s.b
            vis[r, c] = ((not hr and not hc and br == bc)
                         or (not hr and hc and bc < br)
                         or (hr and hc and bc <= br))
    for h in range(s.Hq):
        g = h // (s.Hq // s.Hkv)
        sc = s.scale * (_f64(q[0, h]) @ _f64(k[0, g]).T).numpy()
        sc[~vis] = -np.inf
        m = sc.max(1, keepdims=True)
        p = np.exp(sc - m)
        z = p.sum(1, keepdims=True)
        np.testing.assert_allclose(out[0, h], (p / z) @ _f64(v[0, g]).numpy(),
                                   rtol=0, atol=TIGHT)
        np.testing.assert_allclose(lse[0, h], (m + np.log(z))[:, 0], rtol=0,
                                   atol=TIGHT)


# ----------------------------------------------------------------------------
# invariants


def pin_permutation_within_noisy_block(lib):
    """Permuting q/k/v rows inside one noisy block permutes that block's
    outputs the same way and leaves every other row unchanged."""
    L, b, d = 16, 4, 8
    q, k, v = bd_inputs.fwd_inputs(1, 2, 2, L, d, seed=10)
    s = 0.35
    out, lse = oracle.fwd(q, k, v, L, b, s, lib=lib)
    blk = 2
    perm = torch.tensor([3, 0, 2, 1]) + blk * b
    idx = torch.arange(2 * L)
    idx[blk * b:(blk + 1) * b] = perm
    out2, lse2 = oracle.fwd(q[:, :, idx], k[:, :, idx], v[:, :, idx], L, b, s,
                            lib=lib)
    np.testing.assert_allclose(out2, out[:, :, idx.numpy()], rtol=0,
                               atol=TIGHT)
    np.testing.assert_allclose(lse2, lse[:, :, idx.numpy()], rtol=0,
                               atol=TIGHT)


def pin_permutation_within_earlier_clean_block(lib):
    """Permuting keys/values inside clean block j < k leaves noisy block k's
    rows unchanged (they see clean block j as a set), while the noisy block
    j itself does not see clean block j at all."""
    L, b, d = 16, 4, 8
    q, k, v = bd_inputs.fwd_inputs(1, 1, 1, L, d, seed=11)
    s = 0.35
    out, lse = oracle.fwd(q, k, v, L, b, s, lib=lib)
    j = 1
    idx = torch.arange(2 * L)
    idx[L + j * b:L + (j + 1) * b] = torch.tensor([2, 3, 1, 0]) + L + j * b
    k2, v2 = k[:, :, idx], v[:, :, idx]
    out2, lse2 = oracle.fwd(q, k2, v2, L, b, s, lib=lib)
    rows = list(range((j + 1) * b, L))  # noisy blocks after j
    np.testing.assert_allclose(out2[0, 0, rows], out[0, 0, rows], rtol=0,
                               atol=1e-12)
    np.testing.assert_allclose(lse2[0, 0, rows], lse[0, 0, rows], rtol=0,
                               atol=1e-12)
    # changing clean block j's values must not move noisy rows of blocks <= j
    v3 = v.clone()
    v3[:, :, L + j * b:L + (j + 1) * b] = 3.0
    out3, _ = oracle.fwd(q, k, v3, L, b, s, lib=lib)
    early = list(range(0, (j + 1) * b))
    np.testing.assert_allclose(out3[0, 0, early], out[0, 0, early], rtol=0,
                               atol=0)
    assert np.abs(out3[0, 0, rows] - out[0, 0, rows]).max() > 1e-3


def pin_gqa_grouping(lib):
    """q-head h reads kv-head h // (Hq/Hkv): the grouped call equals the
    ungrouped one with each kv-head repeated for its consecutive q-heads."""
    L, b, d = 8, 2, 8
    q, k, v = bd_inputs.fwd_inputs(2, 6, 2, L, d, seed=12)
    s = 0.4
    out, lse = oracle.fwd(q, k, v, L, b, s, lib=lib)
    ke = k.repeat_interleave(3, dim=1)
    ve = v.repeat_interleave(3, dim=1)
    out2, lse2 = oracle.fwd(q, ke, ve, L, b, s, lib=lib)
    np.testing.assert_array_equal(out, out2)
    np.testing.assert_array_equal(lse, lse2)


def pin_scale_multiplies_scores(lib):
    """scale multiplies q.k: (2q, s/2) gives the same result as (q, s)
    (doubling a bf16 value is exact), and lse carries the scale inside."""
    L, b, d = 8, 4, 16
    q, k, v = bd_inputs.fwd_inputs(1, 2, 2, L, d, seed=13)
    out, lse = oracle.fwd(q, k, v, L, b, 0.5, lib=lib)
    out2, lse2 = oracle.fwd(_bf(q.float() * 2), k, v, L, b, 0.25, lib=lib)
    np.testing.assert_allclose(out2, out, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-13)
    # lse of a row that sees exactly one key is scale * q.k
    o1, l1 = oracle.decode(q[:, :, :1], k[:, :, :1], v[:, :, :1],
                           [0], 1, 0.5, lib=lib)
    qk = (_f64(q[0, 0, 0]) * _f64(k[0, 0, 0])).sum().item()
    assert abs(l1[0, 0, 0] - 0.5 * qk) < 1e-12
    np.testing.assert_allclose(o1[0, 0, 0], _f64(v[0, 0, 0]).numpy(), atol=0)


def pin_decode_matches_fwd_noisy_block(lib):
    """Cross-form identity: decode (mode 0) of noisy block k over a cache
    holding the clean K/V of blocks < k followed by the noisy K/V of block k
    equals the training/prefill result of noisy block k."""
    L, b, d, Hq, Hkv = 16, 4, 16, 4, 2
    q, k, v = bd_inputs.fwd_inputs(1, Hq, Hkv, L, d, seed=14)
    s = 1 / math.sqrt(d)
    out, lse = oracle.fwd(q, k, v, L, b, s, lib=lib)
    for kb in range(L // b):
        n = kb * b
        kc = torch.cat([k[:, :, L:L + n], k[:, :, n:n + b]], dim=2)
        vc = torch.cat([v[:, :, L:L + n], v[:, :, n:n + b]], dim=2)
        o, l_ = oracle.decode(q[:, :, n:n + b].contiguous(), kc.contiguous(),
                              vc.contiguous(), [n], 0, s, lib=lib)
        np.testing.assert_allclose(o, out[:, :, n:n + b], rtol=0, atol=TIGHT)
        np.testing.assert_allclose(l_, lse[:, :, n:n + b], rtol=0, atol=TIGHT)


def pin_combine_of_partition(lib):
    """Merging results over any partition of a row's visible keys (empty
    parts included) gives the unsplit result."""
    B, Hq, Hkv, b, d, S = 1, 2, 1, 4, 16, 64
    q, kc, vc, lens = bd_inputs.decode_inputs(B, Hq, Hkv, b, d, S,
                                              cache_len=[50], seed=15)
    s = 1 / math.sqrt(d)
    out, lse = oracle.decode(q, kc, vc, lens, 0, s, lib=lib)
    n = 54
    for cuts in ((0, 13, 13, 40, 54), (0, 54), (0, 1, 2, 53, 54)):
        for h in range(Hq):
            for j in range(b):
                os_, ls_ = [], []
                for a, z in zip(cuts[:-1], cuts[1:]):
                    if a == z:
                        os_.append(np.zeros(d))
                        ls_.append(-np.inf)
                        continue
                    o, l_ = sdpa_out_lse(q[0, h, j:j + 1], kc[0, 0, a:z],
                                         vc[0, 0, a:z], s)
                    os_.append(o[0].numpy())
                    ls_.append(l_[0].item())
                oo, ll = oracle.combine(np.array(os_), np.array(ls_), lib=lib)
                np.testing.assert_allclose(oo, out[0, h, j], rtol=0,
                                           atol=TIGHT)
                assert abs(ll - lse[0, h, j]) < TIGHT
    oo, ll = oracle.combine(np.zeros((2, d)), np.array([-np.inf, -np.inf]),
                            lib=lib)
    assert ll == -np.inf and (oo == 0).all()


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
