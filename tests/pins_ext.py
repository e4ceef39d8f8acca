"""Pins of the oracle's later parts: cross-attention-only decode (mode 2),
sparse prefix retention (SPRINT) and the KV-cache bookkeeping of
speculative decoding.

``pin_*`` functions here take an oracle library handle (``oracle.load()`` or
a mutated copy); ``cache_pin_*`` functions take the ``oracle.cache_ops``
module (or a mutated copy).  Each checks the oracle against something
outside it: hand-worked fixtures in ``tests/golden/``, textbook attention
from a library routine, a library sort, or an invariant of the definition.
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch

import bd_inputs
import oracle
from pins import GOLDEN, TIGHT, read_mask_fixture, sdpa_out_lse

# ----------------------------------------------------------------------------
# cross-attention-only decode (intra-block mode 2)


def pin_decode_mode2_mask_fixture(lib):
    for hdr, m in read_mask_fixture("decode_mask_mode2_len3_b2.txt"):
        n, b, S, mode = hdr["cache_len"], hdr["b"], hdr["S_cap"], hdr["mode"]
        got = np.array([[lib.bdo_decode_sees(n, b, mode, j, c)
                         for c in range(S)] for j in range(b)])
        assert (got == m).all(), (hdr, got)


def pin_decode_mode2_is_attention_over_prefix(lib):
    """Mode 2: every canvas row attends exactly to the encoder cache
    positions 0 .. cache_len-1 (textbook attention over them); the canvas's
    own rows in the cache are never read.  An empty cache gives out = 0 and
    lse = -inf."""
    B, Hq, Hkv, b, d, S = 3, 4, 2, 6, 16, 40
    q, kc, vc, lens = bd_inputs.decode_inputs(B, Hq, Hkv, b, d, S,
                                              cache_len=[9, 0, 34], seed=31)
    s = 1 / math.sqrt(d)
    out, lse = oracle.decode(q, kc, vc, lens, 2, s, lib=lib)
    for i in range(B):
        n = int(lens[i])
        for h in range(Hq):
            g = h // (Hq // Hkv)
            if n == 0:
                assert (out[i, h] == 0).all() and (lse[i, h] == -np.inf).all()
                continue
            o, l_ = sdpa_out_lse(q[i, h], kc[i, g, :n], vc[i, g, :n], s)
            np.testing.assert_allclose(out[i, h], o.numpy(), rtol=0, atol=TIGHT)
            np.testing.assert_allclose(lse[i, h], l_.numpy(), rtol=0, atol=TIGHT)
    # the canvas rows' own cache slots do not matter
    kc2, vc2 = kc.clone(), vc.clone()
    for i in range(B):
        n = int(lens[i])
        kc2[i, :, n:] = 5.0
        vc2[i, :, n:] = -5.0
    out2, lse2 = oracle.decode(q, kc2, vc2, lens, 2, s, lib=lib)
    np.testing.assert_array_equal(out2, out)
    np.testing.assert_array_equal(lse2, lse)
    # a full cache (cache_len = S_cap) is valid in mode 2 only
    _, _ = oracle.decode(q, kc, vc, [S, 1, 2], 2, s, lib=lib)


# ----------------------------------------------------------------------------
# sparse prefix retention


def read_sprint_fixture():
    cases = []
    cur = None
    with open(os.path.join(GOLDEN, "sprint_small.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("case="):
                cur = {kv.split("=")[0]: kv.split("=")[1] for kv in line.split()}
                cases.append(cur)
            else:
                key, *vals = line.split()
                cur[key] = [float(x) for x in vals]
    return cases


def _sprint_case_inputs(case):
    keys = np.array(case["keys"]).reshape(-1, 2)
    n = keys.shape[0]
    k = torch.tensor(keys, dtype=torch.float32).to(torch.bfloat16)
    assert (k.float().numpy() == keys).all()  # exact in bf16
    k = k.reshape(1, 1, n, 2)
    conf = np.array([case["conf"]], np.float32)
    mod = np.array([case["modality"]], np.uint8)
    return k, conf, mod, n


def pin_sprint_fixture(lib):
    for case in read_sprint_fixture():
        k, conf, mod, n = _sprint_case_inputs(case)
        score, kept, new_len = oracle.sprint_select(
            k, [n], conf, mod, alpha=float(case["alpha"]),
            keep_text=float(case["keep_text"]),
            keep_image=float(case["keep_image"]), lib=lib)
        np.testing.assert_allclose(score[0, :n], case["score"], rtol=0,
                                   atol=1e-12)
        want = [int(x) for x in case["kept"]]
        assert new_len[0] == len(want), (case["case"], new_len)
        assert list(kept[0, :len(want)]) == want, (case["case"], kept)
        assert (kept[0, len(want):] == -1).all()


def _sprint_random(seed, B=3, Hkv=2, d=16, S=64):
    g = torch.Generator("cpu").manual_seed(seed)
    lens = [S, 37, 1][:B]
    k = torch.randn((B, Hkv, S, d), generator=g).to(torch.bfloat16)
    conf = torch.rand((B, S), generator=g).numpy().astype(np.float32)
    mod = (torch.rand((B, S), generator=g) < 0.6).numpy().astype(np.uint8)
    return k, lens, conf, mod


def pin_sprint_alpha_limits_are_sorts(lib):
    """alpha = 0 ranks by confidence alone and alpha = 1 by key norm alone:
    the kept set equals the one a library sort gives (descending score,
    ascending position), the norm taken by torch.linalg.vector_norm over all
    kv-heads and dims of a position."""
    k, lens, conf, mod = _sprint_random(41)
    B, Hkv, S, d = k.shape
    norms = torch.linalg.vector_norm(k.double().permute(0, 2, 1, 3).reshape(
        B, S, Hkv * d), dim=-1).numpy()
    for alpha in (0.0, 1.0):
        for kt, ki in ((0.5, 0.8), (1.0, 0.3), (0.25, 1.0)):
            score, kept, new_len = oracle.sprint_select(
                k, lens, conf, mod, alpha=alpha, keep_text=kt, keep_image=ki,
                lib=lib)
            for i in range(B):
                n = lens[i]
                if alpha == 0.0:
                    sc = conf[i, :n].astype(np.float64)
                else:
                    sc = norms[i, :n] / norms[i, :n].mean()
                    np.testing.assert_allclose(score[i, :n], sc, rtol=1e-13)
                want = []
                for m, r in ((0, kt), (1, ki)):
                    r = float(np.float32(r))  # the interface's precision
                    pos = [p for p in range(n) if (mod[i, p] != 0) == m]
                    cnt = int(math.floor(r * len(pos) + 0.5))
                    order = sorted(pos, key=lambda p: (-sc[p], p))
                    want += order[:cnt]
                want = sorted(want)
                assert new_len[i] == len(want), (alpha, i)
                assert list(kept[i, :new_len[i]]) == want, (alpha, i)


def pin_sprint_invariants(lib):
    """Keeping everything is the identity; keeping nothing empties the
    prefix; scaling every key by 2 (exact in bf16) leaves the mean-normalised
    scores and the kept set unchanged; the kept list is increasing and each
    kept position outranks every dropped position of its modality."""
    k, lens, conf, mod = _sprint_random(43)
    B, Hkv, S, d = k.shape
    _, kept, nl = oracle.sprint_select(k, lens, conf, mod, 0.5, 1.0, 1.0, lib=lib)
    for i in range(B):
        assert nl[i] == lens[i] and list(kept[i, :lens[i]]) == list(range(lens[i]))
    _, kept0, nl0 = oracle.sprint_select(k, lens, conf, mod, 0.5, 0.0, 0.0, lib=lib)
    assert (nl0 == 0).all() and (kept0 == -1).all()
    sc1, kept1, nl1 = oracle.sprint_select(k, lens, conf, mod, 0.5, 0.7, 0.8, lib=lib)
    k2 = (k.float() * 2).to(torch.bfloat16)
    sc2, kept2, nl2 = oracle.sprint_select(k2, lens, conf, mod, 0.5, 0.7, 0.8, lib=lib)
    np.testing.assert_array_equal(sc1, sc2)
    np.testing.assert_array_equal(kept1, kept2)
    np.testing.assert_array_equal(nl1, nl2)
    for i in range(B):
        n = lens[i]
        ks = list(kept1[i, :nl1[i]])
        assert ks == sorted(set(ks))
        for m in (0, 1):
            pos = [p for p in range(n) if (mod[i, p] != 0) == m]
            kin = [p for p in pos if p in ks]
            kout = [p for p in pos if p not in ks]
            r = float(np.float32(0.7 if m == 0 else 0.8))
            assert len(kin) == int(math.floor(r * len(pos) + 0.5))
            for a in kin:
                for z in kout:
                    assert (sc1[i, a] > sc1[i, z] or
                            (sc1[i, a] == sc1[i, z] and a < z)), (i, a, z)


# ----------------------------------------------------------------------------
# KV-cache bookkeeping (oracle.cache_ops)


def read_spec_fixture():
    vals = {}
    with open(os.path.join(GOLDEN, "spec_accept_append.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, rest = line.split(None, 1)
            if "|" in rest:
                vals[key] = [[int(x) for x in part.split()]
                             for part in rest.split("|")]
            else:
                vals[key] = [int(x) for x in rest.split()]
    return vals


def cache_pin_fixture(ops):
    f = read_spec_fixture()
    draft = np.array(f["draft"], np.int32)
    target = np.array(f["target"], np.int32)
    n = ops.accept_len(draft, target)
    assert list(n) == f["accept"], n
    B, b = draft.shape
    Hkv, S, d = 2, 12, 4
    rng = np.random.default_rng(5)
    kc = rng.integers(0, 1 << 16, (B, Hkv, S, d), dtype=np.uint16)
    vc = rng.integers(0, 1 << 16, (B, Hkv, S, d), dtype=np.uint16)
    kn = rng.integers(0, 1 << 16, (B, Hkv, b, d), dtype=np.uint16)
    vn = rng.integers(0, 1 << 16, (B, Hkv, b, d), dtype=np.uint16)
    lens = np.array(f["len_before"], np.int32)
    kc2, vc2, l2 = ops.append(kc, vc, lens, kn, vn, n)
    assert list(l2) == f["len_after"], l2
    for i in range(B):
        a, z = int(lens[i]), int(lens[i]) + int(n[i])
        # the accepted rows, bit for bit, at the end of the old prefix
        assert (kc2[i, :, a:z] == kn[i, :, :z - a]).all()
        assert (vc2[i, :, a:z] == vn[i, :, :z - a]).all()
        # nothing else moves
        assert (kc2[i, :, :a] == kc[i, :, :a]).all()
        assert (kc2[i, :, z:] == kc[i, :, z:]).all()
        assert (vc2[i, :, z:] == vc[i, :, z:]).all()
    assert list(ops.crop(l2, f["crop"][0])) == f["len_cropped"]


def cache_pin_overflow_and_compaction(ops):
    """An append past the capacity is refused; compaction moves the kept
    rows, in order, to the front (a plain gather by torch.index_select)."""
    kc = np.zeros((1, 1, 4, 2), np.uint16)
    try:
        ops.append(kc, kc, np.array([3], np.int32),
                   np.zeros((1, 1, 2, 2), np.uint16),
                   np.zeros((1, 1, 2, 2), np.uint16), np.array([2], np.int32))
    except ValueError:
        pass
    else:
        raise AssertionError("overflowing append accepted")
    rng = np.random.default_rng(7)
    k = rng.integers(0, 1 << 16, (2, 3, 10, 4), dtype=np.uint16)
    v = rng.integers(0, 1 << 16, (2, 3, 10, 4), dtype=np.uint16)
    kept = np.full((2, 10), -1, np.int32)
    kept[0, :4] = [0, 3, 4, 9]
    kept[1, :1] = [5]
    nl = np.array([4, 1], np.int32)
    ko, vo = ops.compact(k, v, kept, nl)
    for i in range(2):
        idx = torch.tensor(kept[i, :nl[i]], dtype=torch.long)
        ref_k = torch.index_select(torch.from_numpy(k[i].astype(np.int64)), 1, idx)
        ref_v = torch.index_select(torch.from_numpy(v[i].astype(np.int64)), 1, idx)
        assert (ko[i, :, :nl[i]] == ref_k.numpy()).all()
        assert (vo[i, :, :nl[i]] == ref_v.numpy()).all()
        assert (ko[i, :, nl[i]:] == 0).all() and (vo[i, :, nl[i]:] == 0).all()


EXT_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
CACHE_PINS = [v for k, v in sorted(globals().items())
              if k.startswith("cache_pin_")]
