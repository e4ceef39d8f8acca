"""Pins of the backward oracle (``oracle.backward``).

Each ``grad_pin_*`` takes the module (or a mutated copy) and checks it
against something outside it: central finite differences of its forward
(itself pinned to the C oracle's forward, which ``pins.py`` pins to the
pages), and torch autograd through a masked attention in fp64 (a library
routine), with the mask from the pinned predicate.
"""
from __future__ import annotations

import math

import numpy as np
import torch
import torch.nn.functional as F

import bd_inputs
import oracle


def _tiny(seed, B=1, Hq=2, Hkv=1, L=6, b=2, d=4):
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn((B, Hq, 2 * L, d), generator=g, dtype=torch.float64)
    k = torch.randn((B, Hkv, 2 * L, d), generator=g, dtype=torch.float64)
    v = torch.randn((B, Hkv, 2 * L, d), generator=g, dtype=torch.float64)
    do = torch.randn((B, Hq, 2 * L, d), generator=g, dtype=torch.float64)
    return q.numpy(), k.numpy(), v.numpy(), do.numpy()


def grad_pin_dense_fwd_is_the_oracle_forward(mod):
    """The dense forward used below equals the C oracle's forward on
    bf16-exact inputs (so the finite differences differentiate the pinned
    definition)."""
    L, b, d = 16, 4, 8
    q, k, v = bd_inputs.fwd_inputs(1, 4, 2, L, d, seed=51)
    s = 0.3
    ro, rl = oracle.fwd(q, k, v, L, b, s)
    mask = oracle.fwd_mask(L, b)
    for h in range(4):
        o, l_ = mod.dense_fwd(q[0, h].double().numpy(), k[0, h // 2].double().numpy(),
                              v[0, h // 2].double().numpy(), mask, s)
        np.testing.assert_allclose(o, ro[0, h], rtol=0, atol=1e-12)
        np.testing.assert_allclose(l_, rl[0, h], rtol=0, atol=1e-12)


def grad_pin_finite_differences(mod):
    """Every entry of dq, dk, dv equals the central difference of
    sum(dout * out) (out from dense_fwd, grouped heads summed for k and v)."""
    for (B, Hq, Hkv, L, b, d, seed) in ((1, 2, 1, 6, 2, 4, 52),
                                        (1, 1, 1, 4, 4, 3, 53),
                                        (1, 3, 1, 3, 1, 2, 54)):
        q, k, v, do = _tiny(seed, B, Hq, Hkv, L, b, d)
        s = 0.7
        mask = oracle.fwd_mask(L, b)
        G = Hq // Hkv

        def loss(q_, k_, v_):
            tot = 0.0
            for h in range(Hq):
                o, _ = mod.dense_fwd(q_[0, h], k_[0, h // G], v_[0, h // G], mask, s)
                tot += float((o * do[0, h]).sum())
            return tot

        dq, dk, dv = mod.fwd_bwd(q, k, v, do, L, b, s)
        eps = 1e-6
        for arr, grad in ((q, dq), (k, dk), (v, dv)):
            it = np.nditer(arr, flags=["multi_index"])
            for _ in it:
                ix = it.multi_index
                old = arr[ix]
                arr[ix] = old + eps
                fp = loss(q, k, v)
                arr[ix] = old - eps
                fm = loss(q, k, v)
                arr[ix] = old
                fd = (fp - fm) / (2 * eps)
                assert abs(fd - grad[ix]) <= 1e-7 * max(1.0, abs(fd)), (ix, fd, grad[ix])


def grad_pin_torch_autograd(mod):
    """dq, dk, dv equal torch autograd of scaled_dot_product_attention in
    fp64 with the block mask as a boolean attn_mask (grouped query heads by
    repeat_interleave of k and v), on several (L, b)."""
    for (B, Hq, Hkv, L, b, d, seed) in ((2, 4, 2, 12, 3, 8, 55),
                                        (1, 2, 2, 16, 16, 4, 56),
                                        (1, 4, 1, 10, 1, 6, 57)):
        q, k, v, do = _tiny(seed, B, Hq, Hkv, L, b, d)
        s = 1 / math.sqrt(d)
        mask = torch.from_numpy(oracle.fwd_mask(L, b))
        qt = torch.from_numpy(q).requires_grad_()
        kt = torch.from_numpy(k).requires_grad_()
        vt = torch.from_numpy(v).requires_grad_()
        G = Hq // Hkv
        out = F.scaled_dot_product_attention(
            qt, kt.repeat_interleave(G, 1), vt.repeat_interleave(G, 1),
            attn_mask=mask, scale=s)
        (out * torch.from_numpy(do)).sum().backward()
        dq, dk, dv = mod.fwd_bwd(q, k, v, do, L, b, s)
        np.testing.assert_allclose(dq, qt.grad.numpy(), rtol=0, atol=1e-11)
        np.testing.assert_allclose(dk, kt.grad.numpy(), rtol=0, atol=1e-11)
        np.testing.assert_allclose(dv, vt.grad.numpy(), rtol=0, atol=1e-11)


def grad_pin_groups_subset(mod):
    """Computing a subset of (batch, kv-head) groups gives the same numbers
    as the full call for those groups."""
    q, k, v, do = _tiny(58, B=2, Hq=4, Hkv=2, L=8, b=2, d=4)
    dq, dk, dv = mod.fwd_bwd(q, k, v, do, 8, 2, 0.5)
    part = mod.fwd_bwd_groups(q, k, v, do, 8, 2, 0.5, groups=[(1, 0)])
    a, bk, c = part[(1, 0)]
    np.testing.assert_array_equal(a, dq[1, 0:2])
    np.testing.assert_array_equal(bk, dk[1, 0])
    np.testing.assert_array_equal(c, dv[1, 0])


GRAD_PINS = [v for k, v in sorted(globals().items()) if k.startswith("grad_pin_")]
