"""Gradient of block-diffusion attention: plain fp64 definition with numpy.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are its only users.  The CUDA library never
imports or calls it; the two share no code.

Training a block-diffusion LM minimises the BDLM loss of "LLaDA2.0-Uni"
(discuss.pytorch.kr), section "Training objective and loss function", eq.
L_BDLM, whose log p(x_{0,k} | x_{0,<k}, x_{t,k}) terms come out of the
training/prefill attention over [x_t ; x_0].  Back-propagating through that
attention needs, given the upstream gradient dO of its output, the
gradients of q, k and v.  For one query head over its kv-head, with the
dense visibility mask M of the three-part block mask ("Nemotron-Labs-
Diffusion-8B-Base 3x decoding speed-up", section 1 "Block Diffusion
Attention"; ``oracle.fwd_mask``):

    S  = scale * Q K^T, set to -inf where M is 0
    P  = softmax of each row of S             (the forward's probabilities)
    dV = P^T dO
    dP = dO V^T
    dS = P * (dP - rowsum(P * dP))            (softmax Jacobian, row by row)
    dQ = scale * dS K
    dK = scale * dS^T Q

With grouped-query attention the q-heads h of a group all read kv-head
h / (Hq / Hkv), so that kv-head's dK and dV are the sums of the group's
terms.  The upstream gradient reaches the output only (the log-sum-exp side
output of the forward is treated as a constant).

Matrix products and exp are library primitives; there is no blocking or
reordering beyond the formulas above.  Inputs are widened to fp64 first.
The module's functions are pinned by ``tests/pins_grad.py`` (central finite
differences of ``dense_fwd``, and torch autograd through a masked attention
in fp64).
"""
from __future__ import annotations

import numpy as np

import oracle


def _f64(t) -> np.ndarray:
    """torch tensor (any float dtype) or array -> fp64 numpy array."""
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().cpu().double().numpy()


def dense_fwd(q, k, v, mask, scale):
    """Masked attention of one head: q [n,d], k, v [m,d], mask [n,m] bool.
    Returns (out [n,d], lse [n]) in fp64; a row with no visible key gives
    out = 0 and lse = -inf."""
    S = scale * (q @ k.T)
    S = np.where(mask, S, -np.inf)
    m = S.max(axis=1, keepdims=True)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    E = np.exp(S - m_safe)
    Z = E.sum(axis=1, keepdims=True)
    P = np.divide(E, Z, out=np.zeros_like(E), where=Z > 0)
    with np.errstate(divide="ignore"):
        lse = np.where(Z[:, 0] > 0, m_safe[:, 0] + np.log(Z[:, 0]), -np.inf)
    return P @ v, lse


def dense_bwd(q, k, v, dout, mask, scale):
    """Gradients of one head's masked attention with respect to q, k, v,
    given the upstream gradient dout [n,d] of its output."""
    S = scale * (q @ k.T)
    S = np.where(mask, S, -np.inf)
    m = S.max(axis=1, keepdims=True)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    E = np.exp(S - m_safe)
    Z = E.sum(axis=1, keepdims=True)
    P = np.divide(E, Z, out=np.zeros_like(E), where=Z > 0)
    dv = P.T @ dout
    dP = dout @ v.T
    D = (P * dP).sum(axis=1, keepdims=True)
    dS = P * (dP - D)
    dq = scale * (dS @ k)
    dk = scale * (dS.T @ q)
    return dq, dk, dv


def fwd_bwd_groups(q, k, v, dout, L: int, b: int, scale: float, groups=None):
    """Training/prefill gradients.  q, dout: [B,Hq,2L,d]; k, v: [B,Hkv,2L,d]
    (torch or numpy, any float dtype; widened to fp64).

    groups: list of (batch, kv-head) pairs to compute, or None for all.
    Returns a dict {(batch, kv_head): (dq [G,2L,d], dk [2L,d], dv [2L,d])}
    where dq holds the G = Hq/Hkv q-heads of that group in order."""
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    assert N == 2 * L and Hq % Hkv == 0
    G = Hq // Hkv
    mask = oracle.fwd_mask(L, b)
    if groups is None:
        groups = [(bi, g) for bi in range(B) for g in range(Hkv)]
    res = {}
    for bi, g in groups:
        kk, vv = _f64(k[bi, g]), _f64(v[bi, g])
        dq = np.zeros((G, N, d))
        dk = np.zeros((N, d))
        dv = np.zeros((N, d))
        for x in range(G):
            h = g * G + x
            a, bk, c = dense_bwd(_f64(q[bi, h]), kk, vv, _f64(dout[bi, h]),
                                 mask, scale)
            dq[x] = a
            dk += bk
            dv += c
        res[(bi, g)] = (dq, dk, dv)
    return res


def fwd_bwd(q, k, v, dout, L: int, b: int, scale: float):
    """All gradients: (dq [B,Hq,2L,d], dk, dv [B,Hkv,2L,d]) in fp64."""
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    dq = np.zeros((B, Hq, N, d))
    dk = np.zeros((B, Hkv, N, d))
    dv = np.zeros((B, Hkv, N, d))
    for (bi, g), (a, bk, c) in fwd_bwd_groups(q, k, v, dout, L, b,
                                              scale).items():
        dq[bi, g * G:(g + 1) * G] = a
        dk[bi, g] = bk
        dv[bi, g] = c
    return dq, dk, dv
