"""GPU parity of the backward (bd_attn_bwd, through the C ABI) against the
fp64 oracle's gradient (``oracle.backward``: the dense definition, pinned by
finite differences and torch autograd).

out and lse come from bd_attn_fwd on the same inputs, as in training; dout
is drawn N(0,1).  The GPU rounds P and dS to bf16 before the gradient
products and the results to bf16, so each gradient tensor is compared in
units of its own scale: max-abs error <= 2^-5 * max|ref| and mean-abs error
<= 2^-8 * mean|ref| (bf16 unit roundoff u = 2^-9; three roundings per term,
sums over up to 2L terms with cancellation).
"""
import math

import numpy as np
import pytest
import torch

import bd_inputs
from oracle import backward
import block_diffusion_lm_attn_b200 as bd
from block_diffusion_lm_attn_b200 import build

pytestmark = pytest.mark.gpu

TOL_MAX, TOL_MEAN = 2.0 ** -5, 2.0 ** -8


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    bd.load()
    assert torch.cuda.is_available()


def _inputs(B, Hq, Hkv, L, d, seed, k_scale=1.0):
    q, k, v = bd_inputs.fwd_inputs(B, Hq, Hkv, L, d, seed=seed, k_scale=k_scale)
    g = torch.Generator("cpu").manual_seed(seed + 1000)
    do = torch.randn((B, Hq, 2 * L, d), generator=g).to(torch.bfloat16)
    return q, k, v, do


def _gpu_grads(q, k, v, do, L, b, scale):
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    out, lse = bd.fwd(qd, kd, vd, L, b, scale)
    dq, dk, dv = bd.bwd(qd, kd, vd, out, lse, dod, L, b, scale)
    torch.cuda.synchronize()
    assert bd.device_status() == bd.BD_OK
    return dq.float().cpu().numpy(), dk.float().cpu().numpy(), dv.float().cpu().numpy()


def check_grad(got, ref, what):
    err = np.abs(got.astype(np.float64) - ref)
    assert np.isfinite(got).all(), what
    mx, mn = np.abs(ref).max(), np.abs(ref).mean()
    assert err.max() <= TOL_MAX * mx, (what, "max", err.max(), mx)
    assert err.mean() <= TOL_MEAN * mn, (what, "mean", err.mean(), mn)
    return err.max() / mx, err.mean() / mn


BWD_GRID = [
    # B, Hq, Hkv, L, b
    (1, 2, 1, 64, 8),
    (1, 2, 2, 200, 8),     # ragged tiles in both halves
    (2, 4, 1, 130, 1),     # b = 1: token-causal clean half
    (1, 2, 1, 256, 256),   # one block per half
    (1, 8, 2, 384, 4),     # GQA 4:1
    (1, 3, 3, 136, 17),    # odd group and block sizes
    (1, 4, 2, 320, 64),
]


@pytest.mark.parametrize("B,Hq,Hkv,L,b", BWD_GRID)
def test_bwd_grid_all_elements(B, Hq, Hkv, L, b):
    d = 128
    q, k, v, do = _inputs(B, Hq, Hkv, L, d, seed=L + b)
    s = 1 / math.sqrt(d)
    dq, dk, dv = _gpu_grads(q, k, v, do, L, b, s)
    rq, rk, rv = backward.fwd_bwd(q, k, v, do, L, b, s)
    for got, ref, n in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        check_grad(got, ref, (n, B, Hq, Hkv, L, b))


@pytest.mark.parametrize("ctas", [1, 5, 37])
def test_bwd_at_grid_sizes(ctas):
    """The dynamic hand-out of both passes at grid sizes other than one CTA
    per SM gives the same gradients."""
    B, Hq, Hkv, L, b, d = 1, 4, 2, 256, 16, 128
    q, k, v, do = _inputs(B, Hq, Hkv, L, d, seed=99)
    s = 1 / math.sqrt(d)
    assert bd.bd_attn_debug_set_grid(ctas) == bd.BD_OK
    try:
        dq, dk, dv = _gpu_grads(q, k, v, do, L, b, s)
    finally:
        bd.bd_attn_debug_set_grid(0)
    rq, rk, rv = backward.fwd_bwd(q, k, v, do, L, b, s)
    for got, ref, n in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        check_grad(got, ref, (n, ctas))


@pytest.mark.parametrize("chunk", [1, 3])
def test_bwd_chunked_work_lists(chunk):
    """Both passes' work lists run chunk by chunk with several chunks and a
    ragged last one (dK/dV: 4 groups; dQ: 8 heads), on 37 CTAs."""
    B, Hq, Hkv, L, b, d = 2, 4, 2, 256, 16, 128
    q, k, v, do = _inputs(B, Hq, Hkv, L, d, seed=40 + chunk)
    s = 1 / math.sqrt(d)
    assert bd.bd_attn_debug_set_chunk(chunk) == bd.BD_OK
    assert bd.bd_attn_debug_set_grid(37) == bd.BD_OK
    try:
        dq, dk, dv = _gpu_grads(q, k, v, do, L, b, s)
    finally:
        bd.bd_attn_debug_set_grid(0)
        bd.bd_attn_debug_set_chunk(0)
    rq, rk, rv = backward.fwd_bwd(q, k, v, do, L, b, s)
    for got, ref, n in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        check_grad(got, ref, (n, chunk))


def test_bwd_training_shape_sampled_groups():
    """The training shape (B=4, Hq=32, Hkv=8, L=2048, b=32, keys x 0.5) in
    the launch configuration the benchmark times; the oracle computes two
    (batch, kv-head) groups in full: every element of their dq (4 q-heads),
    dk and dv."""
    s_ = bd_inputs.FWD_TRAIN
    q, k, v, do = _inputs(s_.B, s_.Hq, s_.Hkv, s_.L, s_.d, seed=s_.seed,
                          k_scale=s_.k_scale)
    dq, dk, dv = _gpu_grads(q, k, v, do, s_.L, s_.b, s_.scale)
    G = s_.Hq // s_.Hkv
    groups = [(0, 0), (s_.B - 1, s_.Hkv - 1)]
    ref = backward.fwd_bwd_groups(q, k, v, do, s_.L, s_.b, s_.scale, groups=groups)
    for (bi, g), (rq, rk, rv) in ref.items():
        check_grad(dq[bi, g * G:(g + 1) * G], rq, ("dq", bi, g))
        check_grad(dk[bi, g], rk, ("dk", bi, g))
        check_grad(dv[bi, g], rv, ("dv", bi, g))
