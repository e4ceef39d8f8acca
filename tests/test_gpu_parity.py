"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances (bf16 out vs fp64): max-abs <= 2e-2 and mean-abs <= 2e-3; fp32
lse: max-abs <= 1e-3.  Small cases compare every element; the full-size
workloads, in the launch configuration the benchmark times, compare a
seeded sample of rows (always including the first and last rows) that the
oracle computes one by one.
"""
import math

import numpy as np
import pytest
import torch

import bd_inputs
import oracle
import block_diffusion_lm_attn_b200 as bd
from block_diffusion_lm_attn_b200 import build

pytestmark = pytest.mark.gpu

OUT_MAX, OUT_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    bd.load()
    assert torch.cuda.is_available()


def check(out_gpu, lse_gpu, out_ref, lse_ref, what=""):
    o = out_gpu.float().cpu().numpy().reshape(out_ref.shape).astype(np.float64)
    l_ = lse_gpu.float().cpu().numpy().reshape(lse_ref.shape).astype(np.float64)
    err = np.abs(o - out_ref)
    lerr = np.abs(l_ - lse_ref)
    assert np.isfinite(o).all() and np.isfinite(l_).all(), what
    assert err.max() <= OUT_MAX, (what, "out max-abs", err.max())
    assert err.mean() <= OUT_MEAN, (what, "out mean-abs", err.mean())
    assert lerr.max() <= LSE_MAX, (what, "lse max-abs", lerr.max())
    return err.max(), err.mean(), lerr.max()


def run_fwd(q, k, v, L, b, scale):
    out, lse = bd.fwd(q.cuda(), k.cuda(), v.cuda(), L, b, scale)
    torch.cuda.synchronize()
    assert bd.device_status() == bd.BD_OK
    return out, lse


def run_decode(q, kc, vc, lens, mode, **kw):
    out, lse = bd.decode(q.cuda(), kc.cuda(), vc.cuda(), lens.cuda(), mode, **kw)
    torch.cuda.synchronize()
    assert bd.device_status() == bd.BD_OK
    return out, lse


# ----------------------------------------------------------------------------
# training / prefill form


def test_fwd_tiny_all_elements():
    s = bd_inputs.FWD_TINY
    q, k, v = bd_inputs.fwd_inputs_for(s)
    out, lse = run_fwd(q, k, v, s.L, s.b, s.scale)
    ro, rl = oracle.fwd(q, k, v, s.L, s.b, s.scale)
    check(out, lse, ro, rl, "fwd tiny")


FWD_GRID = [
    # B, Hq, Hkv, L, b, d
    (1, 1, 1, 8, 1, 32),
    (2, 2, 1, 48, 3, 64),
    (1, 4, 2, 96, 8, 128),
    (1, 2, 2, 200, 8, 128),     # L not a multiple of 64 or 128
    (2, 8, 1, 128, 32, 64),
    (1, 4, 4, 192, 64, 128),
    (1, 2, 1, 256, 128, 128),
    (1, 2, 2, 256, 256, 32),
    (1, 8, 8, 300, 100, 128),   # ragged tails everywhere
    (1, 2, 1, 224, 28, 128),
    (2, 4, 1, 130, 1, 128),
    (1, 16, 2, 384, 4, 128),
    (1, 1, 1, 64, 8, 128),      # fewer work items than SMs
    (3, 2, 2, 136, 17, 128),    # ragged query tiles in both halves
    (1, 4, 1, 512, 512, 128),   # one block per half (b = L)
    (1, 4, 2, 200, 8, 64),      # head dim 64 on the paired kernel, ragged tails
    (2, 3, 3, 136, 17, 64),     # head dim 64 on the one-tile kernel
    (1, 4, 2, 200, 8, 32),      # head dim 32 on the paired kernel, ragged tails
    (2, 3, 3, 136, 17, 32),     # head dim 32 on the one-tile kernel
]


def test_fwd_kernel_selection():
    """Even GQA groups run the paired tcgen05 kernel (the one the benchmark
    times), odd groups the one-tile tcgen05 kernel, at every head dim; so the
    grid below covers each kernel at 128, 64 and 32."""
    assert bd.bd_attn_debug_fwd_kernel(32, 8, 128) == 2
    assert bd.bd_attn_debug_fwd_kernel(4, 2, 128) == 2
    assert bd.bd_attn_debug_fwd_kernel(8, 8, 128) == 1
    assert bd.bd_attn_debug_fwd_kernel(3, 1, 128) == 1
    assert bd.bd_attn_debug_fwd_kernel(4, 2, 64) == 2
    assert bd.bd_attn_debug_fwd_kernel(2, 2, 64) == 1
    assert bd.bd_attn_debug_fwd_kernel(4, 2, 32) == 2
    assert bd.bd_attn_debug_fwd_kernel(2, 2, 32) == 1
    assert bd.bd_attn_debug_fwd_kernel(3, 2, 128) == -1


@pytest.mark.parametrize("B,Hq,Hkv,L,b,d", FWD_GRID)
def test_fwd_grid_all_elements(B, Hq, Hkv, L, b, d):
    q, k, v = bd_inputs.fwd_inputs(B, Hq, Hkv, L, d, seed=L + b + d)
    scale = 1 / math.sqrt(d)
    out, lse = run_fwd(q, k, v, L, b, scale)
    ro, rl = oracle.fwd(q, k, v, L, b, scale)
    check(out, lse, ro, rl, (B, Hq, Hkv, L, b, d))


def test_fwd_other_scale_and_value_ranges():
    L, b, d = 128, 16, 128
    q, k, v = bd_inputs.fwd_inputs(1, 4, 2, L, d, seed=21)
    q = (q.float() * 2.0).to(torch.bfloat16)
    out, lse = run_fwd(q, k, v, L, b, 0.05)
    ro, rl = oracle.fwd(q, k, v, L, b, 0.05)
    check(out, lse, ro, rl, "scale 0.05")


def _fwd_sampled(s, nsample):
    q, k, v = bd_inputs.fwd_inputs_for(s)
    out, lse = run_fwd(q, k, v, s.L, s.b, s.scale)
    # every sampled head contributes the first and last block of each half
    rows = bd_inputs.fwd_sample_rows(s.B, s.Hq, s.L, s.b, nsample)
    ro, rl = oracle.fwd(q, k, v, s.L, s.b, s.scale, rows=rows)
    d = s.d
    o = out.reshape(-1, d)[torch.tensor(rows, device=out.device)]
    l_ = lse.reshape(-1)[torch.tensor(rows, device=out.device)]
    return check(o, l_, ro, rl, s.name)


def test_fwd_training_shape_sampled():
    _fwd_sampled(bd_inputs.FWD_TRAIN, 3000)


@pytest.mark.parametrize("bb", sorted(bd_inputs.FWD_LONG))
def test_fwd_long_context_sampled(bb):
    _fwd_sampled(bd_inputs.FWD_LONG[bb], 800)


@pytest.mark.parametrize("d", [64, 32])
def test_fwd_long_items_at_smaller_head_dims_sampled(d):
    """From 32 query tiles per half the paired kernel runs its variant with
    a quarter of the exponentials on the FMA pipe; the long-context rows
    cover it at head dim 128, this at 64 and 32."""
    s = bd_inputs.FwdShape("fwd_long_items_d%d" % d, 1, 4, 2, 4096, 16, d, seed=31)
    assert s.L // 128 >= 32  # the variant's threshold, in query tiles per half
    assert bd.bd_attn_debug_fwd_kernel(s.Hq, s.Hkv, d) == 2
    _fwd_sampled(s, 600)


def test_fwd_training_shape_invariants():
    """Properties that hold at any size: v = 1 gives out = 1, and the
    result is bit-identical run to run."""
    s = bd_inputs.FWD_TRAIN
    q, k, _ = bd_inputs.fwd_inputs_for(s)
    ones = torch.ones_like(k)
    out, _ = run_fwd(q, k, ones, s.L, s.b, s.scale)
    assert (out.float() - 1).abs().max().item() <= 1e-2
    qd, kd, vd = q.cuda(), k.cuda(), k.cuda()
    o1, l1 = bd.fwd(qd, kd, vd, s.L, s.b, s.scale)
    o2, l2 = bd.fwd(qd, kd, vd, s.L, s.b, s.scale)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# ----------------------------------------------------------------------------
# block-decode form

DEC_GRID = [
    # B, Hq, Hkv, b, d, lens, mode
    (1, 1, 1, 1, 32, [0], 0),
    (1, 1, 1, 1, 32, [0], 1),
    (2, 4, 2, 5, 64, [1, 127], 0),
    (2, 4, 2, 5, 64, [128, 129], 1),
    (3, 32, 8, 32, 128, [0, 300, 1000], 0),
    (3, 32, 8, 28, 128, [511, 64, 2000], 1),
    (2, 8, 8, 8, 128, [4095, 17], 1),
    (4, 16, 2, 16, 128, [5, 900, 31, 257], 0),   # 8 heads x 16 rows = 128
    (2, 16, 1, 20, 64, [100, 3000], 1),          # 320 rows: several row tiles
    (1, 2, 2, 64, 128, [700], 0),
    (1, 8, 1, 40, 128, [5000], 1),       # 320 rows: 3 row tiles, one sequence
    (1, 2, 1, 200, 128, [300], 1),       # b > 128: rows with no key in a piece
    (2, 4, 4, 3, 128, [20000, 1], 0),    # one long unit cut across many CTAs
    (5, 8, 2, 7, 128, [0, 128, 129, 1023, 8000], 1),
    (3, 8, 2, 16, 64, [2, 600, 20000], 0),       # head dim 64, one unit cut across CTAs
]


@pytest.mark.parametrize("B,Hq,Hkv,b,d,lens,mode", DEC_GRID)
def test_decode_grid_all_elements(B, Hq, Hkv, b, d, lens, mode):
    S_cap = max(lens) + b + 3
    q, kc, vc, cl = bd_inputs.decode_inputs(B, Hq, Hkv, b, d, S_cap,
                                            cache_len=lens, seed=b + d)
    out, lse = run_decode(q, kc, vc, cl, mode)
    ro, rl = oracle.decode(q, kc, vc, cl, mode, 1 / math.sqrt(d))
    check(out, lse, ro, rl, (B, Hq, Hkv, b, d, lens, mode))


def test_decode_explicit_workspace_matches_internal():
    B, Hq, Hkv, b, d = 2, 8, 2, 12, 128
    lens = [333, 1200]
    S_cap = 1300
    q, kc, vc, cl = bd_inputs.decode_inputs(B, Hq, Hkv, b, d, S_cap,
                                            cache_len=lens, seed=3)
    o1, l1 = run_decode(q, kc, vc, cl, 1)
    nbytes = bd.workspace_bytes(B, Hq, Hkv, b, d, S_cap)
    ws = torch.full((nbytes,), 0x7f, dtype=torch.uint8, device="cuda")
    o2, l2 = run_decode(q, kc, vc, cl, 1, workspace=ws)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def _decode_sampled(s, nsample):
    q, kc, vc, cl = bd_inputs.decode_inputs_for(s)
    out, lse = run_decode(q, kc, vc, cl, s.mode)
    total = s.B * s.Hq * s.b
    rows = bd_inputs.sample_rows(total, s.b, nsample)
    ro, rl = oracle.decode(q, kc, vc, cl, s.mode, s.scale, rows=rows)
    idx = torch.tensor(rows, device=out.device)
    return check(out.reshape(-1, s.d)[idx], lse.reshape(-1)[idx], ro, rl,
                 s.name)


def test_decode_denoise_sampled():
    _decode_sampled(bd_inputs.DEC_DENOISE, 1500)


def test_decode_verify_sampled():
    _decode_sampled(bd_inputs.DEC_VERIFY, 1500)


def test_decode_matches_fwd_noisy_block():
    """Cross-form identity on the GPU: decode of noisy block k over a cache
    of clean blocks < k plus the block's own noisy K/V equals the training
    form's noisy rows of block k."""
    L, b, d, Hq, Hkv = 256, 32, 128, 8, 2
    q, k, v = bd_inputs.fwd_inputs(1, Hq, Hkv, L, d, seed=31)
    out, lse = run_fwd(q, k, v, L, b, 1 / math.sqrt(d))
    kb = 5
    n = kb * b
    kc = torch.cat([k[:, :, L:L + n], k[:, :, n:n + b]], 2).contiguous()
    vc = torch.cat([v[:, :, L:L + n], v[:, :, n:n + b]], 2).contiguous()
    o2, l2 = run_decode(q[:, :, n:n + b].contiguous(), kc, vc,
                        torch.tensor([n], dtype=torch.int32), 0)
    assert (o2.float() - out[:, :, n:n + b].float()).abs().max() <= 2e-2
    assert (l2 - lse[:, :, n:n + b]).abs().max() <= 1e-3


def test_decode_is_deterministic_and_graph_capturable():
    """Same bits on repeated calls; the call captured in a CUDA graph (with
    an explicit workspace) replays to the same result."""
    B, Hq, Hkv, b, d = 4, 32, 8, 32, 128
    lens = [3000, 17, 2048, 511]
    S_cap = 3100
    q, kc, vc, cl = bd_inputs.decode_inputs(B, Hq, Hkv, b, d, S_cap,
                                            cache_len=lens, seed=9)
    q, kc, vc, cl = q.cuda(), kc.cuda(), vc.cuda(), cl.cuda()
    ws = torch.empty(bd.workspace_bytes(B, Hq, Hkv, b, d, S_cap),
                     dtype=torch.uint8, device="cuda")
    o1, l1 = bd.decode(q, kc, vc, cl, 0, workspace=ws)
    o2, l2 = bd.decode(q, kc, vc, cl, 0, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    out = torch.empty_like(o1)
    lse = torch.empty_like(l1)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        bd.decode(q, kc, vc, cl, 0, out=out, lse=lse, workspace=ws, stream=s)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            bd.decode(q, kc, vc, cl, 0, out=out, lse=lse, workspace=ws, stream=s)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, o1) and torch.equal(lse, l1)
    assert bd.device_status() == bd.BD_OK


def test_decode_bad_cache_len_is_reported():
    B, Hq, Hkv, b, d, S_cap = 2, 4, 2, 8, 64, 100
    q, kc, vc, cl = bd_inputs.decode_inputs(B, Hq, Hkv, b, d, S_cap,
                                            cache_len=[10, 20], seed=5)
    cl = torch.tensor([10, 95], dtype=torch.int32)  # 95 + 8 > 100
    out, lse = bd.decode(q.cuda(), kc.cuda(), vc.cuda(), cl.cuda(), 0)
    assert bd.device_status() == bd.BD_ERR_DEVICE_TIMEOUT
    assert bd.device_status() == bd.BD_OK  # cleared
    assert torch.isnan(lse[1]).all() and torch.isfinite(lse[0]).all()
    ro, rl = oracle.decode(q[:1], kc[:1], vc[:1], [10], 0, 1 / math.sqrt(d))
    check(out[:1], lse[:1], ro, rl, "good sequence next to a bad one")


def test_internal_workspace_under_a_captured_graph():
    """A graph captured with the library's internal decode workspace
    (workspace = NULL) replays correctly after other NULL-workspace calls,
    of other sizes and head dims, ran in between: the buffer is allocated
    once per device, is the same size for every call, and is never freed."""
    B, Hq, Hkv, b, d = 4, 32, 8, 32, 128
    lens = [900, 17, 2048, 511]
    S_cap = 2100
    q, kc, vc, cl = bd_inputs.decode_inputs(B, Hq, Hkv, b, d, S_cap,
                                            cache_len=lens, seed=23)
    qd, kd, vd, cd = q.cuda(), kc.cuda(), vc.cuda(), cl.cuda()
    out = torch.empty_like(qd)
    lse = torch.empty((B, Hq, b), device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        bd.decode(qd, kd, vd, cd, 0, out=out, lse=lse, stream=s)  # allocates
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            bd.decode(qd, kd, vd, cd, 0, out=out, lse=lse, stream=s)
    torch.cuda.synchronize()
    # other sizes and head dims through the same internal buffer
    for (B2, Hq2, Hkv2, b2, d2, n) in [(256, 32, 8, 32, 32, 20), (3, 4, 1, 8, 64, 300)]:
        assert bd.workspace_bytes(B2, Hq2, Hkv2, b2, d2, n + b2) == \
            bd.workspace_bytes(B, Hq, Hkv, b, d, S_cap)
        q2, kc2, vc2, cl2 = bd_inputs.decode_inputs(B2, Hq2, Hkv2, b2, d2, n + b2,
                                                    cache_len=[n] * B2, seed=24)
        bd.decode(q2.cuda(), kc2.cuda(), vc2.cuda(), cl2.cuda(), 1)
    torch.cuda.synchronize()
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert bd.device_status() == bd.BD_OK
    ro, rl = oracle.decode(q, kc, vc, cl, 0, 1 / math.sqrt(d))
    check(out, lse, ro, rl, "graph replay after other calls on the internal workspace")