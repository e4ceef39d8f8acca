"""The persistent head-dim-128 kernels at grid sizes other than one CTA per
SM (bd_attn_debug_set_grid): the forward's dynamic hand-out with few CTAs,
and the decode's stream-K split at different cut positions, including one
CTA that takes everything and grids where a unit spans many ranges.  Every
element is compared with the fp64 oracle at the same tolerances as
test_gpu_parity.py."""
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


@pytest.fixture(autouse=True)
def _lib():
    build.build()
    bd.load()
    assert torch.cuda.is_available()
    yield
    assert bd.bd_attn_debug_set_grid(0) == bd.BD_OK
    assert bd.bd_attn_debug_set_chunk(0) == bd.BD_OK


def check(out, lse, ro, rl, what):
    o = out.float().cpu().numpy().reshape(ro.shape).astype(np.float64)
    l_ = lse.float().cpu().numpy().reshape(rl.shape).astype(np.float64)
    err, lerr = np.abs(o - ro), np.abs(l_ - rl)
    assert np.isfinite(o).all() and np.isfinite(l_).all(), what
    assert err.max() <= OUT_MAX, (what, err.max())
    assert err.mean() <= OUT_MEAN, (what, err.mean())
    assert lerr.max() <= LSE_MAX, (what, lerr.max())


GRIDS = [1, 5, 37, 147]


@pytest.mark.parametrize("ctas", GRIDS)
def test_fwd_at_grid(ctas):
    assert bd.bd_attn_debug_set_grid(ctas) == bd.BD_OK
    for (B, Hq, Hkv, L, b) in [(2, 4, 2, 200, 8), (1, 8, 2, 384, 32)]:
        d = 128
        q, k, v = bd_inputs.fwd_inputs(B, Hq, Hkv, L, d, seed=ctas + L)
        out, lse = bd.fwd(q.cuda(), k.cuda(), v.cuda(), L, b, 1 / math.sqrt(d))
        torch.cuda.synchronize()
        assert bd.device_status() == bd.BD_OK
        ro, rl = oracle.fwd(q, k, v, L, b, 1 / math.sqrt(d))
        check(out, lse, ro, rl, (ctas, B, Hq, Hkv, L, b))


@pytest.mark.parametrize("chunk", [1, 3])
def test_fwd_chunked_work_list(chunk):
    """The forward's work list run chunk by chunk (heaviest item first inside
    a chunk) with several chunks and a ragged last one: on the paired kernel
    (4 and 12 head pairs) and on the one-tile kernel (6 heads of an odd
    group), with a few CTAs so that items of different chunks overlap."""
    assert bd.bd_attn_debug_set_chunk(chunk) == bd.BD_OK
    assert bd.bd_attn_debug_set_grid(37) == bd.BD_OK
    for (B, Hq, Hkv, L, b) in [(2, 4, 2, 200, 8), (3, 8, 2, 256, 32), (2, 3, 1, 200, 8)]:
        d = 128
        q, k, v = bd_inputs.fwd_inputs(B, Hq, Hkv, L, d, seed=chunk + 7 * L + B)
        out, lse = bd.fwd(q.cuda(), k.cuda(), v.cuda(), L, b, 1 / math.sqrt(d))
        torch.cuda.synchronize()
        assert bd.device_status() == bd.BD_OK
        ro, rl = oracle.fwd(q, k, v, L, b, 1 / math.sqrt(d))
        check(out, lse, ro, rl, (chunk, B, Hq, Hkv, L, b))


DEC_CASES = [
    # B, Hq, Hkv, b, lens, mode
    (3, 8, 2, 28, [700, 3000, 129], 1),
    (2, 8, 2, 32, [256, 256], 0),          # whole units when the grid allows
    (2, 4, 1, 16, [9000, 5], 0),           # unbalanced: one unit over many ranges
    (4, 16, 4, 9, [0, 1, 511, 2600], 1),
]


@pytest.mark.parametrize("ctas", GRIDS)
def test_decode_at_grid(ctas):
    assert bd.bd_attn_debug_set_grid(ctas) == bd.BD_OK
    for (B, Hq, Hkv, b, lens, mode) in DEC_CASES:
        d = 128
        S_cap = max(lens) + b + 5
        q, kc, vc, cl = bd_inputs.decode_inputs(B, Hq, Hkv, b, d, S_cap,
                                                cache_len=lens, seed=ctas + b)
        out, lse = bd.decode(q.cuda(), kc.cuda(), vc.cuda(), cl.cuda(), mode)
        torch.cuda.synchronize()
        assert bd.device_status() == bd.BD_OK
        ro, rl = oracle.decode(q, kc, vc, cl, mode, 1 / math.sqrt(d))
        check(out, lse, ro, rl, (ctas, B, Hq, Hkv, b, lens, mode))
