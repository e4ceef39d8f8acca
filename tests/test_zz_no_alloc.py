"""Block decode through bd_attn_decode_noalloc, the entry point for callers
that cannot allocate device memory at decode time (its split-KV scratch is a
fixed array inside the library).  Two calls in a row, with different inputs,
each compared with bd_attn_decode on the same inputs.  Collected last so that
a run stopping at the first failure has already run every other test."""
import numpy as np
import pytest
import torch

import bd_inputs
import block_diffusion_lm_attn_b200 as bd
from block_diffusion_lm_attn_b200 import build

pytestmark = pytest.mark.gpu

OUT_MAX, OUT_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3
SCRATCH_MAX = 32 << 20


def _call_noalloc(q, kc, vc, cl, mode, out, lse):
    B, Hq, b, d = q.shape
    Hkv, S_cap = kc.shape[1], kc.shape[2]
    return bd.bd_attn_decode_noalloc(
        q.data_ptr(), kc.data_ptr(), vc.data_ptr(), cl.data_ptr(),
        out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, b, d, mode,
        torch.cuda.current_stream().cuda_stream, S_cap)


def _compare(o1, l1, o2, l2):
    e = (o1.float() - o2.float()).abs()
    assert e.max().item() <= OUT_MAX and e.mean().item() <= OUT_MEAN
    assert (l1 - l2).abs().max().item() <= LSE_MAX
    assert torch.isfinite(o2.float()).all() and torch.isfinite(l2).all()


def test_noalloc_decode_matches_decode_on_two_calls_in_a_row():
    build.build()
    bd.load()
    cases = [
        # B, Hq, Hkv, b, d, lens, mode
        (16, 32, 8, 32, 128, [2048] * 16, 0),
        (8, 32, 8, 28, 128, [513, 4000, 77, 1024, 3001, 900, 12, 2500], 1),
    ]
    for B, Hq, Hkv, b, d, lens, mode in cases:
        S_cap = max(lens) + b
        assert bd.workspace_bytes(B, Hq, Hkv, b, d, S_cap) <= SCRATCH_MAX
        q, kc, vc, cl = bd_inputs.decode_inputs(B, Hq, Hkv, b, d, S_cap,
                                                cache_len=lens, seed=B + b)
        q, kc, vc, cl = q.cuda(), kc.cuda(), vc.cuda(), cl.cuda()
        ref_o, ref_l = bd.decode(q, kc, vc, cl, mode)
        out = torch.full_like(q, float("nan"))
        lse = torch.full((B, Hq, b), float("nan"), device="cuda")
        assert _call_noalloc(q, kc, vc, cl, mode, out, lse) == bd.BD_OK
        torch.cuda.synchronize()
        assert bd.device_status() == bd.BD_OK
        _compare(ref_o, ref_l, out, lse)

    # a size whose scratch exceeds the fixed array is refused up front
    B, Hq, Hkv, b, d, S_cap = 256, 64, 8, 32, 64, 65536
    assert bd.workspace_bytes(B, Hq, Hkv, b, d, S_cap) > SCRATCH_MAX
    A = 1 << 20
    st = bd.bd_attn_decode_noalloc(A, A, A, A, A, A, B, Hq, Hkv, b, d, 0,
                                   None, S_cap)
    assert st == bd.BD_ERR_UNSUPPORTED
