"""Block decode through bd_attn_decode_noalloc, the entry point for callers
that cannot allocate device memory at decode time (its scratch is a fixed
array inside the library).  Calls in a row at head dims 128, 64 and 32, with
different inputs, each compared with bd_attn_decode on the same inputs, and
once directly with the fp64 oracle; and a call inside a captured CUDA graph
in global capture mode, where any allocation would fail the capture.
Collected last so that a run stopping at the first failure has already run
every other test."""
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


CASES = [
    # B, Hq, Hkv, b, d, lens, mode
    (16, 32, 8, 32, 128, [2048] * 16, 0),
    (8, 32, 8, 28, 128, [513, 4000, 77, 1024, 3001, 900, 12, 2500], 1),
    (4, 8, 2, 16, 64, [300, 5, 1200, 64], 0),
    (3, 4, 4, 8, 64, [100, 0, 40], 1),
    (3, 8, 2, 16, 32, [700, 3, 64], 0),
]


def test_noalloc_decode_matches_decode_on_two_calls_in_a_row():
    build.build()
    bd.load()
    for B, Hq, Hkv, b, d, lens, mode in CASES:
        S_cap = max(lens) + b
        assert bd.workspace_bytes(B, Hq, Hkv, b, d, S_cap) <= 32 << 20  # the fixed array
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


def test_noalloc_decode_matches_the_oracle():
    build.build()
    bd.load()
    B, Hq, Hkv, b, d, lens, mode = 4, 8, 2, 28, 128, [700, 2047, 0, 129], 1
    S_cap = max(lens) + b
    q, kc, vc, cl = bd_inputs.decode_inputs(B, Hq, Hkv, b, d, S_cap,
                                            cache_len=lens, seed=3)
    out = torch.empty((B, Hq, b, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, Hq, b), device="cuda")
    assert _call_noalloc(q.cuda(), kc.cuda(), vc.cuda(), cl.cuda(), mode,
                         out, lse) == bd.BD_OK
    torch.cuda.synchronize()
    assert bd.device_status() == bd.BD_OK
    ro, rl = oracle.decode(q, kc, vc, cl, mode, 1 / math.sqrt(d))
    err = np.abs(out.float().cpu().numpy() - ro)
    assert err.max() <= OUT_MAX and err.mean() <= OUT_MEAN
    assert np.abs(lse.cpu().numpy() - rl).max() <= LSE_MAX


def test_noalloc_decode_inside_a_graph_capture():
    """After one ordinary call (which looks up the array's address), the
    entry point can be recorded in a CUDA graph captured in global mode; the
    replays read the current inputs and match bd_attn_decode."""
    build.build()
    bd.load()
    B, Hq, Hkv, b, d, mode = 8, 32, 8, 32, 128, 0
    lens = [1500, 900, 2000, 64, 1999, 3, 777, 1024]
    S_cap = max(lens) + b
    q, kc, vc, cl = bd_inputs.decode_inputs(B, Hq, Hkv, b, d, S_cap,
                                            cache_len=lens, seed=17)
    q, kc, vc, cl = q.cuda(), kc.cuda(), vc.cuda(), cl.cuda()
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq, b), device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        assert _call_noalloc(q, kc, vc, cl, mode, out, lse) == bd.BD_OK
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="global"):
        assert _call_noalloc(q, kc, vc, cl, mode, out, lse) == bd.BD_OK
    for seed in (18, 19):
        q2, _, _, _ = bd_inputs.decode_inputs(B, Hq, Hkv, b, d, S_cap,
                                              cache_len=lens, seed=seed)
        q.copy_(q2.cuda())
        graph.replay()
        torch.cuda.synchronize()
        ref_o, ref_l = bd.decode(q, kc, vc, cl, mode)
        torch.cuda.synchronize()
        _compare(ref_o, ref_l, out, lse)
    assert bd.device_status() == bd.BD_OK
