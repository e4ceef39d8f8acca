"""Failure detection on the GPU without a GPU fault: a one-shot injected
fault makes one CTA's bounded wait run out; the launch must report
BD_ERR_DEVICE_TIMEOUT through the device status word, and the context must
stay usable (the next call is correct and reports BD_OK)."""
import math

import numpy as np
import pytest
import torch

import bd_inputs
import oracle
import block_diffusion_lm_attn_b200 as bd
from block_diffusion_lm_attn_b200 import build

pytestmark = pytest.mark.gpu


def test_bounded_wait_timeout_is_reported_and_context_survives():
    build.build()
    bd.load()
    L, b, d = 256, 32, 128
    q, k, v = bd_inputs.fwd_inputs(1, 2, 2, L, d, seed=41)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    assert bd.device_status() == bd.BD_OK
    assert bd.bd_attn_debug_inject_fault(1) == bd.BD_OK
    bd.fwd(qd, kd, vd, L, b, 1 / math.sqrt(d))
    assert bd.device_status() == bd.BD_ERR_DEVICE_TIMEOUT
    assert bd.device_status() == bd.BD_OK  # read and cleared
    out, lse = bd.fwd(qd, kd, vd, L, b, 1 / math.sqrt(d))
    torch.cuda.synchronize()
    assert bd.device_status() == bd.BD_OK
    ro, rl = oracle.fwd(q, k, v, L, b, 1 / math.sqrt(d))
    assert np.abs(out.float().cpu().numpy() - ro).max() <= 2e-2
    assert np.abs(lse.cpu().numpy() - rl).max() <= 1e-3


def test_overlapping_launches_on_one_counter_pair_are_reported():
    """Two forwards 64 calls apart draw the same work-counter pair.  With the
    grid capped at 16 CTAs and the two on different streams they run at the
    same time: the overlap must show in the device status (the outputs of
    both are then unreliable, and the test does not look at them).  The same
    sequence on one stream is clean.  Nothing waits on another launch, so
    mixed counts change which items run, never whether a CTA ends."""
    build.build()
    bd.load()
    big = bd_inputs.FWD_LONG[64]
    qb, kb, vb = (t.cuda() for t in bd_inputs.fwd_inputs_for(big))
    qt, kt, vt = (t.cuda() for t in bd_inputs.fwd_inputs(1, 2, 2, 128, 128, seed=43))
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()

    def sequence(second_stream):
        bd.fwd(qb, kb, vb, big.L, big.b, big.scale, stream=sa)
        for _ in range(63):
            bd.fwd(qt, kt, vt, 128, 16, 0.1, stream=second_stream)
        bd.fwd(qt, kt, vt, 128, 16, 0.1, stream=second_stream)  # same pair as the first

    try:
        torch.cuda.synchronize()
        assert bd.bd_attn_debug_reset_sched() == bd.BD_OK
        assert bd.device_status() == bd.BD_OK
        assert bd.bd_attn_debug_set_grid(16) == bd.BD_OK
        sequence(sa)
        torch.cuda.synchronize()
        assert bd.device_status() == bd.BD_OK
        sequence(sb)
        torch.cuda.synchronize()
        assert bd.device_status() == bd.BD_ERR_DEVICE_TIMEOUT
    finally:
        bd.bd_attn_debug_set_grid(0)
        torch.cuda.synchronize()
        assert bd.bd_attn_debug_reset_sched() == bd.BD_OK
        bd.device_status()
    # the library is usable and correct afterwards
    L, b, d = 256, 32, 128
    q, k, v = bd_inputs.fwd_inputs(1, 2, 2, L, d, seed=41)
    out, lse = bd.fwd(q.cuda(), k.cuda(), v.cuda(), L, b, 1 / math.sqrt(d))
    torch.cuda.synchronize()
    assert bd.device_status() == bd.BD_OK
    ro, rl = oracle.fwd(q, k, v, L, b, 1 / math.sqrt(d))
    assert np.abs(out.float().cpu().numpy() - ro).max() <= 2e-2
