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
