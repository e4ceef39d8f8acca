"""GPU parity of the decode-side cache work, through the C ABI, against the
oracle:

* cross-attention-only block decode (intra-block mode 2) on both head-dim
  paths, empty and full encoder caches, and the stream-K split at several
  grid sizes;
* sparse prefix retention: the kept positions and lengths are integers and
  must match exactly; the scores (fp64 on both sides, summed in different
  orders) to 1e-12; the compacted K/V rows bit for bit;
* accepting a speculated block, appending it to the cache and cropping the
  cache: integer and byte work, bit-exact; and the same calls inside a
  captured CUDA graph.
"""
import math

import numpy as np
import pytest
import torch

import bd_inputs
import oracle
from oracle import cache_ops
import block_diffusion_lm_attn_b200 as bd
from block_diffusion_lm_attn_b200 import build

pytestmark = pytest.mark.gpu

OUT_MAX, OUT_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    bd.load()
    assert torch.cuda.is_available()


def _check_attn(out, lse, ro, rl, what):
    o = out.float().cpu().numpy().astype(np.float64).reshape(ro.shape)
    l_ = lse.cpu().numpy().astype(np.float64).reshape(rl.shape)
    fin = np.isfinite(rl)
    # rows with no visible key: out exactly 0, lse -inf
    assert (l_[~fin] == -np.inf).all(), what
    assert (o[~fin] == 0).all(), what
    err = np.abs(o[fin] - ro[fin])
    assert err.max() <= OUT_MAX and err.mean() <= OUT_MEAN, (what, err.max(), err.mean())
    assert np.abs(l_[fin] - rl[fin]).max() <= LSE_MAX, what


# ----------------------------------------------------------------------------
# cross-attention-only decode


@pytest.mark.parametrize("d", [128, 64, 32])
@pytest.mark.parametrize("grid", [0, 5, 37])
def test_decode_mode2_matches_oracle(d, grid):
    B, Hq, Hkv, b = 5, 8, 2, 24
    lens = [0, 1, 130, 700, 1000]
    S_cap = 1000  # the last sequence fills the cache: valid in mode 2 only
    q, kc, vc, cl = bd_inputs.decode_inputs(B, Hq, Hkv, b, d, S_cap + b,
                                            cache_len=lens, seed=71)
    kc, vc = kc[:, :, :S_cap].contiguous(), vc[:, :, :S_cap].contiguous()
    assert bd.bd_attn_debug_set_grid(grid) == bd.BD_OK
    try:
        out, lse = bd.decode(q.cuda(), kc.cuda(), vc.cuda(), cl.cuda(), 2)
        torch.cuda.synchronize()
    finally:
        bd.bd_attn_debug_set_grid(0)
    assert bd.device_status() == bd.BD_OK
    ro, rl = oracle.decode(q, kc, vc, cl, 2, 1 / math.sqrt(d))
    _check_attn(out, lse, ro, rl, ("mode 2", d, grid))


def test_decode_mode2_bad_length_is_reported():
    B, Hq, Hkv, b, d, S_cap = 2, 4, 2, 8, 128, 64
    q = torch.randn((B, Hq, b, d)).to(torch.bfloat16).cuda()
    kc = torch.randn((B, Hkv, S_cap, d)).to(torch.bfloat16).cuda()
    cl = torch.tensor([10, S_cap + 1], dtype=torch.int32).cuda()
    out, lse = bd.decode(q, kc, kc, cl, 2)
    torch.cuda.synchronize()
    assert bd.device_status() == bd.BD_ERR_DEVICE_TIMEOUT
    assert torch.isnan(lse[1]).all() and torch.isfinite(lse[0]).all()


# ----------------------------------------------------------------------------
# sparse prefix retention


def sprint_inputs(B, Hkv, d, S_cap, lens, seed, img_frac=0.6):
    g = torch.Generator("cpu").manual_seed(seed)
    k = torch.randn((B, Hkv, S_cap, d), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Hkv, S_cap, d), generator=g).to(torch.bfloat16)
    conf = torch.rand((B, S_cap), generator=g)
    mod = (torch.rand((B, S_cap), generator=g) < img_frac).to(torch.uint8)
    return k, v, conf, mod, torch.tensor(lens, dtype=torch.int32)


def check_sprint(k, v, conf, mod, cl, alpha, kt, ki):
    B, Hkv, S_cap, d = k.shape
    ko, vo, kept, nl, score = bd.sprint_prune(
        k.cuda(), v.cuda(), cl.cuda(), conf.cuda(), mod.cuda(), alpha, kt, ki,
        want_score=True)
    torch.cuda.synchronize()
    assert bd.device_status() == bd.BD_OK
    rs, rk, rn = oracle.sprint_select(k, cl, conf.numpy(), mod.numpy(), alpha, kt, ki)
    sc = score.cpu().numpy()
    for i in range(B):
        n = int(cl[i])
        np.testing.assert_allclose(sc[i, :n], rs[i, :n], rtol=1e-12, atol=1e-15)
        # the kept set is unique unless two scores straddling a modality's
        # threshold lie within rounding of each other; the seeded inputs have
        # none, so the integers must match exactly
        for m in (0, 1):
            s_m = np.sort(rs[i, :n][(mod[i, :n].numpy() != 0) == m])[::-1]
            r = float(np.float32(kt if m == 0 else ki))  # the interface takes fp32
            want = int(math.floor(r * len(s_m) + 0.5))
            if 0 < want < len(s_m):
                assert s_m[want - 1] - s_m[want] > 1e-9, "near-tie in the inputs"
    np.testing.assert_array_equal(nl.cpu().numpy(), rn)
    np.testing.assert_array_equal(kept.cpu().numpy(), rk)
    # the compacted rows, bit for bit
    rko, rvo = cache_ops.compact(k.view(torch.int16).numpy(),
                                 v.view(torch.int16).numpy(), rk, rn)
    gko = ko.cpu().view(torch.int16).numpy()
    gvo = vo.cpu().view(torch.int16).numpy()
    for i in range(B):
        n = int(rn[i])
        assert (gko[i, :, :n] == rko[i, :, :n]).all()
        assert (gvo[i, :, :n] == rvo[i, :, :n]).all()
    return rn


@pytest.mark.parametrize("alpha,kt,ki", [(0.5, 1.0, 0.8), (0.5, 0.5, 0.3),
                                         (0.0, 0.9, 0.9), (1.0, 1.0, 0.0)])
def test_sprint_small_matches_oracle(alpha, kt, ki):
    k, v, conf, mod, cl = sprint_inputs(4, 2, 64, 1500, [1500, 0, 1, 1029], 72)
    check_sprint(k, v, conf, mod, cl, alpha, kt, ki)


@pytest.mark.parametrize("d", [128, 32])
def test_sprint_ragged_lengths(d):
    lens = [3000, 4095, 17, 2049, 64]
    k, v, conf, mod, cl = sprint_inputs(5, 4, d, 4100, lens, 73, img_frac=0.3)
    check_sprint(k, v, conf, mod, cl, 0.5, 1.0, 0.8)


def test_sprint_prefix_longer_than_register_runs():
    """Prefixes over 16 x 1024 positions take the selection path that keeps
    each thread's run in memory."""
    lens = [20000, 16385, 300]
    k, v, conf, mod, cl = sprint_inputs(3, 1, 32, 20100, lens, 76)
    check_sprint(k, v, conf, mod, cl, 0.5, 0.6, 0.8)


def test_sprint_full_size_denoise_cache():
    """The denoising-decode cache (B=16, Hkv=8, d=128, 8192 cached tokens):
    3/4 image tokens then text, as a prompt of an image and a question."""
    s = bd_inputs.DEC_DENOISE
    B, S_cap = s.B, s.S_cap
    k, v, conf, mod, cl = sprint_inputs(B, s.Hkv, s.d, S_cap, [8192] * B, 74)
    mod[:, :6144] = 1
    mod[:, 6144:] = 0
    rn = check_sprint(k, v, conf, mod, cl, 0.5, 1.0, 0.8)
    assert (rn == 6144 * 8 // 10 + 2048).all()


def test_sprint_bad_length_is_reported():
    k, v, conf, mod, cl = sprint_inputs(2, 2, 64, 100, [50, 50], 75)
    cl[1] = 101
    _, _, kept, nl, _ = bd.sprint_prune(k.cuda(), v.cuda(), cl.cuda(),
                                        conf.cuda(), mod.cuda())
    torch.cuda.synchronize()
    assert bd.device_status() == bd.BD_ERR_DEVICE_TIMEOUT
    assert int(nl[1]) == 0 and (kept[1] == -1).all() and int(nl[0]) > 0


# ----------------------------------------------------------------------------
# accept / append / crop


def _tokens(B, b, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    draft = torch.randint(0, 5, (B, b), generator=g, dtype=torch.int32)
    target = draft.clone()
    # plant the first mismatch at a random position (or none)
    cut = torch.randint(0, b + 1, (B,), generator=g)
    for i in range(B):
        if cut[i] < b:
            target[i, cut[i]] = draft[i, cut[i]] + 1
        # later mismatches must not matter
        if cut[i] + 2 < b:
            target[i, cut[i] + 2] = draft[i, cut[i] + 2] + 7
    return draft, target


@pytest.mark.parametrize("b", [1, 28, 32, 33, 100])
def test_spec_accept_matches_oracle(b):
    B = 70
    draft, target = _tokens(B, b, 80 + b)
    n = bd.spec_accept(draft.cuda(), target.cuda())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(n.cpu().numpy(), cache_ops.accept_len(draft, target))


@pytest.mark.parametrize("copy_rows", [True, False])
def test_cache_append_and_crop_bit_exact(copy_rows):
    B, Hkv, b, d, S_cap = 6, 4, 28, 128, 300
    g = torch.Generator("cpu").manual_seed(81)
    kc = torch.randn((B, Hkv, S_cap, d), generator=g).to(torch.bfloat16)
    vc = torch.randn((B, Hkv, S_cap, d), generator=g).to(torch.bfloat16)
    kn = torch.randn((B, Hkv, b, d), generator=g).to(torch.bfloat16)
    vn = torch.randn((B, Hkv, b, d), generator=g).to(torch.bfloat16)
    lens = torch.tensor([0, 5, 100, 271, 272, 17], dtype=torch.int32)
    draft, target = _tokens(B, b, 82)
    kd, vd, ld = kc.cuda(), vc.cuda(), lens.cuda()
    n = bd.spec_accept(draft.cuda(), target.cuda())
    if copy_rows:
        bd.cache_append(kd, vd, ld, n, kn.cuda(), vn.cuda())
    else:
        bd.cache_append(kd, vd, ld, n)
    torch.cuda.synchronize()
    assert bd.device_status() == bd.BD_OK
    na = cache_ops.accept_len(draft, target)
    i16 = lambda t: t.view(torch.int16).numpy()
    if copy_rows:
        rk, rv, rl = cache_ops.append(i16(kc), i16(vc), lens.numpy(), i16(kn), i16(vn), na)
    else:
        # rows already in place: the cache itself is unchanged
        rk, rv = i16(kc), i16(vc)
        rl = (lens.numpy() + na).astype(np.int32)
    np.testing.assert_array_equal(ld.cpu().numpy(), rl)
    assert (kd.cpu().view(torch.int16).numpy() == rk).all()
    assert (vd.cpu().view(torch.int16).numpy() == rv).all()
    bd.cache_crop(ld, 150)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(ld.cpu().numpy(), cache_ops.crop(rl, 150))


def test_cache_append_overflow_is_reported_and_harmless():
    B, Hkv, b, d, S_cap = 2, 2, 8, 64, 20
    kc = torch.zeros((B, Hkv, S_cap, d), dtype=torch.bfloat16).cuda()
    kn = torch.ones((B, Hkv, b, d), dtype=torch.bfloat16).cuda()
    lens = torch.tensor([15, 3], dtype=torch.int32).cuda()
    n = torch.tensor([8, 8], dtype=torch.int32).cuda()
    bd.cache_append(kc, kc.clone(), lens, n, kn, kn)
    torch.cuda.synchronize()
    assert bd.device_status() == bd.BD_ERR_DEVICE_TIMEOUT
    assert lens.tolist() == [15, 11]
    assert (kc[0] == 0).all() and (kc[1, :, 3:11] == 1).all()


def test_accept_append_crop_capture_in_a_graph():
    """The three calls read every size from device memory, so one captured
    graph serves every step; replays match the oracle."""
    B, Hkv, b, d, S_cap = 4, 2, 16, 128, 200
    g = torch.Generator("cpu").manual_seed(83)
    kc = torch.randn((B, Hkv, S_cap, d), generator=g).to(torch.bfloat16).cuda()
    vc = torch.randn((B, Hkv, S_cap, d), generator=g).to(torch.bfloat16).cuda()
    kn = torch.randn((B, Hkv, b, d), generator=g).to(torch.bfloat16).cuda()
    vn = torch.randn((B, Hkv, b, d), generator=g).to(torch.bfloat16).cuda()
    lens = torch.tensor([0, 10, 50, 100], dtype=torch.int32).cuda()
    draft = torch.zeros((B, b), dtype=torch.int32).cuda()
    target = torch.zeros((B, b), dtype=torch.int32).cuda()
    n = torch.zeros(B, dtype=torch.int32).cuda()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        bd.spec_accept(draft, target, n_accept=n)  # warm-up outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        bd.spec_accept(draft, target, n_accept=n)
        bd.cache_append(kc, vc, lens, n, kn, vn)
        bd.cache_crop(lens, 180)
    ref_k = kc.cpu().view(torch.int16).numpy()
    ref_v = vc.cpu().view(torch.int16).numpy()
    ref_l = lens.cpu().numpy()
    for step in range(3):
        d0, t0 = _tokens(B, b, 90 + step)
        draft.copy_(d0)
        target.copy_(t0)
        graph.replay()
        torch.cuda.synchronize()
        na = cache_ops.accept_len(d0, t0)
        ref_k, ref_v, ref_l = cache_ops.append(ref_k, ref_v, ref_l,
                                               kn.cpu().view(torch.int16).numpy(),
                                               vn.cpu().view(torch.int16).numpy(), na)
        ref_l = cache_ops.crop(ref_l, 180)
        np.testing.assert_array_equal(lens.cpu().numpy(), ref_l)
        assert (kc.cpu().view(torch.int16).numpy() == ref_k).all()
        assert (vc.cpu().view(torch.int16).numpy() == ref_v).all()
    assert bd.device_status() == bd.BD_OK
