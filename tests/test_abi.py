"""The C-ABI library builds, loads and exports every declared entry point,
and rejects bad arguments on the host (no GPU needed: nothing is launched)."""
import os
import re

import pytest

import block_diffusion_lm_attn_b200 as bd
from block_diffusion_lm_attn_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return bd.load()


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names += re.findall(r"\b(bd_\w+)\s*\(", txt)
    return sorted(set(names))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(bd.EXPORTED) <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for s in range(5):
        assert bd.bd_attn_status_string(s)
    assert bd.bd_attn_status_string(99) == "unknown status"


def test_workspace_bytes(lib):
    assert bd.bd_attn_decode_workspace_bytes(16, 32, 8, 32, 128, 8224) > 0
    assert bd.bd_attn_decode_workspace_bytes(0, 32, 8, 32, 128, 8224) == 0
    assert bd.bd_attn_decode_workspace_bytes(1, 6, 4, 32, 128, 64) == 0
    assert bd.bd_attn_decode_workspace_bytes(1, 4, 4, 32, 128, 0) == 0
    # a cache shorter than the block is valid for cross-attention (mode 2)
    assert bd.bd_attn_decode_workspace_bytes(1, 4, 4, 32, 128, 16) > 0
    w = bd.bd_attn_decode_workspace_bytes(16, 32, 8, 32, 128, 8224)
    assert w % 256 == 0
    # stream-K scratch: two (o, lse) slots of 128 x 128 fp32 rows and a cut
    # descriptor per persistent CTA (148), whatever the sizes and head dim
    per = 2 * 148 * 128 * 128 * 4 + 2 * 148 * 128 * 4 + 148 * 16
    assert per <= w < per + 3 * 256
    for args in [(1, 4, 4, 8, 32, 64), (256, 64, 8, 32, 32, 65536),
                 (64, 32, 8, 28, 64, 8224), (3, 8, 2, 16, 128, 20)]:
        assert bd.bd_attn_decode_workspace_bytes(*args) == w, args
    # the no-alloc entry point's fixed array holds it
    assert w <= 32 << 20


A = 1 << 20  # a 16-byte-aligned fake address; never dereferenced


def fwd_args(**kw):
    a = dict(q=A, k=A, v=A, out=A, lse=A, B=1, Hq=2, Hkv=2, L=64, b=8, d=32,
             scale=0.17, stream=None)
    a.update(kw)
    return a


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), bd.BD_ERR_INVALID_ARG),
    (dict(lse=None), bd.BD_ERR_INVALID_ARG),
    (dict(k=A + 8), bd.BD_ERR_INVALID_ARG),
    (dict(out=A + 2), bd.BD_ERR_INVALID_ARG),
    (dict(B=0), bd.BD_ERR_INVALID_ARG),
    (dict(L=-64), bd.BD_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), bd.BD_ERR_INVALID_ARG),
    (dict(L=60, b=8), bd.BD_ERR_INVALID_ARG),
    (dict(scale=0.0), bd.BD_ERR_INVALID_ARG),
    (dict(scale=float("nan")), bd.BD_ERR_INVALID_ARG),
    (dict(d=96), bd.BD_ERR_UNSUPPORTED),
    (dict(d=256), bd.BD_ERR_UNSUPPORTED),
])
def test_fwd_rejects(lib, kw, status):
    assert bd.bd_attn_fwd(**fwd_args(**kw)) == status


def dec_args(**kw):
    a = dict(q_blk=A, k_cache=A, v_cache=A, cache_len=A, out=A, lse=A, B=2,
             Hq=4, Hkv=2, b=8, d=64, intra_block_mode=0, stream=None, S_cap=64,
             workspace=A, workspace_bytes=1 << 30)
    a.update(kw)
    return a


@pytest.mark.parametrize("kw,status", [
    (dict(cache_len=None), bd.BD_ERR_INVALID_ARG),
    (dict(v_cache=A + 4), bd.BD_ERR_INVALID_ARG),
    (dict(cache_len=A + 2), bd.BD_ERR_INVALID_ARG),
    (dict(Hq=3), bd.BD_ERR_INVALID_ARG),
    (dict(S_cap=4), bd.BD_ERR_INVALID_ARG),
    (dict(intra_block_mode=3), bd.BD_ERR_INVALID_ARG),
    (dict(intra_block_mode=-1), bd.BD_ERR_INVALID_ARG),
    (dict(b=0), bd.BD_ERR_INVALID_ARG),
    (dict(workspace_bytes=16), bd.BD_ERR_INVALID_ARG),
    (dict(workspace=A + 16), bd.BD_ERR_INVALID_ARG),
    (dict(d=80), bd.BD_ERR_UNSUPPORTED),
])
def test_decode_rejects(lib, kw, status):
    assert bd.bd_attn_decode(**dec_args(**kw)) == status


def test_product_path_does_not_touch_the_oracle():
    """The library sources and the binding never name the oracle."""
    pkg = os.path.join(ROOT, "block_diffusion_lm_attn_b200")
    for dp, _, fns in os.walk(pkg):
        for fn in fns:
            if fn.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                txt = open(os.path.join(dp, fn)).read()
                assert "oracle" not in txt.lower(), fn


def test_fault_hook_rejects_unknown_kind(lib):
    assert bd.bd_attn_debug_inject_fault(7) == bd.BD_ERR_INVALID_ARG


def test_grid_hook_rejects_out_of_range(lib):
    assert bd.bd_attn_debug_set_grid(-1) == bd.BD_ERR_INVALID_ARG
    assert bd.bd_attn_debug_set_grid(149) == bd.BD_ERR_INVALID_ARG
    assert bd.bd_attn_debug_set_grid(0) == bd.BD_OK
    assert bd.bd_attn_debug_set_chunk(-1) == bd.BD_ERR_INVALID_ARG
    assert bd.bd_attn_debug_set_chunk(0) == bd.BD_OK


def test_cache_and_sprint_reject_bad_arguments(lib):
    I = bd.BD_ERR_INVALID_ARG
    U = bd.BD_ERR_UNSUPPORTED
    assert bd.bd_spec_accept(None, A, A, 4, 8, None) == I
    assert bd.bd_spec_accept(A, A + 2, A, 4, 8, None) == I
    assert bd.bd_spec_accept(A, A, A, 0, 8, None) == I
    # k_new and v_new must be both given or both NULL
    assert bd.bd_cache_append(A, A, A, A, None, A, 2, 2, 4, 64, 32, None) == I
    assert bd.bd_cache_append(A, A + 8, A, None, None, A, 2, 2, 4, 64, 32, None) == I
    assert bd.bd_cache_append(A, A, A, None, None, A, 2, 2, 4, 80, 32, None) == U
    assert bd.bd_cache_crop(A, 4, -1, None) == I
    assert bd.bd_cache_crop(None, 4, 3, None) == I
    ws = bd.bd_sprint_workspace_bytes(2, 64)
    assert ws > 0 and ws % 256 == 0 and bd.bd_sprint_workspace_bytes(0, 64) == 0

    def sp(**kw):
        a = dict(k_cache=A, v_cache=A + 4096, cache_len=A, conf=A, modality=A,
                 alpha=0.5, keep_text=1.0, keep_image=0.8, k_out=A + 8192,
                 v_out=A + 12288, kept=A, new_len=A, score=None, B=2, Hkv=2,
                 d=64, S_cap=64, stream=None, workspace=A, workspace_bytes=ws)
        a.update(kw)
        return bd.bd_sprint_prune(**a)
    assert sp(conf=None) == I
    assert sp(alpha=1.5) == I
    assert sp(keep_image=-0.1) == I
    assert sp(keep_text=float("nan")) == I
    assert sp(k_out=A) == I                  # output aliases the input cache
    assert sp(workspace_bytes=ws - 1) == I
    assert sp(workspace=A + 16) == I
    assert sp(score=A + 4) == I
    assert sp(d=48) == U
    assert sp(S_cap=65537, workspace_bytes=1 << 40) == U
