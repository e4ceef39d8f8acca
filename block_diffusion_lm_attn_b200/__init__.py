"""Python binding of libbdattn.so, the B200 block-diffusion attention library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/bd_attn.h``.  There is no
CPU or PyTorch fallback; if the library is missing or cannot be loaded,
every call raises.

Two layers:
  * ``bd_attn_fwd`` / ``bd_attn_decode`` / ``bd_attn_decode_workspace_bytes``
    / ``bd_attn_get_device_status`` / ``bd_attn_status_string`` take the C
    arguments one to one (device pointers as ints, stream as an int handle)
    and return the status code.
  * ``fwd`` / ``decode`` take torch CUDA tensors, check shapes, allocate the
    outputs if not given, call the C entry point on the current stream and
    raise ``BdAttnError`` on a non-OK status.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbdattn.so")

BD_OK = 0
BD_ERR_INVALID_ARG = 1
BD_ERR_UNSUPPORTED = 2
BD_ERR_CUDA = 3
BD_ERR_DEVICE_TIMEOUT = 4

EXPORTED = ("bd_attn_fwd", "bd_attn_decode", "bd_attn_decode_workspace_bytes",
            "bd_attn_get_device_status", "bd_attn_status_string",
            "bd_spec_accept", "bd_cache_append", "bd_cache_crop",
            "bd_sprint_prune", "bd_sprint_workspace_bytes", "bd_attn_bwd",
            "bd_attn_bwd_workspace_bytes")


class BdAttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__("%s failed: %s (status %d)" %
                         (what, bd_attn_status_string(status), status))
        self.status = status


_lib = None


def load(path: str = LIB_PATH):
    """Load libbdattn.so (built by ``build.build()``); raises if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(
            "libbdattn.so not built at %s: run "
            "`python -m block_diffusion_lm_attn_b200.build`" % path)
    lib = ctypes.CDLL(path)
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.bd_attn_fwd.restype = i
    lib.bd_attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, vp]
    lib.bd_attn_decode.restype = i
    lib.bd_attn_decode.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i,
                                   vp, i, vp, ctypes.c_size_t]
    lib.bd_attn_decode_workspace_bytes.restype = ctypes.c_size_t
    lib.bd_attn_decode_workspace_bytes.argtypes = [i, i, i, i, i, i]
    lib.bd_attn_get_device_status.restype = i
    lib.bd_attn_get_device_status.argtypes = [vp]
    lib.bd_attn_status_string.restype = ctypes.c_char_p
    lib.bd_attn_status_string.argtypes = [i]
    lib.bd_attn_bwd.restype = i
    lib.bd_attn_bwd.argtypes = [vp] * 9 + [i, i, i, i, i, i, f, vp, vp,
                                           ctypes.c_size_t]
    lib.bd_attn_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.bd_attn_bwd_workspace_bytes.argtypes = [i, i, i]
    lib.bd_spec_accept.restype = i
    lib.bd_spec_accept.argtypes = [vp, vp, vp, i, i, vp]
    lib.bd_cache_append.restype = i
    lib.bd_cache_append.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp]
    lib.bd_cache_crop.restype = i
    lib.bd_cache_crop.argtypes = [vp, i, i, vp]
    lib.bd_sprint_prune.restype = i
    lib.bd_sprint_prune.argtypes = [vp, vp, vp, vp, vp, f, f, f, vp, vp, vp,
                                    vp, vp, i, i, i, i, vp, vp,
                                    ctypes.c_size_t]
    lib.bd_sprint_workspace_bytes.restype = ctypes.c_size_t
    lib.bd_sprint_workspace_bytes.argtypes = [i, i]
    _lib = lib
    return lib


# ---------------------------------------------------------------------------
# one-to-one C entry points


def bd_attn_fwd(q, k, v, out, lse, B, Hq, Hkv, L, b, d, scale, stream):
    return load().bd_attn_fwd(q, k, v, out, lse, B, Hq, Hkv, L, b, d, scale,
                              stream)


def bd_attn_decode(q_blk, k_cache, v_cache, cache_len, out, lse, B, Hq, Hkv,
                   b, d, intra_block_mode, stream, S_cap, workspace,
                   workspace_bytes):
    return load().bd_attn_decode(q_blk, k_cache, v_cache, cache_len, out, lse,
                                 B, Hq, Hkv, b, d, intra_block_mode, stream,
                                 S_cap, workspace, workspace_bytes)


def bd_attn_decode_workspace_bytes(B, Hq, Hkv, b, d, S_cap):
    return int(load().bd_attn_decode_workspace_bytes(B, Hq, Hkv, b, d, S_cap))


def bd_attn_get_device_status(stream):
    return load().bd_attn_get_device_status(stream)


def bd_attn_status_string(status):
    return load().bd_attn_status_string(status).decode()


def bd_attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, Hq, Hkv, L, b, d,
                scale, stream, workspace, workspace_bytes):
    return load().bd_attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, Hq, Hkv,
                              L, b, d, scale, stream, workspace,
                              workspace_bytes)


def bd_attn_bwd_workspace_bytes(B, Hq, L):
    return int(load().bd_attn_bwd_workspace_bytes(B, Hq, L))


def bd_spec_accept(draft, target, n_accept, B, b, stream):
    return load().bd_spec_accept(draft, target, n_accept, B, b, stream)


def bd_cache_append(k_cache, v_cache, cache_len, k_new, v_new, n_new, B, Hkv,
                    b, d, S_cap, stream):
    return load().bd_cache_append(k_cache, v_cache, cache_len, k_new, v_new,
                                  n_new, B, Hkv, b, d, S_cap, stream)


def bd_cache_crop(cache_len, B, max_len, stream):
    return load().bd_cache_crop(cache_len, B, max_len, stream)


def bd_sprint_prune(k_cache, v_cache, cache_len, conf, modality, alpha,
                    keep_text, keep_image, k_out, v_out, kept, new_len, score,
                    B, Hkv, d, S_cap, stream, workspace, workspace_bytes):
    return load().bd_sprint_prune(k_cache, v_cache, cache_len, conf, modality,
                                  alpha, keep_text, keep_image, k_out, v_out,
                                  kept, new_len, score, B, Hkv, d, S_cap,
                                  stream, workspace, workspace_bytes)


def bd_sprint_workspace_bytes(B, S_cap):
    return int(load().bd_sprint_workspace_bytes(B, S_cap))


def bd_attn_debug_inject_fault(kind):
    """Test hook (include/bd_attn_debug.h): arm (1) or disarm (0) a one-shot
    fault that makes a bounded wait of the next head-dim-128 launch run out."""
    fn = load().bd_attn_debug_inject_fault
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_int]
    return fn(kind)


def bd_attn_debug_fwd_kernel(Hq, Hkv, d):
    """Test hook (include/bd_attn_debug.h): which forward kernel runs for
    these sizes (2 paired tcgen05, 1 one-tile tcgen05, 0 mma.sync, -1 none)."""
    fn = load().bd_attn_debug_fwd_kernel
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_int] * 3
    return fn(Hq, Hkv, d)


def bd_attn_debug_reset_sched():
    """Test hook (include/bd_attn_debug.h): synchronise the device and zero
    every work-counter pair of the persistent kernels."""
    fn = load().bd_attn_debug_reset_sched
    fn.restype = ctypes.c_int
    fn.argtypes = []
    return fn()


def bd_attn_debug_set_grid(ctas):
    """Test hook (include/bd_attn_debug.h): cap the grid of the persistent
    head-dim-128 kernels at `ctas` CTAs (0 restores one CTA per SM)."""
    fn = load().bd_attn_debug_set_grid
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_int]
    return fn(ctas)


def bd_attn_debug_set_chunk(groups):
    """Test hook (include/bd_attn_debug.h): fix the chunk size of the work
    lists at `groups` heads / head pairs / kv-head groups (0 restores the
    defaults)."""
    fn = load().bd_attn_debug_set_chunk
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_int]
    return fn(groups)


# ---------------------------------------------------------------------------
# torch-tensor conveniences


def _stream_handle(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def fwd(q, k, v, L: int, b: int, scale: float | None = None, out=None,
        lse=None, stream=None):
    """Training/prefill block-diffusion attention on CUDA tensors.

    q [B,Hq,2L,d], k, v [B,Hkv,2L,d] bf16 contiguous.  Returns (out, lse)."""
    import torch
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if N != 2 * L or tuple(k.shape) != (B, Hkv, N, d) or v.shape != k.shape:
        raise ValueError("shape mismatch")
    for t in (q, k, v):
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()):
            raise ValueError("q, k, v must be contiguous bf16 CUDA tensors")
    if scale is None:
        scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, N), device=q.device, dtype=torch.float32)
    st = bd_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                     lse.data_ptr(), B, Hq, Hkv, L, b, d, float(scale),
                     _stream_handle(stream))
    if st != BD_OK:
        raise BdAttnError(st, "bd_attn_fwd")
    return out, lse


def bwd(q, k, v, out, lse, dout, L: int, b: int, scale: float | None = None,
        dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Backward of ``fwd``: gradients of q, k, v given dout (the gradient of
    out), out and lse from the forward.  Returns (dq, dk, dv)."""
    import torch
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if N != 2 * L or tuple(k.shape) != (B, Hkv, N, d) or v.shape != k.shape:
        raise ValueError("shape mismatch")
    if out.shape != q.shape or dout.shape != q.shape or tuple(lse.shape) != (B, Hq, N):
        raise ValueError("shape mismatch")
    for t_, w in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _check(t_, torch.bfloat16, w)
    _check(lse, torch.float32, "lse")
    if scale is None:
        scale = d ** -0.5
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    nb = bd_attn_bwd_workspace_bytes(B, Hq, L)
    if workspace is None:
        workspace = torch.empty(nb, dtype=torch.uint8, device=q.device)
    st = bd_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                     lse.data_ptr(), dout.data_ptr(), dq.data_ptr(),
                     dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, L, b, d,
                     float(scale), _stream_handle(stream), workspace.data_ptr(),
                     workspace.numel() * workspace.element_size())
    if st != BD_OK:
        raise BdAttnError(st, "bd_attn_bwd")
    return dq, dk, dv


def decode(q_blk, k_cache, v_cache, cache_len, mode: int, out=None, lse=None,
           workspace=None, stream=None):
    """Block-decode attention on CUDA tensors.

    q_blk [B,Hq,b,d]; k_cache, v_cache [B,Hkv,S_cap,d] bf16; cache_len int32
    [B] on the device; mode 0 bidirectional, 1 causal, 2 cross-attention to
    the prefix only.  ``workspace`` is an
    optional uint8 CUDA tensor of at least ``workspace_bytes(...)`` bytes
    (None: the library's own per-device buffer).  Returns (out, lse)."""
    import torch
    B, Hq, b, d = q_blk.shape
    Hkv, S_cap = k_cache.shape[1], k_cache.shape[2]
    if tuple(k_cache.shape) != (B, Hkv, S_cap, d) or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    if not (cache_len.is_cuda and cache_len.dtype == torch.int32
            and cache_len.numel() == B):
        raise ValueError("cache_len must be an int32 CUDA tensor of B entries")
    for t in (q_blk, k_cache, v_cache):
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()):
            raise ValueError("q_blk and caches must be contiguous bf16 CUDA")
    if out is None:
        out = torch.empty_like(q_blk)
    if lse is None:
        lse = torch.empty((B, Hq, b), device=q_blk.device, dtype=torch.float32)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    st = bd_attn_decode(q_blk.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                        cache_len.data_ptr(), out.data_ptr(), lse.data_ptr(),
                        B, Hq, Hkv, b, d, int(mode), _stream_handle(stream),
                        S_cap, ws_ptr, ws_bytes)
    if st != BD_OK:
        raise BdAttnError(st, "bd_attn_decode")
    return out, lse


def _check(t, dtype, what):
    import torch
    if not (t.is_cuda and t.dtype == dtype and t.is_contiguous()):
        raise ValueError("%s must be a contiguous %s CUDA tensor" % (what, dtype))


def spec_accept(draft, target, n_accept=None, stream=None):
    """Longest matching prefix of draft and target ([B, b] int32 CUDA).
    Returns n_accept [B] int32 on the device."""
    import torch
    _check(draft, torch.int32, "draft")
    _check(target, torch.int32, "target")
    B, b = draft.shape
    if tuple(target.shape) != (B, b):
        raise ValueError("shape mismatch")
    if n_accept is None:
        n_accept = torch.empty(B, dtype=torch.int32, device=draft.device)
    st = bd_spec_accept(draft.data_ptr(), target.data_ptr(),
                        n_accept.data_ptr(), B, b, _stream_handle(stream))
    if st != BD_OK:
        raise BdAttnError(st, "bd_spec_accept")
    return n_accept


def cache_append(k_cache, v_cache, cache_len, n_new, k_new=None, v_new=None,
                 stream=None):
    """Append rows 0..n_new[i]-1 of k_new/v_new [B,Hkv,b,d] (or of the rows
    already at the cache tail, if None) and advance cache_len, in place."""
    import torch
    B, Hkv, S_cap, d = k_cache.shape
    for t, w in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        _check(t, torch.bfloat16, w)
    _check(cache_len, torch.int32, "cache_len")
    _check(n_new, torch.int32, "n_new")
    if k_new is None:
        b = S_cap
        kp = vp = None
    else:
        b = k_new.shape[2]
        kp, vp = k_new.data_ptr(), v_new.data_ptr()
    st = bd_cache_append(k_cache.data_ptr(), v_cache.data_ptr(),
                         cache_len.data_ptr(), kp, vp, n_new.data_ptr(), B,
                         Hkv, b, d, S_cap, _stream_handle(stream))
    if st != BD_OK:
        raise BdAttnError(st, "bd_cache_append")


def cache_crop(cache_len, max_len: int, stream=None):
    import torch
    _check(cache_len, torch.int32, "cache_len")
    st = bd_cache_crop(cache_len.data_ptr(), cache_len.numel(), int(max_len),
                       _stream_handle(stream))
    if st != BD_OK:
        raise BdAttnError(st, "bd_cache_crop")


def sprint_prune(k_cache, v_cache, cache_len, conf, modality, alpha=0.5,
                 keep_text=1.0, keep_image=0.8, k_out=None, v_out=None,
                 want_score=False, workspace=None, stream=None):
    """Sparse prefix retention on CUDA tensors.  Returns (k_out, v_out,
    kept [B,S_cap] int32, new_len [B] int32, score [B,S_cap] fp64 or None)."""
    import torch
    B, Hkv, S_cap, d = k_cache.shape
    for t, w in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        _check(t, torch.bfloat16, w)
    _check(cache_len, torch.int32, "cache_len")
    _check(conf, torch.float32, "conf")
    _check(modality, torch.uint8, "modality")
    dev = k_cache.device
    if k_out is None:
        k_out = torch.empty_like(k_cache)
    if v_out is None:
        v_out = torch.empty_like(v_cache)
    kept = torch.empty((B, S_cap), dtype=torch.int32, device=dev)
    new_len = torch.empty(B, dtype=torch.int32, device=dev)
    score = (torch.zeros((B, S_cap), dtype=torch.float64, device=dev)
             if want_score else None)
    nb = bd_sprint_workspace_bytes(B, S_cap)
    if workspace is None:
        workspace = torch.empty(nb, dtype=torch.uint8, device=dev)
    st = bd_sprint_prune(k_cache.data_ptr(), v_cache.data_ptr(),
                         cache_len.data_ptr(), conf.data_ptr(),
                         modality.data_ptr(), float(alpha), float(keep_text),
                         float(keep_image), k_out.data_ptr(), v_out.data_ptr(),
                         kept.data_ptr(), new_len.data_ptr(),
                         score.data_ptr() if score is not None else None,
                         B, Hkv, d, S_cap, _stream_handle(stream),
                         workspace.data_ptr(),
                         workspace.numel() * workspace.element_size())
    if st != BD_OK:
        raise BdAttnError(st, "bd_sprint_prune")
    return k_out, v_out, kept, new_len, score


def workspace_bytes(B, Hq, Hkv, b, d, S_cap) -> int:
    return bd_attn_decode_workspace_bytes(B, Hq, Hkv, b, d, S_cap)


def device_status(stream=None) -> int:
    return bd_attn_get_device_status(_stream_handle(stream))


def bd_attn_decode_noalloc(q_blk, k_cache, v_cache, cache_len, out, lse, B,
                           Hq, Hkv, b, d, intra_block_mode, stream, S_cap):
    """One-to-one binding of the C entry point that decodes without
    allocating: its split-KV scratch is a fixed array inside the library
    (see include/bd_attn.h), for callers that cannot allocate device memory
    at decode time."""
    fn = load().bd_attn_decode_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.restype = i
    fn.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp, i]
    return fn(q_blk, k_cache, v_cache, cache_len, out, lse, B, Hq, Hkv, b, d,
              intra_block_mode, stream, S_cap)
