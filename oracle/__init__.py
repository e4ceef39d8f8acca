"""Plain fp64 CPU oracle for block-diffusion attention.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are its only users.  The CUDA library never
imports, links or calls it; the two share no code.

The arithmetic lives in ``bd_oracle.c`` (plain C, fp64, OpenMP over query
rows).  This module compiles it with gcc on first use and marshals arrays
through ctypes; it adds no arithmetic of its own.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
(hand-written mask fixtures, closed forms, library-routine special cases and
invariants); none is unpinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bd_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libbdoracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle to a shared library with gcc (-O2, OpenMP)."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    tmp = out + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-shared", "-fPIC",
           "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


_i64p = ctypes.POINTER(ctypes.c_int64)
_i32p = ctypes.POINTER(ctypes.c_int32)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_f64p = ctypes.POINTER(ctypes.c_double)
_f32p = ctypes.POINTER(ctypes.c_float)
_u8p = ctypes.POINTER(ctypes.c_uint8)


def _bind(lib):
    lib.bdo_max_threads.restype = ctypes.c_int
    lib.bdo_fwd_sees.restype = ctypes.c_int
    lib.bdo_fwd_sees.argtypes = [ctypes.c_int] * 4
    lib.bdo_decode_sees.restype = ctypes.c_int
    lib.bdo_decode_sees.argtypes = [ctypes.c_int] * 5
    lib.bdo_fwd_rows.restype = ctypes.c_int
    lib.bdo_fwd_rows.argtypes = [_u16p, _u16p, _u16p] + [ctypes.c_int] * 6 + [
        ctypes.c_double, _i64p, ctypes.c_int64, _f64p, _f64p]
    lib.bdo_decode_rows.restype = ctypes.c_int
    lib.bdo_decode_rows.argtypes = [_u16p, _u16p, _u16p, _i32p] + [
        ctypes.c_int] * 7 + [ctypes.c_double, _i64p, ctypes.c_int64, _f64p,
                             _f64p]
    lib.bdo_fwd_row_probs.restype = ctypes.c_int
    lib.bdo_fwd_row_probs.argtypes = [_u16p, _u16p] + [ctypes.c_int] * 6 + [
        ctypes.c_double, ctypes.c_int64, _f64p]
    lib.bdo_fwd_mask.restype = ctypes.c_int
    lib.bdo_fwd_mask.argtypes = [ctypes.c_int, ctypes.c_int, _u8p]
    lib.bdo_sprint_select.restype = ctypes.c_int
    lib.bdo_sprint_select.argtypes = [_u16p, _i32p, _f32p, _u8p] + [
        ctypes.c_int] * 4 + [ctypes.c_float] * 3 + [_f64p, _i32p, _i32p]
    lib.bdo_combine.restype = None
    lib.bdo_combine.argtypes = [ctypes.c_int, ctypes.c_int, _f64p, _f64p,
                                _f64p, _f64p]
    return lib


def load(path: str | None = None):
    """Load (compiling first if needed) the oracle library.  ``path`` loads a
    separately compiled copy instead (used by the mutation tests)."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _bits(t) -> np.ndarray:
    """bf16 tensor (torch, CPU) or uint16 array -> contiguous uint16 bits."""
    if isinstance(t, np.ndarray):
        assert t.dtype == np.uint16
        return np.ascontiguousarray(t)
    import torch
    assert t.dtype == torch.bfloat16, t.dtype
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(
        np.uint16)


def _ptr(a: np.ndarray, typ):
    return a.ctypes.data_as(typ)


def max_threads(lib=None) -> int:
    return int((lib or load()).bdo_max_threads())


def fwd_sees(L: int, b: int, r: int, c: int, lib=None) -> bool:
    return bool((lib or load()).bdo_fwd_sees(L, b, r, c))


def decode_sees(cache_len: int, b: int, mode: int, j: int, c: int,
                lib=None) -> bool:
    return bool((lib or load()).bdo_decode_sees(cache_len, b, mode, j, c))


def fwd(q, k, v, L: int, b: int, scale: float, rows=None, lib=None):
    """Training/prefill form.  q: [B,Hq,2L,d] bf16; k, v: [B,Hkv,2L,d] bf16.

    Returns (out, lse) in fp64: [B,Hq,2L,d] and [B,Hq,2L] when ``rows`` is
    None, else [n,d] and [n] for the flat row ids in ``rows``."""
    lib = lib or load()
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    assert N == 2 * L and tuple(k.shape) == (B, Hkv, N, d)
    assert tuple(v.shape) == tuple(k.shape)
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    if rows is None:
        n = B * Hq * N
        rp = None
    else:
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        n = rows.size
        rp = _ptr(rows, _i64p)
    out = np.empty((n, d), np.float64)
    lse = np.empty((n,), np.float64)
    rc = lib.bdo_fwd_rows(_ptr(qb, _u16p), _ptr(kb, _u16p), _ptr(vb, _u16p),
                          B, Hq, Hkv, L, b, d, float(scale), rp, n,
                          _ptr(out, _f64p), _ptr(lse, _f64p))
    if rc != 0:
        raise ValueError("oracle fwd rejected its arguments")
    if rows is None:
        return out.reshape(B, Hq, N, d), lse.reshape(B, Hq, N)
    return out, lse


def decode(q_blk, k_cache, v_cache, cache_len, mode: int, scale: float,
           rows=None, lib=None):
    """Block-decode form.  q_blk: [B,Hq,b,d]; caches [B,Hkv,S_cap,d];
    cache_len: int sequence of B; mode 0 (bidirectional block), 1 (causal
    block) or 2 (prefix only).  Returns fp64 (out, lse) shaped
    [B,Hq,b,d], [B,Hq,b] (or [n,d], [n] for ``rows``)."""
    lib = lib or load()
    B, Hq, b, d = q_blk.shape
    Hkv, S_cap = k_cache.shape[1], k_cache.shape[2]
    assert tuple(k_cache.shape) == (B, Hkv, S_cap, d)
    assert tuple(v_cache.shape) == tuple(k_cache.shape)
    qb, kb, vb = _bits(q_blk), _bits(k_cache), _bits(v_cache)
    lens = np.ascontiguousarray(np.asarray(cache_len, dtype=np.int32))
    assert lens.shape == (B,)
    if rows is None:
        n = B * Hq * b
        rp = None
    else:
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        n = rows.size
        rp = _ptr(rows, _i64p)
    out = np.empty((n, d), np.float64)
    lse = np.empty((n,), np.float64)
    rc = lib.bdo_decode_rows(_ptr(qb, _u16p), _ptr(kb, _u16p), _ptr(vb, _u16p),
                             _ptr(lens, _i32p), B, Hq, Hkv, b, d, S_cap,
                             int(mode), float(scale), rp, n, _ptr(out, _f64p),
                             _ptr(lse, _f64p))
    if rc != 0:
        raise ValueError("oracle decode rejected its arguments")
    if rows is None:
        return out.reshape(B, Hq, b, d), lse.reshape(B, Hq, b)
    return out, lse


def fwd_row_probs(q, k, L: int, b: int, scale: float, row: int, lib=None):
    """Attention probabilities of one flat query row over all 2L keys."""
    lib = lib or load()
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    qb, kb = _bits(q), _bits(k)
    p = np.empty((N,), np.float64)
    rc = lib.bdo_fwd_row_probs(_ptr(qb, _u16p), _ptr(kb, _u16p), B, Hq, Hkv,
                               L, b, d, float(scale), int(row),
                               _ptr(p, _f64p))
    if rc != 0:
        raise ValueError("oracle probs rejected its arguments")
    return p


def combine(o_parts, lse_parts, lib=None):
    """Merge per-part (o_s [n,d], lse_s [n]) of one row into (out [d], lse)."""
    lib = lib or load()
    o = np.ascontiguousarray(np.asarray(o_parts, dtype=np.float64))
    l_ = np.ascontiguousarray(np.asarray(lse_parts, dtype=np.float64))
    n, d = o.shape
    out = np.empty((d,), np.float64)
    lse = np.empty((1,), np.float64)
    lib.bdo_combine(n, d, _ptr(o, _f64p), _ptr(l_, _f64p), _ptr(out, _f64p),
                    _ptr(lse, _f64p))
    return out, float(lse[0])


def fwd_mask(L: int, b: int, lib=None) -> np.ndarray:
    """The training/prefill visibility predicate as a dense [2L, 2L] bool
    matrix (row = query position, column = key position)."""
    lib = lib or load()
    m = np.empty((2 * L, 2 * L), np.uint8)
    if lib.bdo_fwd_mask(L, b, _ptr(m, _u8p)) != 0:
        raise ValueError("oracle mask rejected its arguments")
    return m.astype(bool)


def sprint_select(k_cache, cache_len, conf, modality, alpha=0.5,
                  keep_text=1.0, keep_image=0.8, lib=None):
    """Sparse prefix retention scores and kept positions.

    k_cache [B,Hkv,S_cap,d] bf16; cache_len [B]; conf [B,S_cap] fp32 top-1
    confidences; modality [B,S_cap] uint8 (0 text, else image).  Returns
    (score [B,S_cap] fp64, kept [B,S_cap] int32 -- kept positions in order,
    then -1 --, new_len [B] int32).  alpha and the keep ratios are rounded
    to single precision first, as the library's interface takes them."""
    lib = lib or load()
    B, Hkv, S_cap, d = k_cache.shape
    kb = _bits(k_cache)
    lens = np.ascontiguousarray(np.asarray(cache_len, dtype=np.int32))
    cf = np.ascontiguousarray(np.asarray(conf, dtype=np.float32))
    md = np.ascontiguousarray(np.asarray(modality, dtype=np.uint8))
    assert lens.shape == (B,) and cf.shape == (B, S_cap) and md.shape == (B, S_cap)
    score = np.empty((B, S_cap), np.float64)
    kept = np.empty((B, S_cap), np.int32)
    new_len = np.empty((B,), np.int32)
    rc = lib.bdo_sprint_select(_ptr(kb, _u16p), _ptr(lens, _i32p),
                               _ptr(cf, _f32p), _ptr(md, _u8p), B, Hkv, d,
                               S_cap, float(alpha), float(keep_text),
                               float(keep_image), _ptr(score, _f64p),
                               _ptr(kept, _i32p), _ptr(new_len, _i32p))
    if rc != 0:
        raise ValueError("oracle sprint_select rejected its arguments")
    return score, kept, new_len
