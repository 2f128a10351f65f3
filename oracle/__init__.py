"""fp64 CPU oracle for paged-KV-cache attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It wraps ``pkv_oracle.c`` (plain C,
OpenMP over query rows) through ctypes and shares no code with the CUDA
library: it does not import ``paged_kv_cache_380_b200`` and that package does
not import it.

Typed arrays are passed as numpy arrays plus a dtype tag:
``'f32'`` (float32), ``'bf16'`` (uint16 bit patterns), ``'f16'`` (float16 or
uint16 bits), ``'i8'`` (int8 codes, with fp16 scales), ``'f64'`` (float64).

Every function cites the definition it follows in ``pkv_oracle.c``'s header
(attention over a KV cache, the paged layout and block table, GQA head
mapping, bottom-right causal alignment of a prefill chunk, symmetric INT8
quantisation, slot-mapping scatter).
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pkv_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

DTYPES = {"f32": 0, "bf16": 1, "f16": 2, "i8": 3, "f64": 4}
_NP = {"f32": np.float32, "bf16": np.uint16, "f16": np.uint16, "i8": np.int8, "f64": np.float64}
_ERRORS = {-1: "bad argument", -2: "index out of range", -3: "out of memory"}


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, strict IEEE: no fast-math)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-fno-fast-math", "-ffp-contract=off", "-o", tmp, src, "-lm"])
        os.replace(tmp, out)
    return out


def _open(path):
    lib = ctypes.CDLL(path)
    P, I, I64, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.oracle_decode.argtypes = [P, I, P, P, I, P, P, P, P, D, I, I, I, I, I, I, I, I64,
                                  P, I64, P, P]
    lib.oracle_prefill.argtypes = [P, I, P, P, I, P, P, P, P, P, I, D, I, I, I, I, I, I, I,
                                   I64, P, I64, P, P]
    lib.oracle_kv_cache_write.argtypes = [P, P, P, I64, P, P, I64, I64]
    lib.oracle_quantize_int8.argtypes = [P, I, I64, I, P, P]
    lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_to_double.restype = D
    lib.oracle_f16_to_double.argtypes = [ctypes.c_uint16]
    lib.oracle_f16_to_double.restype = D
    lib.oracle_float_to_f16.argtypes = [ctypes.c_float]
    lib.oracle_float_to_f16.restype = ctypes.c_uint16
    lib.oracle_set_threads.argtypes = [I]
    lib.oracle_max_threads.restype = I
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _open(build())
    return _lib


@contextlib.contextmanager
def using_library(path: str):
    """Temporarily route every oracle call through another build of the C
    source (the mutation tests use this to check that the pins catch planted
    mistakes)."""
    global _lib
    _load()
    old = _lib
    _lib = _open(path)
    try:
        yield
    finally:
        _lib = old


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _typed(a, tag):
    want = _NP[tag]
    a = np.ascontiguousarray(a)
    if tag == "f16" and a.dtype == np.float16:
        a = a.view(np.uint16)
    if a.dtype != want:
        raise TypeError(f"dtype tag {tag!r} expects {np.dtype(want)}, got {a.dtype}")
    return a


def _check(rc):
    if rc != 0:
        raise ValueError(f"oracle: {_ERRORS.get(rc, rc)}")


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def bf16_to_f64(bits) -> np.ndarray:
    """Exact widening of bf16 bit patterns (element-wise through the C decoder)."""
    lib = _load()
    b = np.asarray(bits, dtype=np.uint16)
    return np.array([lib.oracle_bf16_to_double(int(x)) for x in b.ravel()]).reshape(b.shape)


def f16_to_f64(bits) -> np.ndarray:
    lib = _load()
    b = np.asarray(bits).view(np.uint16) if np.asarray(bits).dtype == np.float16 else np.asarray(bits, np.uint16)
    return np.array([lib.oracle_f16_to_double(int(x)) for x in b.ravel()]).reshape(b.shape)


def float_to_f16_bits(x) -> np.ndarray:
    lib = _load()
    a = np.asarray(x, dtype=np.float32)
    return np.array([lib.oracle_float_to_f16(float(v)) for v in a.ravel()],
                    dtype=np.uint16).reshape(a.shape)


def kv_cache_write(k, v, slot_mapping, k_pool, v_pool):
    """Scatter rows of k/v ([T, ...]) into the pools ([P, ps, ...]) in place.

    Row t goes to slot slot_mapping[t] (= page * page_size + offset); negative
    slots are skipped.  Byte copy, so any dtype works.
    """
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    if not (k_pool.flags.c_contiguous and v_pool.flags.c_contiguous):
        raise ValueError("pools must be C-contiguous (written in place)")
    T = sm.shape[0]
    if k.shape[0] != T or v.shape != k.shape or k.dtype != k_pool.dtype:
        raise ValueError("shape/dtype mismatch")
    row_bytes = k[0].nbytes if T else 1
    num_slots = k_pool.nbytes // row_bytes
    if T and (k_pool.nbytes % row_bytes or v_pool.nbytes != k_pool.nbytes):
        raise ValueError("pool is not a whole number of rows")
    _check(_load().oracle_kv_cache_write(_ptr(k), _ptr(v), _ptr(sm), T, _ptr(k_pool),
                                         _ptr(v_pool), row_bytes, num_slots))


def quantize_int8(x, tag: str):
    """Symmetric INT8 quantisation of the last axis (one fp16 scale per row).

    Returns (codes int8 with x's shape, scales uint16 fp16 bits with x's shape
    minus the last axis).
    """
    x = _typed(x, tag)
    d = x.shape[-1]
    rows = x.size // d
    codes = np.empty(x.shape, dtype=np.int8)
    scales = np.empty(x.shape[:-1], dtype=np.uint16)
    _check(_load().oracle_quantize_int8(_ptr(x), DTYPES[tag], rows, d, _ptr(codes), _ptr(scales)))
    return codes, scales


def _sel(sel):
    if sel is None:
        return None, 0
    s = np.ascontiguousarray(sel, dtype=np.int64)
    return s, s.shape[0]


def decode(q, q_tag, k_pages, v_pages, kv_tag, block_tables, context_lens, scale,
           k_scales=None, v_scales=None, items=None, return_lse=False, window=0):
    """fp64 decode attention: one query row per sequence.

    q [B, Hq, D]; pools [P, ps, Hkv, D]; block_tables int32 [B, MP];
    context_lens int32 [B].  ``items`` selects flat (b*Hq + h) rows; the
    result is then [len(items), D], else [B, Hq, D].  ``window`` > 0 keeps only
    the last ``window`` keys (local attention).
    """
    q = _typed(q, q_tag)
    kp = _typed(k_pages, kv_tag)
    vp = _typed(v_pages, kv_tag)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    B, Hq, D = q.shape
    P, ps, Hkv, D2 = kp.shape
    assert D2 == D and vp.shape == kp.shape and bt.shape[0] == B and cl.shape == (B,)
    ks = vs = None
    if kv_tag == "i8":
        ks = np.ascontiguousarray(k_scales, dtype=np.uint16)
        vs = np.ascontiguousarray(v_scales, dtype=np.uint16)
        assert ks.shape == (P, ps, Hkv) and vs.shape == ks.shape
    sel, n_sel = _sel(items)
    n_out = n_sel if sel is not None else B * Hq
    out = np.zeros((n_out, D), dtype=np.float64)
    lse = np.zeros(n_out, dtype=np.float64)
    _check(_load().oracle_decode(_ptr(q), DTYPES[q_tag], _ptr(kp), _ptr(vp), DTYPES[kv_tag],
                                 _ptr(ks), _ptr(vs), _ptr(bt), _ptr(cl), float(scale), int(window), B, Hq, Hkv,
                                 D, ps, bt.shape[1], P, _ptr(sel), n_sel, _ptr(out), _ptr(lse)))
    if sel is None:
        out = out.reshape(B, Hq, D)
        lse = lse.reshape(B, Hq)
    return (out, lse) if return_lse else out


def prefill(q, q_tag, k_pages, v_pages, kv_tag, block_tables, q_start, context_lens, causal,
            scale, k_scales=None, v_scales=None, items=None, return_lse=False, window=0):
    """fp64 chunked-prefill attention over packed query rows q [Ttot, Hq, D].

    Rows q_start[b]..q_start[b+1]-1 belong to sequence b at absolute
    positions ctx-n..ctx-1 (bottom-right); causal row r sees keys 0..ctx-n+r.
    ``items`` selects flat (t*Hq + h) rows.
    """
    q = _typed(q, q_tag)
    kp = _typed(k_pages, kv_tag)
    vp = _typed(v_pages, kv_tag)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    qs = np.ascontiguousarray(q_start, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    T, Hq, D = q.shape
    P, ps, Hkv, D2 = kp.shape
    B = cl.shape[0]
    assert D2 == D and qs.shape == (B + 1,) and int(qs[-1]) == T and bt.shape[0] == B
    ks = vs = None
    if kv_tag == "i8":
        ks = np.ascontiguousarray(k_scales, dtype=np.uint16)
        vs = np.ascontiguousarray(v_scales, dtype=np.uint16)
    sel, n_sel = _sel(items)
    n_out = n_sel if sel is not None else T * Hq
    out = np.zeros((n_out, D), dtype=np.float64)
    lse = np.zeros(n_out, dtype=np.float64)
    _check(_load().oracle_prefill(_ptr(q), DTYPES[q_tag], _ptr(kp), _ptr(vp), DTYPES[kv_tag],
                                  _ptr(ks), _ptr(vs), _ptr(bt), _ptr(qs), _ptr(cl),
                                  1 if causal else 0, float(scale), int(window), B, Hq, Hkv, D, ps,
                                  bt.shape[1], P, _ptr(sel), n_sel, _ptr(out), _ptr(lse)))
    if sel is None:
        out = out.reshape(T, Hq, D)
        lse = lse.reshape(T, Hq)
    return (out, lse) if return_lse else out
