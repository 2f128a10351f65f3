"""Thin ctypes binding of libpagedkv (argument marshalling only).

Every function here forwards device pointers, sizes and the current torch CUDA
stream to the C ABI declared in ``include/pagedkv.h``; all work runs in the
library's CUDA kernels.  There is no fallback: if ``libpagedkv.so`` is missing
or cannot be loaded, the first call raises.

Tensor arguments are torch CUDA tensors (torch is used only for device memory
and streams).  bf16 pools may also be passed as int16/uint16 views.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpagedkv.so")
_lock = threading.Lock()
_lib = None

PKV_F32, PKV_BF16, PKV_F16, PKV_I8 = 0, 1, 2, 3
_DT = {torch.float32: PKV_F32, torch.bfloat16: PKV_BF16, torch.float16: PKV_F16, torch.int8: PKV_I8}

# every symbol include/pagedkv.h declares
EXPORTS = ("pkv_error_string", "pkv_kv_cache_write", "pkv_kv_cache_write_quant", "pkv_paged_attention_decode",
           "pkv_decode_workspace_size", "pkv_decode_plan", "pkv_paged_attention_decode_noalloc",
           "pkv_paged_attention_decode_ex", "pkv_paged_attention_prefill_ex",
           "pkv_paged_attention_prefill",
           "pkv_get_device_status", "pkv_bm_create", "pkv_bm_destroy", "pkv_bm_add_sequence", "pkv_bm_fork",
           "pkv_bm_append", "pkv_bm_free_sequence", "pkv_bm_block_tables", "pkv_bm_num_free_pages",
           "pkv_bm_page_refcount", "pkv_bm_num_sequences", "pkv_copy_pages", "pkv_selftest_wait_timeout")


class PagedKVError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {error_string(code)} (code {code})")


def load(path: str = _LIB_PATH):
    """Load the shared library and declare the C signatures (raises if absent)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise ImportError(f"libpagedkv.so not built at {path}: run "
                              "`python -m paged_kv_cache_380_b200.build` (needs nvcc)")
        lib = ctypes.CDLL(path)
        P, I, I64, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        lib.pkv_error_string.argtypes = [I]
        lib.pkv_error_string.restype = ctypes.c_char_p
        lib.pkv_kv_cache_write.argtypes = [P, P, P, I64, P, P, I, I, I, I64, I, P, P, P, P, P]
        lib.pkv_kv_cache_write.restype = I
        lib.pkv_kv_cache_write_quant.argtypes = [P, P, I, P, I64, P, P, P, P, I, I, I, I64, P]
        lib.pkv_kv_cache_write_quant.restype = I
        lib.pkv_paged_attention_decode.argtypes = [P, P, P, P, P, F, P, I, I, I, I, I, I, I64, I, I,
                                                   P, P, P, SZ, I, P]
        lib.pkv_paged_attention_decode.restype = I
        lib.pkv_paged_attention_decode_ex.argtypes = [P, P, P, P, P, F, P, I, I, I, I, I, I, I64, I, I,
                                                      P, P, P, SZ, I, I, P]
        lib.pkv_paged_attention_decode_ex.restype = I
        lib.pkv_paged_attention_prefill_ex.argtypes = [P, P, P, P, P, P, I, F, P, I, I, I, I, I, I, I, I,
                                                       I64, I, I, P]
        lib.pkv_paged_attention_prefill_ex.restype = I
        lib.pkv_paged_attention_decode_noalloc.argtypes = [P, P, P, P, P, F, P, I, I, I, I, I, I, I64, I, I,
                                                           P, P, I, P]
        lib.pkv_paged_attention_decode_noalloc.restype = I
        lib.pkv_decode_workspace_size.argtypes = [I, I, I, I, I, I, I, I]
        lib.pkv_decode_workspace_size.restype = SZ
        lib.pkv_decode_plan.argtypes = [I, I, I, I, I, I, I, I, ctypes.POINTER(I), ctypes.POINTER(I)]
        lib.pkv_decode_plan.restype = I
        lib.pkv_paged_attention_prefill.argtypes = [P, P, P, P, P, P, I, F, P, I, I, I, I, I, I, I, I,
                                                    I64, I, P]
        lib.pkv_paged_attention_prefill.restype = I
        lib.pkv_get_device_status.argtypes = [P, ctypes.POINTER(I64)]
        lib.pkv_get_device_status.restype = I
        lib.pkv_selftest_wait_timeout.argtypes = [P]
        lib.pkv_selftest_wait_timeout.restype = I
        lib.pkv_bm_create.argtypes = [I64, I, I]
        lib.pkv_bm_create.restype = P
        lib.pkv_bm_destroy.argtypes = [P]
        lib.pkv_bm_destroy.restype = None
        lib.pkv_bm_add_sequence.argtypes = [P, ctypes.POINTER(I64)]
        lib.pkv_bm_fork.argtypes = [P, I64, ctypes.POINTER(I64)]
        lib.pkv_bm_append.argtypes = [P, I64, I, P, P, P, ctypes.POINTER(I)]
        lib.pkv_bm_free_sequence.argtypes = [P, I64]
        lib.pkv_bm_block_tables.argtypes = [P, P, I, P, P]
        lib.pkv_bm_num_free_pages.argtypes = [P]
        lib.pkv_bm_num_free_pages.restype = I64
        lib.pkv_bm_page_refcount.argtypes = [P, ctypes.c_int32]
        lib.pkv_bm_num_sequences.argtypes = [P]
        lib.pkv_copy_pages.argtypes = [P, P, P, P, I, I64, I64, P]
        for f in (lib.pkv_bm_add_sequence, lib.pkv_bm_fork, lib.pkv_bm_append, lib.pkv_bm_free_sequence,
                  lib.pkv_bm_block_tables, lib.pkv_bm_page_refcount, lib.pkv_bm_num_sequences, lib.pkv_copy_pages):
            f.restype = I
        _lib = lib
    return _lib


def error_string(code: int) -> str:
    return load().pkv_error_string(int(code)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc: int, what: str):
    if rc != 0:
        raise PagedKVError(rc, what)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype in _DT:
        return _DT[t.dtype]
    raise TypeError(f"unsupported dtype {t.dtype}")


def _out_like(q, out):
    """The output tensor: a new one like q, or the caller's, which must match q."""
    if out is None:
        return torch.empty_like(q)
    if out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError(f"out must match q: got {tuple(out.shape)} {out.dtype}, want {tuple(q.shape)} {q.dtype}")
    return out


def _cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def kv_cache_write(k, v, slot_mapping, k_pages, v_pages, *, k_scale=None, v_scale=None,
                   k_scale_pages=None, v_scale_pages=None, stream=None) -> None:
    """Scatter new K/V rows ``[T, Hkv, D]`` into pools ``[P, ps, Hkv, D]`` at
    ``slot_mapping`` (int64 ``[T]``; negative = skip).  INT8 pools also take
    the per-row fp16 scales ``[T, Hkv]`` and scale pools ``[P, ps, Hkv]``."""
    _cuda(k, v, slot_mapping, k_pages, v_pages, k_scale, v_scale, k_scale_pages, v_scale_pages)
    P, ps, Hkv, D = k_pages.shape
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    if k.shape[1:] != (Hkv, D) or v.shape != k.shape or k.dtype != k_pages.dtype:
        raise ValueError("k/v must be [T, num_kv_heads, head_dim] of the pool's dtype")
    _check(load().pkv_kv_cache_write(_ptr(k), _ptr(v), _ptr(slot_mapping), k.shape[0], _ptr(k_pages),
                                     _ptr(v_pages), Hkv, D, ps, P, _dtype_code(k_pages), _ptr(k_scale),
                                     _ptr(v_scale), _ptr(k_scale_pages), _ptr(v_scale_pages),
                                     _stream(stream)), "kv_cache_write")


def kv_cache_write_quant(k, v, slot_mapping, k_pages, v_pages, k_scale_pages, v_scale_pages, *,
                         stream=None) -> None:
    """Quantise new K/V rows ``[T, Hkv, D]`` (bf16/f16/f32) to int8 with one fp16
    scale per (token, head) and scatter them into the INT8 pools
    ``[P, ps, Hkv, D]`` and scale pools ``[P, ps, Hkv]`` at ``slot_mapping``."""
    _cuda(k, v, slot_mapping, k_pages, v_pages, k_scale_pages, v_scale_pages)
    P, ps, Hkv, D = k_pages.shape
    if k_pages.dtype != torch.int8 or k_scale_pages.dtype != torch.float16:
        raise TypeError("INT8 pools and fp16 scale pools expected")
    if k.shape[1:] != (Hkv, D) or v.shape != k.shape or slot_mapping.dtype != torch.int64:
        raise ValueError("k/v must be [T, num_kv_heads, head_dim]; slot_mapping int64")
    _check(load().pkv_kv_cache_write_quant(_ptr(k), _ptr(v), _dtype_code(k), _ptr(slot_mapping), k.shape[0],
                                           _ptr(k_pages), _ptr(v_pages), _ptr(k_scale_pages),
                                           _ptr(v_scale_pages), Hkv, D, ps, P, _stream(stream)),
           "kv_cache_write_quant")


def decode_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, page_size, max_pages_per_seq,
                kv_dtype=torch.bfloat16, num_splits=0):
    """(partitions per sequence, partition length in tokens) the decode call uses."""
    s, t = ctypes.c_int(0), ctypes.c_int(0)
    _check(load().pkv_decode_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, page_size,
                                  max_pages_per_seq, _DT[kv_dtype], num_splits, ctypes.byref(s),
                                  ctypes.byref(t)), "decode_plan")
    return s.value, t.value


def decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, page_size, max_pages_per_seq,
                          kv_dtype=torch.bfloat16, num_splits=0) -> int:
    return int(load().pkv_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, page_size,
                                                max_pages_per_seq, _DT[kv_dtype], num_splits))


def paged_attention_decode(q, k_pages, v_pages, block_tables, context_lens, scale, out=None, *,
                           k_scales=None, v_scales=None, workspace=None, num_splits=0, window=0, stream=None):
    """Decode attention: ``q [B, Hq, D]`` against pools ``[P, ps, Hkv, D]``
    through ``block_tables int32 [B, MP]`` and ``context_lens int32 [B]``.
    Returns ``out`` (allocated like ``q`` if not given).  A workspace of
    ``decode_workspace_size(...)`` bytes is allocated with torch when the
    caller passes none."""
    _cuda(q, k_pages, v_pages, block_tables, context_lens, k_scales, v_scales, out, workspace)
    B, Hq, D = q.shape
    P, ps, Hkv, D2 = k_pages.shape
    if D2 != D or v_pages.shape != k_pages.shape or block_tables.shape[0] != B:
        raise ValueError("shape mismatch")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    out = _out_like(q, out)
    MP = block_tables.shape[1]
    kv_dt = k_pages.dtype
    if workspace is None:
        need = decode_workspace_size(B, Hq, Hkv, D, ps, MP, kv_dt, num_splits)
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    lib = load()
    args = (_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_tables), _ptr(context_lens), float(scale),
            _ptr(out), B, Hq, Hkv, D, ps, MP, P, _dtype_code(q), _dtype_code(k_pages), _ptr(k_scales),
            _ptr(v_scales), _ptr(workspace), workspace.numel(), int(num_splits))
    if window > 0:
        _check(lib.pkv_paged_attention_decode_ex(*args, int(window), _stream(stream)), "paged_attention_decode_ex")
    else:
        _check(lib.pkv_paged_attention_decode(*args, _stream(stream)), "paged_attention_decode")
    return out


def paged_attention_decode_noalloc(q, k_pages, v_pages, block_tables, context_lens, scale, out=None, *,
                                   k_scales=None, v_scales=None, num_splits=0, stream=None):
    """Decode attention through the entry point that needs no workspace: the
    split-KV scratch is a fixed array inside the library (for callers that
    cannot allocate device memory).  ``out`` must be given by callers that
    cannot allocate; when omitted it is allocated here with torch."""
    _cuda(q, k_pages, v_pages, block_tables, context_lens, k_scales, v_scales, out)
    B, Hq, D = q.shape
    P, ps, Hkv, _ = k_pages.shape
    out = _out_like(q, out)
    _check(load().pkv_paged_attention_decode_noalloc(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_tables), _ptr(context_lens), float(scale), _ptr(out),
        B, Hq, Hkv, D, ps, block_tables.shape[1], P, _dtype_code(q), _dtype_code(k_pages), _ptr(k_scales),
        _ptr(v_scales), int(num_splits), _stream(stream)), "paged_attention_decode_noalloc")
    return out


def paged_attention_prefill(q, k_pages, v_pages, block_tables, q_start, context_lens, causal, scale,
                            out=None, *, max_q_len=None, window=0, stream=None):
    """Chunked prefill: packed ``q [Ttot, Hq, D]``, rows ``q_start[b]..q_start[b+1]-1``
    of sequence b at positions ``ctx-n..ctx-1``; causal rows see keys up to
    their own position.  ``max_q_len`` (the longest chunk) sizes the grid;
    when omitted it is read from ``q_start`` (a device-to-host copy)."""
    _cuda(q, k_pages, v_pages, block_tables, q_start, context_lens, out)
    T, Hq, D = q.shape
    P, ps, Hkv, D2 = k_pages.shape
    B = context_lens.shape[0]
    if D2 != D or q_start.shape[0] != B + 1:
        raise ValueError("shape mismatch")
    out = _out_like(q, out)
    if max_q_len is None:
        max_q_len = int((q_start[1:] - q_start[:-1]).max().item()) if B else 0
    lib = load()
    args = (_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_tables), _ptr(q_start), _ptr(context_lens),
            1 if causal else 0, float(scale), _ptr(out), B, T, int(max_q_len), Hq, Hkv, D, ps,
            block_tables.shape[1], P, _dtype_code(q))
    if window > 0:
        _check(lib.pkv_paged_attention_prefill_ex(*args, int(window), _stream(stream)), "paged_attention_prefill_ex")
    else:
        _check(lib.pkv_paged_attention_prefill(*args, _stream(stream)), "paged_attention_prefill")
    return out


def selftest_wait_timeout(stream=None) -> None:
    """Launch a bounded wait that nothing completes (about 1 s); the device status
    word then holds PKV_ERR_DEVICE_TIMEOUT."""
    _check(load().pkv_selftest_wait_timeout(_stream(stream)), "selftest_wait_timeout")


def device_status(stream=None):
    """Synchronise the stream; return (code, detail) of the device status word and clear it."""
    detail = ctypes.c_int64(-1)
    code = load().pkv_get_device_status(_stream(stream), ctypes.byref(detail))
    return int(code), int(detail.value)


def copy_pages(k_pages, v_pages, src, dst, *, stream=None) -> None:
    """Copy whole pages src[i] -> dst[i] (int32 CUDA tensors) of both pools."""
    _cuda(k_pages, v_pages, src, dst)
    P = k_pages.shape[0]
    page_bytes = k_pages[0].numel() * k_pages.element_size()
    _check(load().pkv_copy_pages(_ptr(k_pages), _ptr(v_pages), _ptr(src), _ptr(dst), int(src.numel()), page_bytes,
                                 P, _stream(stream)), "copy_pages")


class BlockManager:
    """Host-side page allocator of the C library: refcounted pages, fork with
    shared pages, copy-on-write on append, release that deletes the table entry."""

    def __init__(self, num_pages: int, page_size: int, max_pages_per_seq: int):
        self._lib = load()
        self._h = self._lib.pkv_bm_create(int(num_pages), int(page_size), int(max_pages_per_seq))
        if not self._h:
            raise ValueError("invalid block manager sizes")
        self.page_size, self.max_pages_per_seq = page_size, max_pages_per_seq

    def __del__(self):
        if getattr(self, "_h", None):
            self._lib.pkv_bm_destroy(self._h)
            self._h = None

    def add_sequence(self) -> int:
        out = ctypes.c_int64()
        _check(self._lib.pkv_bm_add_sequence(self._h, ctypes.byref(out)), "bm_add_sequence")
        return out.value

    def fork(self, parent: int) -> int:
        out = ctypes.c_int64()
        _check(self._lib.pkv_bm_fork(self._h, int(parent), ctypes.byref(out)), "bm_fork")
        return out.value

    def append(self, seq: int, num_tokens: int):
        """Returns (slots int64 numpy [num_tokens], copies [(src, dst)])."""
        import numpy as np
        slots = np.empty(max(num_tokens, 1), dtype=np.int64)
        src, dst, n = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int()
        _check(self._lib.pkv_bm_append(self._h, int(seq), int(num_tokens), slots.ctypes.data_as(ctypes.c_void_p),
                                       ctypes.byref(src), ctypes.byref(dst), ctypes.byref(n)), "bm_append")
        return slots[:num_tokens], ([(src.value, dst.value)] if n.value else [])

    def free(self, seq: int) -> None:
        _check(self._lib.pkv_bm_free_sequence(self._h, int(seq)), "bm_free_sequence")

    def block_tables(self, seq_ids):
        """(int32 [len(seq_ids), max_pages_per_seq] tables, int32 context lengths)."""
        import numpy as np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        table = np.empty((ids.shape[0], self.max_pages_per_seq), dtype=np.int32)
        lens = np.empty(ids.shape[0], dtype=np.int32)
        _check(self._lib.pkv_bm_block_tables(self._h, ids.ctypes.data_as(ctypes.c_void_p), ids.shape[0],
                                             table.ctypes.data_as(ctypes.c_void_p),
                                             lens.ctypes.data_as(ctypes.c_void_p)), "bm_block_tables")
        return table, lens

    def num_free_pages(self) -> int:
        return int(self._lib.pkv_bm_num_free_pages(self._h))

    def refcount(self, page: int) -> int:
        r = self._lib.pkv_bm_page_refcount(self._h, int(page))
        if r < 0:
            raise PagedKVError(r, "bm_page_refcount")
        return r

    def num_sequences(self) -> int:
        return int(self._lib.pkv_bm_num_sequences(self._h))
