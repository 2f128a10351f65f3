"""The C-ABI library: it loads, exports every symbol include/*.h declares, and
its pure host logic (validation, split planning, error strings) behaves.
No GPU needed: nothing here launches a kernel."""
import ctypes
import glob
import os
import re

import pytest
import torch

from paged_kv_cache_380_b200 import build, ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ops.load()


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(pkv_\w+)\s*\(", text))
    return sorted(names)


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert names, "no declarations found"
    for n in names:
        assert hasattr(lib, n), f"{n} declared but not exported"
    assert set(ops.EXPORTS) == set(names)


def test_library_targets_sm100a_only():
    src = open(os.path.join(ROOT, "paged_kv_cache_380_b200", "build.py")).read()
    assert "arch=compute_100a,code=sm_100a" in src


def test_error_strings(lib):
    for code in (0, -1, -2, -3, -4, -5, -6, 12345):
        assert isinstance(ops.error_string(code), str) and ops.error_string(code)


def test_split_planner_on_the_workloads(lib):
    # Llama-2-7B decode: contexts up to 4096 tokens (256 pages of 16)
    assert ops.decode_plan(64, 32, 32, 128, 16, 256) == (2, 2048)
    # Llama-2-70B GQA decode: up to 8192 tokens
    assert ops.decode_plan(128, 64, 8, 128, 16, 512) == (4, 2048)
    # long context: 131072 tokens in 512 pages of 256 -> 64 partitions of 8 pages
    assert ops.decode_plan(4, 32, 8, 128, 256, 512, torch.int8) == (64, 2048)
    # few (sequence, head) units -> shorter partitions, never below 256 tokens
    s, t = ops.decode_plan(1, 8, 1, 128, 16, 64)
    assert t == 256 and s == 4
    # Llama-2-7B shapes at smaller batches (148 SMs): halved while under 12 CTAs per SM, kept at
    # 512 tokens or more while the grid fills a wave (3 CTAs per SM)
    assert ops.decode_plan(16, 32, 32, 128, 16, 256) == (4, 1024)
    assert ops.decode_plan(4, 32, 32, 128, 16, 256) == (8, 512)
    assert ops.decode_plan(1, 32, 32, 128, 16, 256) == (16, 256)
    # explicit split count, and fp32 never splits
    assert ops.decode_plan(2, 4, 2, 64, 16, 7, num_splits=3)[0] == 3
    assert ops.decode_plan(2, 4, 2, 64, 16, 7, torch.float32) == (1, 112)


def test_split_planner_properties(lib):
    """Random shapes: the partitions cover the longest context with none left empty, hold whole
    pages, never go below 256 tokens or above 2048 (or one page) unless the caller asks for a
    split count, shorten only while the grid is small (under 12 CTAs per SM above 512 tokens,
    under 3 above 256; the host reports 148 SMs when no GPU is visible), grow with the number of
    (sequence, KV head) units, and the workspace is sized for exactly that plan."""
    import random
    rng = random.Random(3)
    sms = torch.cuda.get_device_properties(0).multi_processor_count if torch.cuda.is_available() else 148
    dtypes = (torch.bfloat16, torch.float16, torch.int8, torch.float32)
    for _ in range(3000):
        B, Hkv = rng.randint(1, 300), rng.choice((1, 2, 4, 8, 16, 32, 64))
        Hq, D = Hkv * rng.choice((1, 2, 4, 8)), rng.choice((64, 128))
        ps, mp = rng.choice((16, 32, 64, 128, 256)), rng.randint(1, 1500)
        dt = rng.choice(dtypes)
        ns = 0 if rng.random() < 0.7 else rng.randint(1, 80)
        tokens = mp * ps
        s, t = ops.decode_plan(B, Hq, Hkv, D, ps, mp, dt, num_splits=ns)
        assert s >= 1 and t > 0 and t % 16 == 0
        assert s * t >= tokens and (s - 1) * t < tokens, (B, Hkv, ps, mp, dt, ns, s, t)
        if dt == torch.float32:
            assert s == 1
        else:
            assert t % ps == 0
            if ns > 0:
                assert s <= ns
            else:
                assert 256 <= t <= max(2048, ps)
                if ps == 16:                       # no rounding to whole pages: the fill rule exactly
                    ctas = B * Hkv * s
                    assert t == 256 or ctas >= 3 * sms
                    assert t <= 512 or ctas >= 12 * sms
                    if t < 2048:                   # halved: the longer partition left the grid small
                        c2 = B * Hkv * -(-tokens // (2 * t))
                        assert c2 < 12 * sms if 2 * t > 512 else c2 < 3 * sms
                    s2, t2 = ops.decode_plan(B + 1, Hq, Hkv, D, ps, mp, dt)
                    assert t2 >= t
        rows = B * Hq * s
        want = 0 if s <= 1 else (rows * D * 4 + 255) // 256 * 256 + rows * 4
        assert ops.decode_workspace_size(B, Hq, Hkv, D, ps, mp, dt, num_splits=ns) == want


def test_workspace_size_matches_plan(lib):
    s, _ = ops.decode_plan(4, 32, 8, 128, 256, 512, torch.bfloat16)
    rows = 4 * 32 * s
    want = (rows * 128 * 4 + 255) // 256 * 256 + rows * 4
    assert ops.decode_workspace_size(4, 32, 8, 128, 256, 512) == want
    assert ops.decode_workspace_size(2, 4, 2, 64, 16, 7, torch.float32) == 0
    assert ops.decode_workspace_size(0, 4, 2, 64, 16, 7) == 0


def test_host_validation_rejects_before_launch(lib):
    P = ctypes.c_void_p
    fake = P(0x10000)   # never dereferenced: validation fails first
    # null pool pointer
    rc = lib.pkv_kv_cache_write(fake, fake, fake, 4, None, fake, 8, 128, 16, 10, 1, None, None, None,
                                None, None)
    assert rc == -1
    # Hq not a multiple of Hkv
    rc = lib.pkv_paged_attention_decode(fake, fake, fake, fake, fake, 1.0, fake, 2, 6, 4, 128, 16, 4,
                                        10, 1, 1, None, None, None, 0, 0, None)
    assert rc == -1
    # unsupported dtype combination (bf16 q with f16 pages)
    rc = lib.pkv_paged_attention_decode(fake, fake, fake, fake, fake, 1.0, fake, 2, 8, 2, 128, 16, 4,
                                        10, 1, 2, None, None, None, 0, 0, None)
    assert rc == -2
    # INT8 pages without scales
    rc = lib.pkv_paged_attention_decode(fake, fake, fake, fake, fake, 1.0, fake, 2, 8, 2, 128, 16, 4,
                                        10, 1, 3, None, None, None, 0, 0, None)
    assert rc == -1
    # page size not a multiple of 16 on the tensor-core path
    rc = lib.pkv_paged_attention_decode(fake, fake, fake, fake, fake, 1.0, fake, 2, 8, 2, 128, 8, 4,
                                        10, 1, 1, None, None, None, 0, 0, None)
    assert rc == -2
    # workspace too small for a split plan (contexts up to 16384 tokens)
    rc = lib.pkv_paged_attention_decode(fake, fake, fake, fake, fake, 1.0, fake, 2, 8, 2, 128, 16, 1024,
                                        10, 1, 1, None, None, None, 0, 0, None)
    assert rc == -3
    # prefill: head_dim 96 unsupported (64 and 128 are), fp32 unsupported, scale must be > 0
    rc = lib.pkv_paged_attention_prefill(fake, fake, fake, fake, fake, fake, 1, 1.0, fake, 2, 8, 4, 8, 2,
                                         96, 16, 4, 10, 1, None)
    assert rc == -2
    for bad_scale in (0.0, -0.5):
        rc = lib.pkv_paged_attention_prefill(fake, fake, fake, fake, fake, fake, 1, bad_scale, fake, 2, 8, 4, 8,
                                             2, 128, 16, 4, 10, 1, None)
        assert rc == -1
    rc = lib.pkv_paged_attention_prefill(fake, fake, fake, fake, fake, fake, 1, 1.0, fake, 2, 8, 4, 8, 2,
                                         128, 16, 4, 10, 0, None)
    assert rc == -2
    # prefill output written with 16-byte stores: a 4-byte-aligned out is refused up front
    rc = lib.pkv_paged_attention_prefill(fake, fake, fake, fake, fake, fake, 1, 1.0, P(0x10004), 2, 8, 4, 8, 2,
                                         128, 16, 4, 10, 1, None)
    assert rc == -1
    # empty problems are no-ops
    assert lib.pkv_paged_attention_decode(None, None, None, None, None, 1.0, None, 0, 8, 2, 128, 16, 4,
                                          10, 1, 1, None, None, None, 0, 0, None) == 0
    assert lib.pkv_kv_cache_write(None, None, None, 0, None, None, 8, 128, 16, 10, 1, None, None, None,
                                  None, None) == 0


def test_binding_fails_loudly_without_library(tmp_path):
    saved = ops._lib
    ops._lib = None
    try:
        with pytest.raises(ImportError):
            ops.load(str(tmp_path / "missing.so"))
    finally:
        ops._lib = saved
