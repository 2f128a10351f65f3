"""GPU parity: the cache append (slot-mapping scatter) is bit-exact against the
oracle's byte copy, over the WHOLE pool (untouched rows must not change)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_status_ok, dev, host_bits
from paged_kv_cache_380_b200 import ops
from paged_kv_cache_380_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _check_scatter(k_new, v_new, slots, k_pool, v_pool, tag):
    kp, vp = dev(k_pool, tag), dev(v_pool, tag)
    ops.kv_cache_write(dev(k_new, tag), dev(v_new, tag), dev(slots, "i64"), kp, vp)
    torch.cuda.synchronize()
    assert_status_ok()
    ref_k, ref_v = k_pool.copy(), v_pool.copy()
    oracle.kv_cache_write(k_new, v_new, slots, ref_k, ref_v)
    assert host_bits(kp).tobytes() == ref_k.tobytes()
    assert host_bits(vp).tobytes() == ref_v.tobytes()


@pytest.mark.parametrize("Hkv,D,tag", [(8, 128, "bf16"), (32, 128, "bf16"), (2, 64, "f32"),
                                       (1, 3, "f16")])
def test_scatter_small_bit_exact(Hkv, D, tag):
    rng = np.random.default_rng(100 + Hkv + D)
    P, ps, T = 37, 16, 200
    mk = {"bf16": lambda s: rng.integers(0, 65536, s, dtype=np.uint16),
          "f16": lambda s: rng.integers(0, 65536, s, dtype=np.uint16),
          "f32": lambda s: rng.standard_normal(s).astype(np.float32),
          "i8": lambda s: rng.integers(-128, 128, s, dtype=np.int8)}[tag]
    k_pool, v_pool = mk((P, ps, Hkv, D)), mk((P, ps, Hkv, D))
    k_new, v_new = mk((T, Hkv, D)), mk((T, Hkv, D))
    slots = rng.choice(P * ps, T, replace=False).astype(np.int64)
    slots[::17] = -1                                   # padding rows are skipped
    _check_scatter(k_new, v_new, slots, k_pool, v_pool, tag)


def test_scatter_int8_with_scales_bit_exact():
    rng = np.random.default_rng(7)
    P, ps, Hkv, D, T = 20, 16, 8, 128, 50
    kc = rng.integers(-127, 128, (P, ps, Hkv, D), dtype=np.int8)
    vc = rng.integers(-127, 128, (P, ps, Hkv, D), dtype=np.int8)
    ks = rng.integers(0, 0x7C00, (P, ps, Hkv), dtype=np.uint16)
    vs = rng.integers(0, 0x7C00, (P, ps, Hkv), dtype=np.uint16)
    nk = rng.integers(-127, 128, (T, Hkv, D), dtype=np.int8)
    nv = rng.integers(-127, 128, (T, Hkv, D), dtype=np.int8)
    nks = rng.integers(0, 0x7C00, (T, Hkv), dtype=np.uint16)
    nvs = rng.integers(0, 0x7C00, (T, Hkv), dtype=np.uint16)
    slots = rng.choice(P * ps, T, replace=False).astype(np.int64)
    dk, dv, dks, dvs = dev(kc, "i8"), dev(vc, "i8"), dev(ks, "f16"), dev(vs, "f16")
    ops.kv_cache_write(dev(nk, "i8"), dev(nv, "i8"), dev(slots, "i64"), dk, dv,
                       k_scale=dev(nks, "f16"), v_scale=dev(nvs, "f16"), k_scale_pages=dks,
                       v_scale_pages=dvs)
    torch.cuda.synchronize()
    assert_status_ok()
    for pool, new in ((kc, nk), (vc, nv), (ks, nks), (vs, nvs)):
        oracle.kv_cache_write(new, new, slots, pool, pool.copy())
    assert host_bits(dk).tobytes() == kc.tobytes() and host_bits(dv).tobytes() == vc.tobytes()
    assert host_bits(dks).tobytes() == ks.tobytes() and host_bits(dvs).tobytes() == vs.tobytes()


def test_scatter_llama2_7b_new_tokens_bit_exact():
    c = W.llama2_7b_mha_decode()
    _check_scatter(c.k_new, c.v_new, c.slot_mapping, c.k_pages, c.v_pages, "bf16")


def test_scatter_full_cache_bit_exact():
    """The bandwidth case bench.py times: all 143 k cached rows of the Llama-2-7B-shaped
    batch written through a seeded random permutation of the pool's slots."""
    c = W.llama2_7b_mha_decode()
    src, dst = W.full_cache_scatter(c)
    Hkv, D = c.num_kv_heads, c.head_dim
    k_rows = c.k_pages.reshape(-1, Hkv, D)[src]
    v_rows = c.v_pages.reshape(-1, Hkv, D)[src]
    _check_scatter(k_rows, v_rows, dst, c.k_pages, c.v_pages, "bf16")


def test_scatter_prefill_chunk_bit_exact():
    c = W.chunked_prefill_shared_prefix()
    _check_scatter(c.k_new, c.v_new, c.slot_mapping, c.k_pages, c.v_pages, "bf16")


def test_scatter_out_of_range_slot_is_recorded_not_written():
    rng = np.random.default_rng(9)
    P, ps, Hkv, D, T = 8, 16, 2, 64, 10
    k_pool = rng.integers(0, 65536, (P, ps, Hkv, D), dtype=np.uint16)
    v_pool = k_pool ^ 0x5555
    k_new = rng.integers(0, 65536, (T, Hkv, D), dtype=np.uint16)
    v_new = k_new ^ 0x3333
    slots = rng.choice(P * ps, T, replace=False).astype(np.int64)
    slots[4] = P * ps + 5                               # past the pool
    kp, vp = dev(k_pool, "bf16"), dev(v_pool, "bf16")
    ops.kv_cache_write(dev(k_new, "bf16"), dev(v_new, "bf16"), dev(slots, "i64"), kp, vp)
    code, detail = ops.device_status()
    assert code == -5 and detail == P * ps + 5
    keep = np.ones(T, bool); keep[4] = False
    ref_k, ref_v = k_pool.copy(), v_pool.copy()
    oracle.kv_cache_write(k_new[keep], v_new[keep], slots[keep], ref_k, ref_v)
    assert host_bits(kp).tobytes() == ref_k.tobytes() and host_bits(vp).tobytes() == ref_v.tobytes()
    assert_status_ok()                                  # the status word was cleared


# ---- quantise-on-write (INT8 pages with per-(token, head) fp16 scales) --------------

def _quant_rows(rng, T, Hkv, D, src):
    mag = 10.0 ** rng.integers(-7, 3, (T, Hkv, 1))          # includes subnormal-scale rows
    x = (rng.standard_normal((T, Hkv, D)) * mag).astype(np.float32)
    x[0, 0] = 0.0                                            # zero row -> zero scale and codes
    x[1, 0, 5] = np.nan                                      # NaN element -> code 0, ignored by the max
    if src == "bf16":
        return W.to_bf16_bits(np.nan_to_num(x, nan=0.0)) | np.where(np.isnan(x), 0x7FC0, 0).astype(np.uint16)
    if src == "f16":
        return x.astype(np.float16).view(np.uint16)
    return x


@pytest.mark.parametrize("src", ["bf16", "f16", "f32"])
def test_quantise_on_write_bit_exact(src):
    rng = np.random.default_rng(11)
    P, ps, Hkv, D, T = 24, 16, 4, 128, 150
    kx, vx = _quant_rows(rng, T, Hkv, D, src), _quant_rows(rng, T, Hkv, D, src)
    slots = rng.choice(P * ps, T, replace=False).astype(np.int64)
    slots[7] = -1
    kc = rng.integers(-128, 128, (P, ps, Hkv, D), dtype=np.int8)
    vc = kc.copy()
    ks = rng.integers(0, 0x7C00, (P, ps, Hkv), dtype=np.uint16)
    vs = ks.copy()
    dk, dv, dks, dvs = dev(kc, "i8"), dev(vc, "i8"), dev(ks, "f16"), dev(vs, "f16")
    ops.kv_cache_write_quant(dev(kx, src), dev(vx, src), dev(slots, "i64"), dk, dv, dks, dvs)
    torch.cuda.synchronize()
    assert_status_ok()
    qk, sk = oracle.quantize_int8(kx, src)
    qv, sv = oracle.quantize_int8(vx, src)
    oracle.kv_cache_write(qk, qv, slots, kc, vc)
    oracle.kv_cache_write(sk, sv, slots, ks, vs)
    assert host_bits(dk).tobytes() == kc.tobytes() and host_bits(dv).tobytes() == vc.tobytes()
    assert host_bits(dks).tobytes() == ks.tobytes() and host_bits(dvs).tobytes() == vs.tobytes()


def test_quantise_long_context_pool_bit_exact():
    """The whole bf16 pool of the long-context workload (2560 pages of 256
    tokens, 8 KV heads) quantised on the GPU equals the oracle's quantiser."""
    c = W.long_ctx_split_kv()
    P, ps, Hkv, D = c.k_pages.shape
    kb = dev(c.k_pages, "bf16").view(P * ps, Hkv, D)
    vb = dev(c.v_pages, "bf16").view(P * ps, Hkv, D)
    dk = torch.empty((P, ps, Hkv, D), dtype=torch.int8, device="cuda")
    dv = torch.empty_like(dk)
    dks = torch.empty((P, ps, Hkv), dtype=torch.float16, device="cuda")
    dvs = torch.empty_like(dks)
    ops.kv_cache_write_quant(kb, vb, torch.arange(P * ps, dtype=torch.int64, device="cuda"), dk, dv, dks, dvs)
    torch.cuda.synchronize()
    assert_status_ok()
    qk, sk = oracle.quantize_int8(c.k_pages, "bf16")
    assert host_bits(dk).tobytes() == qk.tobytes() and host_bits(dks).tobytes() == sk.tobytes()
    qv, sv = oracle.quantize_int8(c.v_pages, "bf16")
    assert host_bits(dv).tobytes() == qv.tobytes() and host_bits(dvs).tobytes() == sv.tobytes()
