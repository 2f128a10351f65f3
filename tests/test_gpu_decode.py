"""GPU parity: decode attention (split-KV, GQA, INT8 pages) against the fp64
oracle, on the same seeded inputs.  Tolerances (max abs error): 2e-2 for bf16
and fp16, 1e-4 for fp32, 5e-2 for INT8 pages against the dequantised oracle."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_close, assert_status_ok, dev, f64
from paged_kv_cache_380_b200 import ops
from paged_kv_cache_380_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-2, "f16": 2e-2, "f32": 1e-4, "i8": 5e-2}


def run_case(case, kv="same", num_splits=0, write_new=False, items=None, window=0):
    """Run the GPU decode on a workloads.Case and compare with the oracle."""
    tag = case.dtype
    k_host, v_host = case.k_pages, case.v_pages
    kq = vq = ks = vs = None
    if kv == "i8":
        kq, ks = oracle.quantize_int8(k_host, tag)
        vq, vs = oracle.quantize_int8(v_host, tag)
    if kv == "i8":
        kp, vp = dev(kq, "i8"), dev(vq, "i8")
        dks, dvs = dev(ks, "f16"), dev(vs, "f16")
    else:
        kp, vp = dev(k_host, tag), dev(v_host, tag)
        dks = dvs = None
    if write_new:
        assert kv != "i8"
        ops.kv_cache_write(dev(case.k_new, tag), dev(case.v_new, tag), dev(case.slot_mapping, "i64"), kp, vp)
        k_host, v_host = k_host.copy(), v_host.copy()
        oracle.kv_cache_write(case.k_new, case.v_new, case.slot_mapping, k_host, v_host)
    q = dev(case.q, tag)
    bt, cl = dev(case.block_tables, "i32"), dev(case.context_lens, "i32")
    out = ops.paged_attention_decode(q, kp, vp, bt, cl, case.scale, k_scales=dks, v_scales=dvs,
                                     num_splits=num_splits, window=window)
    torch.cuda.synchronize()
    assert_status_ok()
    if kv == "i8":
        want = oracle.decode(case.q, tag, kq, vq, "i8", case.block_tables, case.context_lens, case.scale,
                             k_scales=ks, v_scales=vs, items=items, window=window)
    else:
        want = oracle.decode(case.q, tag, k_host, v_host, tag, case.block_tables, case.context_lens,
                             case.scale, items=items, window=window)
    got = f64(out)
    if items is not None:
        got = got.reshape(-1, got.shape[-1])[items]
    assert_close(got, want, TOL["i8" if kv == "i8" else tag], case.name)
    return out


def small_case(idx, *, Hq, Hkv, D=128, ps=16, dtype="bf16", ctx=(1, 15, 16, 17, 33, 100, 0, 1000)):
    return W.decode_case(name=f"small{idx}", config_index=100 + idx, batch=len(ctx), num_q_heads=Hq,
                         num_kv_heads=Hkv, head_dim=D, page_size=ps, dtype=dtype,
                         context_lens=np.array(ctx))


# ---- the tiny fp32 workload ---------------------------------------------------

def test_tiny_decode_f32():
    run_case(W.tiny_decode_f32())


def test_f32_path_edge_contexts():
    run_case(small_case(1, Hq=4, Hkv=2, D=64, dtype="f32", ctx=(1, 16, 0, 45)))


# ---- bf16/f16 tensor-core path: group sizes, context edges, splits -----------

@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 4), (8, 2), (16, 2), (32, 2)])
@pytest.mark.parametrize("num_splits", [0, 1, 3])
def test_group_sizes_and_splits(Hq, Hkv, num_splits):
    run_case(small_case(Hq + Hkv, Hq=Hq, Hkv=Hkv), num_splits=num_splits)


@pytest.mark.parametrize("ps", [16, 32, 256])
@pytest.mark.parametrize("D", [64, 128])
def test_page_sizes_and_head_dims(ps, D):
    run_case(small_case(ps + D, Hq=8, Hkv=2, D=D, ps=ps, ctx=(1, 31, 32, 257, 600)), num_splits=2)


@pytest.mark.parametrize("num_splits", [0, 2])
def test_partition_boundaries(num_splits):
    # contexts on either side of the 1024-token split partitions and of whole pages
    run_case(small_case(9, Hq=16, Hkv=4, ctx=(1023, 1024, 1025, 2047, 2048, 2049, 4096, 1)), num_splits=num_splits)


def test_fp16_pages():
    run_case(small_case(50, Hq=16, Hkv=4, dtype="f16"), num_splits=2)


def test_many_splits_short_partitions():
    # 100-way split of a 1600-token context: 1 chunk per partition
    c = small_case(51, Hq=8, Hkv=2, ctx=(1600, 17, 1599))
    run_case(c, num_splits=100)


def test_append_then_decode():
    c = W.decode_case(name="append", config_index=52, batch=6, num_q_heads=8, num_kv_heads=2,
                      head_dim=128, page_size=16, dtype="bf16",
                      context_lens=np.array([1, 16, 17, 300, 48, 2]), new_tokens="append")
    run_case(c, write_new=True)


# ---- INT8 pages ----------------------------------------------------------------

@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (8, 1), (12, 3), (32, 8)])
def test_int8_pages(Hq, Hkv):
    run_case(small_case(60 + Hkv, Hq=Hq, Hkv=Hkv, ctx=(1, 16, 17, 500, 0, 33)), kv="i8", num_splits=2)


def test_int8_pages_fp16_queries():
    run_case(small_case(70, Hq=8, Hkv=2, dtype="f16", ctx=(5, 260, 1000)), kv="i8")


# ---- the full-size workloads, in the launch configuration the bench times ------

def test_llama2_7b_mha_decode_full():
    run_case(W.llama2_7b_mha_decode(), write_new=True)


def test_llama2_70b_gqa_decode_full():
    run_case(W.llama2_70b_gqa_decode())


def test_long_context_split_kv_bf16_full():
    run_case(W.long_ctx_split_kv())


def test_long_context_split_kv_int8_full():
    run_case(W.long_ctx_split_kv(), kv="i8")


# ---- device-side range checks ------------------------------------------------------

def test_out_of_range_page_is_recorded_not_faulted():
    c = small_case(80, Hq=8, Hkv=2, ctx=(40, 70))
    bt = c.block_tables.copy()
    bt[1, 2] = c.num_pages + 3
    q = dev(c.q, "bf16")
    out = ops.paged_attention_decode(q, dev(c.k_pages, "bf16"), dev(c.v_pages, "bf16"), dev(bt, "i32"),
                                     dev(c.context_lens, "i32"), c.scale)
    code, detail = ops.device_status()
    assert code == -5 and detail == c.num_pages + 3
    # the other sequence is unaffected
    want = oracle.decode(c.q, "bf16", c.k_pages, c.v_pages, "bf16", c.block_tables, c.context_lens, c.scale)
    assert_close(f64(out)[0], want[0], 2e-2, "unaffected sequence")
    assert_status_ok()


def test_int8_pages_large_queries():
    """Queries far beyond the fp16 range (bf16 allows them): the INT8 path scales each
    head by a power of two before its fp16 MMA and folds the factor back exactly."""
    c = small_case(71, Hq=8, Hkv=2, ctx=(40, 300))
    q = W.bf16_bits_to_f32(c.q) * np.float32(3.0e5)
    q[0, 1] *= np.float32(1e-3)                     # heads of very different magnitudes
    c.q = W.to_bf16_bits(q)
    c.scale = 1e-5
    run_case(c, kv="i8")


# ---- local (sliding-window) attention ---------------------------------------------

@pytest.mark.parametrize("window", [1, 16, 17, 100, 5000])
@pytest.mark.parametrize("num_splits", [0, 3])
def test_sliding_window_decode(window, num_splits):
    run_case(small_case(90, Hq=8, Hkv=2, ctx=(1, 15, 16, 17, 33, 100, 0, 1000)), num_splits=num_splits,
             window=window)


def test_sliding_window_decode_int8_and_fp32():
    run_case(small_case(91, Hq=8, Hkv=2, ctx=(5, 260, 1000)), kv="i8", window=70)
    run_case(small_case(92, Hq=4, Hkv=2, D=64, dtype="f32", ctx=(1, 16, 0, 45)), window=9)
