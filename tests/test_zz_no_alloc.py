"""The decode entry point for callers that cannot allocate device memory.

pkv_paged_attention_decode_noalloc takes no workspace: its split-KV scratch
is a fixed array inside the library.  It exists for callers that cannot hand
the library a scratch buffer on demand (a server that reserved all HBM for
its KV-cache pool at start-up, a plain-C host without a device allocator, a
decode loop that must not risk a synchronising allocation).  Here it is
called through the C ABI twice in a row, with different problems, and must
agree with the fp64 oracle and with the workspace entry point within the
bf16 tolerance (2e-2); a problem needing more scratch than the array holds
is refused before launch.

This file is named to be collected last, and passes alone in a fresh process
as well as after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_close, assert_status_ok, dev, f64
from paged_kv_cache_380_b200 import ops
from paged_kv_cache_380_b200 import workloads as W

pytestmark = pytest.mark.gpu

PKV_BF16 = 1
PKV_ERR_WORKSPACE = -3
SCRATCH_BYTES = 48 * 1024 * 1024


def _noalloc(lib, q, kp, vp, bt, cl, scale, out, num_splits=0):
    B, Hq, D = q.shape
    P, ps, Hkv, _ = kp.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.pkv_paged_attention_decode_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kp.data_ptr()), ctypes.c_void_p(vp.data_ptr()),
        ctypes.c_void_p(bt.data_ptr()), ctypes.c_void_p(cl.data_ptr()), float(scale),
        ctypes.c_void_p(out.data_ptr()), B, Hq, Hkv, D, ps, bt.shape[1], P, PKV_BF16, PKV_BF16, None, None,
        int(num_splits), stream)


def _case(call):
    if call == 0:   # several partitions per sequence, ragged contexts
        return W.decode_case(name="noalloc0", config_index=400, batch=6, num_q_heads=16, num_kv_heads=4,
                             head_dim=128, page_size=16, dtype="bf16",
                             context_lens=np.array([1, 3000, 17, 2049, 1024, 600]))
    return W.llama2_7b_mha_decode()


def test_noalloc_decode_matches_workspace_decode_on_two_calls():
    lib = ops.load()
    for call in range(2):
        c = _case(call)
        q, kp, vp = dev(c.q, "bf16"), dev(c.k_pages, "bf16"), dev(c.v_pages, "bf16")
        bt, cl = dev(c.block_tables, "i32"), dev(c.context_lens, "i32")
        splits, _ = ops.decode_plan(c.batch, c.num_q_heads, c.num_kv_heads, c.head_dim, c.page_size,
                                    c.max_pages_per_seq)
        assert splits > 1, "the problem must use the split-KV scratch"
        want = ops.paged_attention_decode(q, kp, vp, bt, cl, c.scale)
        got = torch.full_like(q, float("nan"))
        rc = _noalloc(lib, q, kp, vp, bt, cl, c.scale, got)
        assert rc == 0, ops.error_string(rc)
        torch.cuda.synchronize()
        assert_status_ok()
        g, w = f64(got), f64(want)
        assert np.isfinite(g).all()
        assert np.max(np.abs(g - w)) <= 2e-2
        # and against the oracle: every (sequence, head) of the small problem, a sample of the large one
        n_items = c.batch * c.num_q_heads
        items = (np.arange(n_items) if call == 0 else
                 np.sort(np.random.default_rng(3).choice(n_items, 256, replace=False)))
        ref = oracle.decode(c.q, "bf16", c.k_pages, c.v_pages, "bf16", c.block_tables, c.context_lens, c.scale,
                            items=items)
        assert_close(g.reshape(n_items, -1)[items], ref, 2e-2, c.name)


def test_noalloc_decode_refuses_problems_beyond_the_scratch():
    lib = ops.load()
    # 512 sequences x 64 heads x 8 partitions x 129 floats > 48 MiB
    need = ops.decode_workspace_size(512, 64, 8, 128, 16, 512)
    assert need > SCRATCH_BYTES
    q = torch.zeros((512, 64, 128), dtype=torch.bfloat16, device="cuda")
    kp = torch.zeros((1, 16, 8, 128), dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros((512, 512), dtype=torch.int32, device="cuda")
    cl = torch.ones(512, dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    assert _noalloc(lib, q, kp, kp, bt, cl, 0.1, out) == PKV_ERR_WORKSPACE
    # the same problem with fewer partitions fits and runs
    assert _noalloc(lib, q, kp, kp, bt, cl, 0.1, out, num_splits=2) == 0
    torch.cuda.synchronize()
    assert_status_ok()
