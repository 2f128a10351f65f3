"""GPU: the bounded mbarrier wait of the prefill kernel runs out on a barrier that
nothing completes, records PKV_ERR_DEVICE_TIMEOUT in the device status word, and
leaves the context usable (a prefill right after still matches the oracle)."""
import time

import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_close, dev, f64
from paged_kv_cache_380_b200 import ops
from paged_kv_cache_380_b200 import workloads as W

pytestmark = pytest.mark.gpu

PKV_ERR_DEVICE_TIMEOUT = -6


def test_wait_runs_out_and_is_reported():
    assert ops.device_status()[0] == 0                 # clean before
    t0 = time.perf_counter()
    ops.selftest_wait_timeout()
    code, _ = ops.device_status()                      # synchronises
    dt = time.perf_counter() - t0
    assert code == PKV_ERR_DEVICE_TIMEOUT
    assert 0.9 < dt < 30.0                             # the 1 s bound, not a hang
    assert ops.device_status()[0] == 0                 # read-and-clear

    # the context is still usable: a small causal prefill matches the oracle
    c = W.prefill_case(name="after_timeout", config_index=230, num_seqs=2, num_q_heads=4, num_kv_heads=2,
                       head_dim=128, page_size=16, dtype="bf16", shared_prefix=16, chunk_lens=np.array([5, 40]))
    kp, vp = dev(c.k_pages, "bf16"), dev(c.v_pages, "bf16")
    ops.kv_cache_write(dev(c.k_new, "bf16"), dev(c.v_new, "bf16"), dev(c.slot_mapping, "i64"), kp, vp)
    out = ops.paged_attention_prefill(dev(c.q, "bf16"), kp, vp, dev(c.block_tables, "i32"), dev(c.q_start, "i32"),
                                      dev(c.context_lens, "i32"), True, c.scale, max_q_len=40)
    torch.cuda.synchronize()
    assert ops.device_status()[0] == 0
    kh, vh = c.k_pages.copy(), c.v_pages.copy()
    oracle.kv_cache_write(c.k_new, c.v_new, c.slot_mapping, kh, vh)
    want = oracle.prefill(c.q, "bf16", kh, vh, "bf16", c.block_tables, c.q_start, c.context_lens, True, c.scale)
    assert_close(f64(out), want, 2e-2, c.name)
