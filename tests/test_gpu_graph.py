"""GPU: the decode step captured in a CUDA graph matches the fp64 oracle
(max abs error 2e-2, bf16) and equals the eager launches bit for bit, also
after the inputs are updated in place between replays."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_close, assert_status_ok, dev, f64, host_bits
from paged_kv_cache_380_b200 import ops
from paged_kv_cache_380_b200 import workloads as W
from paged_kv_cache_380_b200.graph import DecodeStepGraph

pytestmark = pytest.mark.gpu


def test_graph_replay_matches_eager_and_follows_updates():
    c = W.decode_case(name="graph", config_index=500, batch=8, num_q_heads=16, num_kv_heads=4, head_dim=128,
                      page_size=16, dtype="bf16", context_lens=np.array([1, 17, 300, 2000, 64, 5, 1500, 33]),
                      new_tokens="append")
    q, bt, cl = dev(c.q, "bf16"), dev(c.block_tables, "i32"), dev(c.context_lens, "i32")
    kn, vn, sl = dev(c.k_new, "bf16"), dev(c.v_new, "bf16"), dev(c.slot_mapping, "i64")
    kp_g, vp_g = dev(c.k_pages, "bf16"), dev(c.v_pages, "bf16")
    kp_e, vp_e = kp_g.clone(), vp_g.clone()

    g = DecodeStepGraph(q, kp_g, vp_g, bt, cl, c.scale, k_new=kn, v_new=vn, slot_mapping=sl)

    def eager():
        ops.kv_cache_write(kn, vn, sl, kp_e, vp_e)
        return ops.paged_attention_decode(q, kp_e, vp_e, bt, cl, c.scale)

    k_host, v_host = c.k_pages.copy(), c.v_pages.copy()
    for step in range(3):
        got = g.replay().clone()
        want = eager()
        torch.cuda.synchronize()
        assert_status_ok()
        # the oracle: the same append, then decode, on host copies of this step's inputs
        oracle.kv_cache_write(host_bits(kn), host_bits(vn), c.slot_mapping, k_host, v_host)
        ref = oracle.decode(host_bits(q), "bf16", k_host, v_host, "bf16", c.block_tables,
                            cl.cpu().numpy(), c.scale)
        assert_close(f64(got), ref, 2e-2, f"graph replay, step {step}")
        assert torch.equal(got.view(torch.int16), want.view(torch.int16)), f"step {step}"
        assert torch.equal(kp_g.view(torch.int16), kp_e.view(torch.int16))
        # next step: new queries, one sequence shorter, another's newest row rewritten
        q.copy_(torch.randn_like(q, dtype=torch.float32).to(torch.bfloat16))
        cl[3] -= 7
        kn.copy_(torch.randn_like(kn, dtype=torch.float32).to(torch.bfloat16))
