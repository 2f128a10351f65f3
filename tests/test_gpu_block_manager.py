"""GPU: the page copy of copy-on-write is bit-exact, and a fork / copy-on-write
/ append / decode pipeline driven by the block manager gives the attention of
each sequence's logical tokens (oracle on an unshared, in-order layout)."""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_close, assert_status_ok, dev, f64, host_bits
from paged_kv_cache_380_b200 import ops
from paged_kv_cache_380_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_copy_pages_bit_exact():
    rng = np.random.default_rng(3)
    P, ps, Hkv, D = 40, 16, 4, 128
    kp = rng.integers(0, 65536, (P, ps, Hkv, D), dtype=np.uint16)
    vp = rng.integers(0, 65536, (P, ps, Hkv, D), dtype=np.uint16)
    src = rng.choice(P, 12, replace=False).astype(np.int32)
    dst = rng.choice(np.setdiff1d(np.arange(P), src), 12, replace=False).astype(np.int32)
    dk, dv = dev(kp, "bf16"), dev(vp, "bf16")
    ops.copy_pages(dk, dv, dev(src, "i32"), dev(dst, "i32"))
    torch.cuda.synchronize()
    assert_status_ok()
    kp[dst], vp[dst] = kp[src], vp[src]
    assert host_bits(dk).tobytes() == kp.tobytes() and host_bits(dv).tobytes() == vp.tobytes()


def test_fork_cow_append_decode_end_to_end():
    rng = np.random.default_rng(4)
    P, ps, Hkv, Hq, D, mp = 64, 16, 2, 8, 128, 16
    bm = ops.BlockManager(P, ps, mp)
    kp = torch.full((P, ps, Hkv, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    vp = torch.full_like(kp, float("nan"))
    logical = {}                                        # seq -> (list of K rows, list of V rows), bf16 bits

    def rows(n):
        return W.to_bf16_bits(rng.standard_normal((n, Hkv, D)).astype(np.float32))

    def append(s, n):
        slots, copies = bm.append(s, n)
        if copies:
            src = torch.tensor([c[0] for c in copies], dtype=torch.int32, device="cuda")
            dst = torch.tensor([c[1] for c in copies], dtype=torch.int32, device="cuda")
            ops.copy_pages(kp, vp, src, dst)
        k, v = rows(n), rows(n)
        ops.kv_cache_write(dev(k, "bf16"), dev(v, "bf16"), dev(slots, "i64"), kp, vp)
        logical[s][0].extend(k)
        logical[s][1].extend(v)
        return copies

    root = bm.add_sequence()
    logical[root] = ([], [])
    append(root, 40)
    kids = []
    for n in (5, 20, 1, 0):
        kid = bm.fork(root)
        logical[kid] = (list(logical[root][0]), list(logical[root][1]))
        kids.append(kid)
        if n:
            assert append(kid, n), "a fork's first append into the shared half-filled page copies it"
    append(root, 7)
    gone = kids.pop(1)
    bm.free(gone)                                       # a finished request releases its pages
    del logical[gone]
    append(kids[0], 33)

    ids = [root] + kids
    table, lens = bm.block_tables(ids)
    q = W.to_bf16_bits(rng.standard_normal((len(ids), Hq, D)).astype(np.float32))
    scale = 1 / math.sqrt(D)
    out = ops.paged_attention_decode(dev(q, "bf16"), kp, vp, dev(table, "i32"), dev(lens, "i32"), scale)
    torch.cuda.synchronize()
    assert_status_ok()
    # oracle: each sequence's logical rows laid out privately and in order
    n_max = max(len(logical[s][0]) for s in ids)
    pages = -(-n_max // ps)
    kq = np.full((len(ids) * pages, ps, Hkv, D), 0x7FC0, dtype=np.uint16)
    vq = kq.copy()
    bt = np.arange(len(ids) * pages, dtype=np.int32).reshape(len(ids), pages)
    for b, s in enumerate(ids):
        n = len(logical[s][0])
        assert lens[b] == n
        flat_k = kq.reshape(-1, Hkv, D)
        flat_v = vq.reshape(-1, Hkv, D)
        flat_k[b * pages * ps: b * pages * ps + n] = np.array(logical[s][0])
        flat_v[b * pages * ps: b * pages * ps + n] = np.array(logical[s][1])
    want = oracle.decode(q, "bf16", kq, vq, "bf16", bt, lens, scale)
    assert_close(f64(out), want, 2e-2, "block-manager pipeline")
    for s in ids:
        bm.free(s)
    assert bm.num_free_pages() == P
