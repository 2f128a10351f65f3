"""GPU parity: causal chunked prefill over a paged cache with a shared prefix,
against the fp64 oracle (max abs error 2e-2 for bf16/fp16)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_close, assert_status_ok, dev, f64
from paged_kv_cache_380_b200 import ops
from paged_kv_cache_380_b200 import workloads as W

pytestmark = pytest.mark.gpu


def run_prefill(case, causal=True, items=None, tol=2e-2, window=0):
    """Append the chunk's K/V (cache write), then prefill; compare with the oracle."""
    tag = case.dtype
    kp, vp = dev(case.k_pages, tag), dev(case.v_pages, tag)
    ops.kv_cache_write(dev(case.k_new, tag), dev(case.v_new, tag), dev(case.slot_mapping, "i64"), kp, vp)
    k_host, v_host = case.k_pages.copy(), case.v_pages.copy()
    oracle.kv_cache_write(case.k_new, case.v_new, case.slot_mapping, k_host, v_host)
    q = dev(case.q, tag)
    max_q = int(np.max(np.diff(case.q_start))) if case.batch else 0
    out = ops.paged_attention_prefill(q, kp, vp, dev(case.block_tables, "i32"), dev(case.q_start, "i32"),
                                      dev(case.context_lens, "i32"), causal, case.scale, max_q_len=max_q,
                                      window=window)
    torch.cuda.synchronize()
    assert_status_ok()
    want = oracle.prefill(case.q, tag, k_host, v_host, tag, case.block_tables, case.q_start,
                          case.context_lens, causal, case.scale, items=items, window=window)
    got = f64(out)
    got = got.reshape(-1, got.shape[-1])[items] if items is not None else got
    assert_close(got, want, tol, case.name)


def case(idx, chunks, private_prefix=0, shared_prefix=32, Hq=8, Hkv=2, ps=16, dtype="bf16", D=128):
    return W.prefill_case(name=f"prefill{idx}", config_index=200 + idx, num_seqs=len(chunks),
                          num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D, page_size=ps, dtype=dtype,
                          shared_prefix=shared_prefix, chunk_lens=np.array(chunks),
                          private_prefix=private_prefix)


@pytest.mark.parametrize("causal", [True, False])
def test_ragged_chunks_and_prefixes(causal):
    # chunks shorter than a tile, exactly a tile, ragged tails; chunks start mid-page
    run_prefill(case(1, chunks=(1, 5, 64, 130, 200, 128), private_prefix=7), causal=causal)


def test_no_prefix():
    run_prefill(case(2, chunks=(1, 17, 300), shared_prefix=0))


def test_long_prefix_short_chunk():
    run_prefill(case(3, chunks=(3, 1, 70), shared_prefix=1024, private_prefix=100))


def test_mha_and_large_pages():
    run_prefill(case(4, chunks=(90, 257), Hq=4, Hkv=4, ps=256, shared_prefix=256, private_prefix=3))


def test_fp16():
    run_prefill(case(5, chunks=(40, 129), dtype="f16", private_prefix=11))


def test_empty_sequence_in_batch():
    run_prefill(case(6, chunks=(0, 50, 0, 3)))


def test_chunked_prefill_shared_prefix_full():
    """8 x 512 rows after a shared 1024-token prefix; sampled rows checked."""
    c = W.chunked_prefill_shared_prefix()
    rng = np.random.default_rng(0)
    Hq = c.num_q_heads
    T = c.q.shape[0]
    items = set(rng.choice(T * Hq, 3000, replace=False).tolist())
    for t in (0, 1, 127, 128, 255, 511, 512, 1023, 2047, 4095):   # tile edges, sequence edges
        items |= {t * Hq + h for h in range(Hq)}
    run_prefill(c, items=np.array(sorted(items)))


# ---- local (sliding-window) attention ---------------------------------------------

@pytest.mark.parametrize("window", [512, 128])
def test_chunked_prefill_shared_prefix_full_window(window):
    """The full chunked-prefill workload under local attention, in the launch shape the
    bench times: every work unit has only a few key tiles, so a CTA walks many short units
    (the load-step barrier's last arrival of each CTA must wait like a K tile, or it can
    complete an earlier step's phase while the V warp still lags behind an epilogue)."""
    c = W.chunked_prefill_shared_prefix()
    rng = np.random.default_rng(1)
    Hq = c.num_q_heads
    T = c.q.shape[0]
    items = set(rng.choice(T * Hq, 2000, replace=False).tolist())
    for t in (0, 127, 128, 511, 512, 4095):
        items |= {t * Hq + h for h in range(Hq)}
    run_prefill(c, items=np.array(sorted(items)), window=window)


@pytest.mark.parametrize("window", [1, 64, 128, 129, 300])
def test_sliding_window_prefill(window):
    run_prefill(case(20, chunks=(1, 5, 64, 130, 200, 128), private_prefix=7, shared_prefix=256), window=window)


def test_sliding_window_prefill_non_causal():
    run_prefill(case(21, chunks=(40, 129), private_prefix=3), causal=False, window=50)


# ---- more page sizes, GQA groups and batch shapes ----------------------------------

@pytest.mark.parametrize("ps", [32, 64])
def test_mid_size_pages(ps):
    # 2 or 4 sixteen-row TMA page groups per page; chunks start mid-page
    run_prefill(case(7 + ps // 32, chunks=(1, 31, 129, 200), private_prefix=5, shared_prefix=64, ps=ps))


@pytest.mark.parametrize("Hq,Hkv", [(16, 2), (16, 1)])
def test_large_gqa_groups(Hq, Hkv):
    # 8 and 16 query heads read the same KV head
    run_prefill(case(10 + Hkv, chunks=(77, 130), Hq=Hq, Hkv=Hkv, private_prefix=9))


def test_many_ragged_sequences():
    # 40 sequences, seeded chunk lengths 0..149 (some empty), one shared prefix
    chunks = np.random.default_rng(7).integers(0, 150, 40)
    run_prefill(case(13, chunks=tuple(int(c) for c in chunks), private_prefix=3, shared_prefix=48))


# ---- head_dim 64, and query-head groups that cannot be paired ----------------------

@pytest.mark.parametrize("causal", [True, False])
def test_head_dim_64(causal):
    # ragged chunks after a shared and a private prefix, chunks starting mid-page
    run_prefill(case(30, chunks=(1, 5, 64, 130, 200, 128), private_prefix=7, D=64), causal=causal)


@pytest.mark.parametrize("window", [1, 100, 129])
def test_head_dim_64_sliding_window(window):
    run_prefill(case(31, chunks=(3, 140, 77), private_prefix=5, shared_prefix=256, D=64), window=window)


def test_head_dim_64_fp16_large_pages():
    run_prefill(case(32, chunks=(90, 257), Hq=4, Hkv=4, ps=256, shared_prefix=256, private_prefix=3, D=64,
                     dtype="f16"))


@pytest.mark.parametrize("Hq,Hkv", [(6, 2), (3, 1)])
def test_odd_group_sizes(Hq, Hkv):
    # groups of 3 query heads: one query tile per CTA instead of a pair
    run_prefill(case(33 + Hq, chunks=(17, 130, 256), Hq=Hq, Hkv=Hkv, private_prefix=9))


# ---- many work units per CTA (the kernel walks its units persistently) --------------

@pytest.mark.parametrize("window", [0, 200])
def test_many_units_per_cta(window):
    # 160 sequences with seeded chunk lengths 0..400 and private prefixes: several hundred
    # (head pair, sequence, query tile) units, many of them empty, walked by each CTA in turn
    rng = np.random.default_rng(11)
    chunks = tuple(int(c) for c in rng.integers(0, 400, 160))
    run_prefill(case(40, chunks=chunks, private_prefix=5, shared_prefix=32, Hq=4, Hkv=2), window=window)


def test_many_units_head_dim_64_non_causal():
    rng = np.random.default_rng(12)
    chunks = tuple(int(c) for c in rng.integers(1, 300, 120))
    run_prefill(case(41, chunks=chunks, private_prefix=0, shared_prefix=64, Hq=6, Hkv=3, D=64), causal=False)


# ---- scores whose row maximum keeps rising (the reference-max raise path) ----------

def _to_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    return W.to_bf16_bits(x) if dtype == "bf16" else x.astype(np.float16).view(np.uint16)


def _from_bits(b: np.ndarray, dtype: str) -> np.ndarray:
    return W.bf16_bits_to_f32(b) if dtype == "bf16" else b.view(np.float16).astype(np.float32)


def rising_scores(c, step_log2: float = 12.0):
    """Rewrite a prefill case so that, for even query heads, the scaled score of key
    position t grows by about step_log2 (log2 units) every 64 keys: every half of every
    128-key tile raises the row maximum past the lazy-rescale threshold.  Odd heads see
    the mirror image (falling scores: the first keys hold the maximum)."""
    dt, D, ps = c.dtype, c.head_dim, c.page_size
    rng = np.random.default_rng(5)
    u = np.ones(D, dtype=np.float32) / np.sqrt(D)
    slope = step_log2 / 64.0 / (c.scale * np.log2(np.e))         # q.k growth per key
    q = 0.1 * rng.standard_normal(c.q.shape).astype(np.float32)
    q[:, 0::2, :] += u
    q[:, 1::2, :] -= u
    c.q = _to_bits(q, dt)
    kp, kn = _from_bits(c.k_pages, dt), _from_bits(c.k_new, dt)
    for b in range(len(c.context_lens)):
        ctx, n = int(c.context_lens[b]), int(c.q_start[b + 1] - c.q_start[b])
        for t in range(ctx):
            row = slope * t * u + 0.1 * rng.standard_normal((c.num_kv_heads, D)).astype(np.float32)
            if t < ctx - n:
                pg = int(c.block_tables[b, t // ps])
                kp[pg, t % ps] = row
            else:
                kn[int(c.q_start[b]) + t - (ctx - n)] = row
    c.k_pages, c.k_new = _to_bits(kp, dt), _to_bits(kn, dt)
    return c


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("f16", 128), ("bf16", 64)])
def test_rising_row_maximum(dtype, D):
    # chunks over several key tiles, ragged, after shared and private prefixes
    c = rising_scores(case(50 + D // 64 + (dtype == "f16"), chunks=(300, 129, 40), private_prefix=9,
                           shared_prefix=64, dtype=dtype, D=D))
    run_prefill(c)


def test_rising_row_maximum_window_and_non_causal():
    c = rising_scores(case(55, chunks=(260, 77), private_prefix=5, shared_prefix=128))
    run_prefill(c, window=150)
    c = rising_scores(case(56, chunks=(260, 77), private_prefix=5, shared_prefix=128))
    run_prefill(c, causal=False)
