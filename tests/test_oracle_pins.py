"""Pins for the fp64 oracle: it is checked against things other than itself.

Closed forms, invariants the method must keep, a library routine
(torch scaled_dot_product_attention / logsumexp in fp64 on CPU, numpy and
torch dtype conversions), brute force on tiny inputs, and hand-derived
golden fixtures under tests/golden/.  CPU only.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_380_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---- helpers (test side: gather with numpy fancy indexing, not the oracle) ----

def gather(pool, bt_row, ps, n):
    """Logical tokens 0..n-1 of one sequence as a contiguous [n, Hkv, D] array."""
    P = pool.shape[0]
    flat = pool.reshape(P * ps, *pool.shape[2:])
    i = np.arange(n)
    return flat[bt_row[i // ps].astype(np.int64) * ps + i % ps]


def as_f64(a, tag):
    if tag == "bf16":
        return W.bf16_bits_to_f32(a).astype(np.float64)
    if tag == "f16":
        return np.asarray(a).view(np.float16).astype(np.float64)
    return np.asarray(a, dtype=np.float64)


def random_paged(rng, B=3, Hq=4, Hkv=2, D=8, ps=4, ctx=(5, 1, 11), extra_pages=3, tag="f64"):
    ctx = np.array(ctx, dtype=np.int32)
    npages = [int(math.ceil(c / ps)) for c in ctx]
    P = sum(npages) + extra_pages
    perm = rng.permutation(P).astype(np.int32)
    bt = np.full((B, max(npages)), -1, dtype=np.int32)
    pos = 0
    for b, n in enumerate(npages):
        bt[b, :n] = perm[pos:pos + n]
        pos += n
    mk = (lambda s: rng.standard_normal(s)) if tag == "f64" else \
        (lambda s: W.to_bf16_bits(rng.standard_normal(s).astype(np.float32)))
    return dict(q=mk((B, Hq, D)), k=mk((P, ps, Hkv, D)), v=mk((P, ps, Hkv, D)), bt=bt, ctx=ctx,
                ps=ps, tag=tag)


def run_decode(c, scale, **kw):
    return oracle.decode(c["q"], c["tag"], c["k"], c["v"], c["tag"], c["bt"], c["ctx"], scale,
                         **kw)


def sdpa_decode(c, scale):
    """torch SDPA (fp64, CPU) on the gathered contiguous K/V, GQA expanded."""
    B, Hq, D = c["q"].shape
    Hkv = c["k"].shape[2]
    out = np.zeros((B, Hq, D))
    for b in range(B):
        n = int(c["ctx"][b])
        if n == 0:
            continue
        K = torch.from_numpy(as_f64(gather(c["k"], c["bt"][b], c["ps"], n), c["tag"]))
        V = torch.from_numpy(as_f64(gather(c["v"], c["bt"][b], c["ps"], n), c["tag"]))
        K = K.permute(1, 0, 2).repeat_interleave(Hq // Hkv, dim=0)  # [Hq, n, D]
        V = V.permute(1, 0, 2).repeat_interleave(Hq // Hkv, dim=0)
        q = torch.from_numpy(as_f64(c["q"][b], c["tag"])).unsqueeze(1)  # [Hq, 1, D]
        o = torch.nn.functional.scaled_dot_product_attention(q, K, V, scale=scale)
        out[b] = o[:, 0, :].numpy()
    return out


# ---- golden fixtures ---------------------------------------------------------

def test_golden_decode_closed_form():
    g = json.load(open(os.path.join(GOLDEN, "decode_closed_form.json")))
    D, ps, P = g["head_dim"], g["page_size"], g["num_pages"]
    bt = np.array([g["block_table"]], dtype=np.int32)
    k = np.full((P, ps, 1, D), np.nan)
    v = np.full((P, ps, 1, D), np.nan)
    for i, (kk, vv) in enumerate(zip(g["keys_logical"], g["values_logical"])):
        k[bt[0, i // ps], i % ps, 0] = kk
        v[bt[0, i // ps], i % ps, 0] = vv
    q = np.array([[g["q"]]])
    out, lse = oracle.decode(q, "f64", k, v, "f64", bt, np.array([3]), g["scale"],
                             return_lse=True)
    np.testing.assert_allclose(out[0, 0], g["expected_out"], rtol=0, atol=1e-12)
    assert abs(lse[0, 0] - g["expected_lse"]) < 1e-12


def test_golden_int8_quant_rows():
    g = json.load(open(os.path.join(GOLDEN, "int8_quant_rows.json")))
    x = np.array(g["rows_f32"], dtype=np.float32)
    codes, scales = oracle.quantize_int8(x, "f32")
    assert scales.tolist() == g["expected_scale_bits"]
    assert codes.tolist() == g["expected_codes"]


# ---- closed forms and invariants named for the oracle ------------------------

def test_single_token_context_returns_v_exactly():
    rng = np.random.default_rng(1)
    c = random_paged(rng, ctx=(1, 1, 1))
    out = run_decode(c, 0.37)
    for b in range(3):
        for h in range(4):
            v0 = gather(c["v"], c["bt"][b], c["ps"], 1)[0, h // 2]
            assert np.array_equal(out[b, h], v0)


def test_constant_v_gives_constant_output():
    rng = np.random.default_rng(2)
    c = random_paged(rng, ctx=(7, 3, 12))
    c["v"][:] = 1.75
    out = run_decode(c, 0.5)
    assert np.max(np.abs(out - 1.75)) < 1e-12


def test_page_permutation_invariance_is_bitwise():
    rng = np.random.default_rng(3)
    c = random_paged(rng, ctx=(9, 4, 13))
    base = run_decode(c, 0.3)
    P = c["k"].shape[0]
    sigma = rng.permutation(P)              # physical page p moves to sigma[p]
    k2 = np.empty_like(c["k"]); v2 = np.empty_like(c["v"])
    k2[sigma] = c["k"]; v2[sigma] = c["v"]
    bt2 = np.where(c["bt"] >= 0, sigma[np.maximum(c["bt"], 0)], -1).astype(np.int32)
    out = run_decode(dict(c, k=k2, v=v2, bt=bt2), 0.3)
    assert np.array_equal(out, base)


@pytest.mark.parametrize("tag", ["f64", "bf16"])
def test_paged_equals_contiguous_sdpa(tag):
    rng = np.random.default_rng(4)
    c = random_paged(rng, B=4, Hq=8, Hkv=2, D=16, ps=4, ctx=(1, 4, 5, 23), tag=tag)
    out = run_decode(c, 0.25)
    ref = sdpa_decode(c, 0.25)
    assert np.max(np.abs(out - ref)) < 1e-12


def test_shared_prefix_equals_private_copies_bitwise():
    rng = np.random.default_rng(5)
    ps, D, Hkv = 4, 8, 2
    prefix_pages, own = 3, 2
    P = prefix_pages + 3 * own + 3 * prefix_pages
    k = rng.standard_normal((P, ps, Hkv, D)); v = rng.standard_normal((P, ps, Hkv, D))
    q = rng.standard_normal((3, 4, D))
    shared = np.arange(prefix_pages)
    bt_shared = np.zeros((3, prefix_pages + own), dtype=np.int32)
    bt_priv = np.zeros_like(bt_shared)
    for b in range(3):
        ownp = prefix_pages + b * own + np.arange(own)
        copy = prefix_pages + 3 * own + b * prefix_pages + np.arange(prefix_pages)
        k[copy] = k[shared]; v[copy] = v[shared]
        bt_shared[b] = np.concatenate([shared, ownp])
        bt_priv[b] = np.concatenate([copy, ownp])
    ctx = np.array([18, 20, 13], dtype=np.int32)
    a = oracle.decode(q, "f64", k, v, "f64", bt_shared, ctx, 0.4)
    b_ = oracle.decode(q, "f64", k, v, "f64", bt_priv, ctx, 0.4)
    assert np.array_equal(a, b_)


def test_brute_force_tiny():
    """Per-key loop with math.exp on tiny inputs (D <= 4, ctx <= 5)."""
    rng = np.random.default_rng(6)
    for trial in range(20):
        D = int(rng.integers(1, 5)); n = int(rng.integers(1, 6)); ps = int(rng.integers(1, 4))
        c = random_paged(rng, B=1, Hq=2, Hkv=1, D=D, ps=ps, ctx=(n,), extra_pages=1)
        scale = float(rng.uniform(0.1, 2.0))
        out = run_decode(c, scale)
        K = gather(c["k"], c["bt"][0], ps, n)[:, 0]
        V = gather(c["v"], c["bt"][0], ps, n)[:, 0]
        for h in range(2):
            qv = c["q"][0, h]
            scores = [scale * sum(qv[d] * K[i][d] for d in range(D)) for i in range(n)]
            m = max(scores)
            w = [math.exp(s - m) for s in scores]
            tot = sum(w)
            want = [sum(w[i] * V[i][d] for i in range(n)) / tot for d in range(D)]
            assert np.max(np.abs(out[0, h] - want)) < 1e-12


def test_one_hot_query_large_scale_picks_argmax_value():
    rng = np.random.default_rng(7)
    c = random_paged(rng, B=1, Hq=1, Hkv=1, D=4, ps=4, ctx=(10,))
    K = gather(c["k"], c["bt"][0], 4, 10)[:, 0]
    c["q"][:] = 0.0
    c["q"][0, 0, 2] = 1.0
    j = int(np.argmax(K[:, 2]))
    gap = np.sort(K[:, 2])[-1] - np.sort(K[:, 2])[-2]
    scale = 800.0 / max(gap, 1e-3)          # scores ~ 1e3 and more: exp would overflow unshifted
    out = run_decode(c, scale)
    V = gather(c["v"], c["bt"][0], 4, 10)[:, 0]
    assert np.max(np.abs(out[0, 0] - V[j])) < 1e-9


def test_zero_query_gives_mean_of_values():
    rng = np.random.default_rng(8)
    c = random_paged(rng, ctx=(6, 2, 9))
    c["q"][:] = 0.0
    out = run_decode(c, 1.0)
    for b in range(3):
        V = gather(c["v"], c["bt"][b], c["ps"], int(c["ctx"][b]))
        for h in range(4):
            assert np.max(np.abs(out[b, h] - V[:, h // 2].mean(axis=0))) < 1e-12


def test_gqa_contiguous_group_mapping():
    """Query head h reads KV head h // (Hq/Hkv) (repeat_interleave), not h % Hkv."""
    rng = np.random.default_rng(9)
    c = random_paged(rng, B=1, Hq=4, Hkv=2, ctx=(7,))
    c["v"][:, :, 0, :] = -1.0
    c["v"][:, :, 1, :] = 5.0
    out = run_decode(c, 0.7)
    assert np.allclose(out[0, 0], -1) and np.allclose(out[0, 1], -1)
    assert np.allclose(out[0, 2], 5) and np.allclose(out[0, 3], 5)


def test_zero_context_gives_zero_row():
    rng = np.random.default_rng(10)
    c = random_paged(rng, ctx=(0, 3, 5))
    out = run_decode(c, 1.0)
    assert np.array_equal(out[0], np.zeros_like(out[0]))


def test_lse_matches_torch_logsumexp():
    rng = np.random.default_rng(11)
    c = random_paged(rng, ctx=(5, 8, 3))
    _, lse = run_decode(c, 0.6, return_lse=True)
    for b in range(3):
        n = int(c["ctx"][b])
        K = torch.from_numpy(gather(c["k"], c["bt"][b], c["ps"], n))
        for h in range(4):
            s = 0.6 * (K[:, h // 2, :] @ torch.from_numpy(c["q"][b, h]))
            assert abs(lse[b, h] - torch.logsumexp(s, 0).item()) < 1e-12


def test_split_kv_merge_algebra():
    """Two partial results over disjoint key ranges, merged by log-sum-exp
    weights, equal the unsplit result (the rule the split-KV combine uses)."""
    rng = np.random.default_rng(12)
    ps = 4
    c = random_paged(rng, B=1, Hq=4, Hkv=2, ps=ps, ctx=(22,), extra_pages=0)
    full = run_decode(c, 0.45)
    cut = 12                                 # a page boundary
    o1, l1 = run_decode(dict(c, ctx=np.array([cut], np.int32)), 0.45, return_lse=True)
    bt2 = np.full_like(c["bt"], -1)
    rest = c["bt"][0, cut // ps:]
    bt2[0, :rest.shape[0]] = rest
    o2, l2 = run_decode(dict(c, bt=bt2, ctx=np.array([22 - cut], np.int32)), 0.45,
                        return_lse=True)
    lse = np.logaddexp(l1, l2)
    merged = np.exp(l1 - lse)[..., None] * o1 + np.exp(l2 - lse)[..., None] * o2
    assert np.max(np.abs(merged - full)) < 1e-12


def test_int8_dequant_path_equals_explicit_dequant():
    rng = np.random.default_rng(13)
    c = random_paged(rng, ctx=(6, 9, 4), tag="bf16")
    kc, ks = oracle.quantize_int8(c["k"], "bf16")
    vc, vs = oracle.quantize_int8(c["v"], "bf16")
    a = oracle.decode(c["q"], "bf16", kc, vc, "i8", c["bt"], c["ctx"], 0.3, k_scales=ks,
                      v_scales=vs)
    kd = kc.astype(np.float64) * as_f64(ks, "f16")[..., None]
    vd = vc.astype(np.float64) * as_f64(vs, "f16")[..., None]
    b_ = oracle.decode(c["q"], "bf16", kd, vd, "f64", c["bt"], c["ctx"], 0.3)
    assert np.array_equal(a, b_)


# ---- prefill ---------------------------------------------------------------

def _prefill_case(rng, chunks=(3, 1, 6), prefix=(5, 0, 7), Hq=4, Hkv=2, D=8, ps=4):
    B = len(chunks)
    ctx = np.array([p + n for p, n in zip(prefix, chunks)], dtype=np.int32)
    c = random_paged(rng, B=B, Hq=Hq, Hkv=Hkv, D=D, ps=ps, ctx=tuple(ctx))
    qs = np.zeros(B + 1, dtype=np.int32)
    qs[1:] = np.cumsum(chunks)
    q = rng.standard_normal((int(qs[-1]), Hq, D))
    return c, q, qs, ctx


@pytest.mark.parametrize("causal", [True, False])
def test_prefill_matches_sdpa_bottom_right(causal):
    rng = np.random.default_rng(14)
    c, q, qs, ctx = _prefill_case(rng)
    out = oracle.prefill(q, "f64", c["k"], c["v"], "f64", c["bt"], qs, ctx, causal, 0.35)
    Hq, Hkv = 4, 2
    for b in range(len(ctx)):
        n, L = int(qs[b + 1] - qs[b]), int(ctx[b])
        K = torch.from_numpy(gather(c["k"], c["bt"][b], c["ps"], L)).permute(1, 0, 2)
        V = torch.from_numpy(gather(c["v"], c["bt"][b], c["ps"], L)).permute(1, 0, 2)
        K = K.repeat_interleave(Hq // Hkv, 0); V = V.repeat_interleave(Hq // Hkv, 0)
        Q = torch.from_numpy(q[qs[b]:qs[b + 1]]).permute(1, 0, 2)      # [Hq, n, D]
        mask = None
        if causal:   # row r sits at position L-n+r and sees keys 0..L-n+r
            mask = torch.arange(L)[None, :] <= (L - n + torch.arange(n))[:, None]
        ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask,
                                                               scale=0.35)
        got = torch.from_numpy(out[qs[b]:qs[b + 1]]).permute(1, 0, 2)
        assert (got - ref).abs().max().item() < 1e-12


def test_prefill_last_row_equals_decode_and_first_row_without_prefix():
    rng = np.random.default_rng(15)
    c, q, qs, ctx = _prefill_case(rng, chunks=(4, 6), prefix=(3, 0))
    out = oracle.prefill(q, "f64", c["k"], c["v"], "f64", c["bt"], qs, ctx, True, 0.5)
    last = np.stack([q[qs[b + 1] - 1] for b in range(2)])
    dec = oracle.decode(last, "f64", c["k"], c["v"], "f64", c["bt"], ctx, 0.5)
    for b in range(2):
        assert np.max(np.abs(out[qs[b + 1] - 1] - dec[b])) < 1e-12
    # sequence 1 has no prefix: its first query row sees key 0 only -> v_0 exactly
    v0 = gather(c["v"], c["bt"][1], c["ps"], 1)[0]
    for h in range(4):
        assert np.array_equal(out[qs[1], h], v0[h // 2])


def test_prefill_rejects_chunk_longer_than_context():
    rng = np.random.default_rng(16)
    c, q, qs, ctx = _prefill_case(rng)
    bad = ctx.copy(); bad[0] = 1
    with pytest.raises(ValueError):
        oracle.prefill(q, "f64", c["k"], c["v"], "f64", c["bt"], qs, bad, True, 0.5)


def test_item_selection_matches_full():
    rng = np.random.default_rng(17)
    c, q, qs, ctx = _prefill_case(rng)
    full = oracle.prefill(q, "f64", c["k"], c["v"], "f64", c["bt"], qs, ctx, True, 0.5)
    items = np.array([0, 7, 13, 38, 5])
    sel = oracle.prefill(q, "f64", c["k"], c["v"], "f64", c["bt"], qs, ctx, True, 0.5,
                         items=items)
    assert np.array_equal(sel, full.reshape(-1, 8)[items])


def test_out_of_range_page_is_an_error():
    rng = np.random.default_rng(18)
    c = random_paged(rng)
    c["bt"][1, 0] = c["k"].shape[0]
    with pytest.raises(ValueError):
        run_decode(c, 1.0)


# ---- element conversions and the quantiser -----------------------------------

def test_bf16_widening_matches_torch_for_all_patterns():
    bits = np.arange(65536, dtype=np.uint16)
    got = oracle.bf16_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])


def test_f16_widening_and_rounding_match_numpy():
    bits = np.arange(65536, dtype=np.uint16)
    got = oracle.f16_to_f64(bits)
    ref = bits.view(np.float16).astype(np.float64)
    ok = ~np.isnan(ref)
    assert np.array_equal(np.isnan(got), ~ok) and np.array_equal(got[ok], ref[ok])
    rng = np.random.default_rng(19)
    x = np.concatenate([rng.standard_normal(4000).astype(np.float32) * 10.0 ** rng.integers(-9, 6, 4000),
                        np.array([65504, 65519.99, 65520, 1e-8, 2.0 ** -24, 2.0 ** -25,
                                  3 * 2.0 ** -26, 6.1e-5, -0.0, 0.0], dtype=np.float32)]).astype(np.float32)
    with np.errstate(over="ignore"):          # values past the fp16 range round to inf on purpose
        want = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(oracle.float_to_f16_bits(x), want)


def test_quantiser_bounds_and_symmetry():
    rng = np.random.default_rng(20)
    x32 = (rng.standard_normal((200, 128)) * rng.uniform(0.01, 5, (200, 1))).astype(np.float32)
    x = W.to_bf16_bits(x32)
    codes, scales = oracle.quantize_int8(x, "bf16")
    xf = W.bf16_bits_to_f32(x).astype(np.float64)
    s = scales.view(np.float16).astype(np.float64)[:, None]
    assert np.all(np.abs(codes.astype(np.int32)) <= 127)
    assert np.all(np.abs(xf - codes * s) <= 0.5 * s * (1 + 1e-6))        # rounding error bound
    am = np.argmax(np.abs(xf), axis=1)
    assert np.all(np.abs(codes[np.arange(200), am]) == 127)              # abs-max maps to +-127
    neg = W.to_bf16_bits(-W.bf16_bits_to_f32(x))
    codes_n, scales_n = oracle.quantize_int8(neg, "bf16")
    assert np.array_equal(scales_n, scales) and np.array_equal(codes_n, -codes)


# ---- scatter -------------------------------------------------------------------

def test_scatter_matches_fancy_index_assignment():
    rng = np.random.default_rng(21)
    P, ps, Hkv, D, T = 6, 4, 2, 8, 9
    kp = W.to_bf16_bits(rng.standard_normal((P, ps, Hkv, D)).astype(np.float32))
    vp = kp.copy() ^ 0x1234
    kn = W.to_bf16_bits(rng.standard_normal((T, Hkv, D)).astype(np.float32))
    vn = kn ^ 0x0F0F
    slots = rng.choice(P * ps, T, replace=False).astype(np.int64)
    slots[3] = -1
    ref_k = kp.copy().reshape(P * ps, Hkv, D); ref_v = vp.copy().reshape(P * ps, Hkv, D)
    keep = slots >= 0
    ref_k[slots[keep]] = kn[keep]; ref_v[slots[keep]] = vn[keep]
    oracle.kv_cache_write(kn, vn, slots, kp, vp)
    assert np.array_equal(kp.reshape(P * ps, Hkv, D), ref_k)
    assert np.array_equal(vp.reshape(P * ps, Hkv, D), ref_v)


def test_scatter_out_of_range_slot_is_an_error():
    kp = np.zeros((2, 4, 1, 8), np.uint16); vp = kp.copy()
    with pytest.raises(ValueError):
        oracle.kv_cache_write(np.ones((1, 1, 8), np.uint16), np.ones((1, 1, 8), np.uint16),
                              np.array([8]), kp, vp)


# ---- local (sliding-window) attention ------------------------------------------

def test_window_covering_the_context_equals_no_window():
    rng = np.random.default_rng(30)
    c = random_paged(rng, ctx=(5, 8, 13))
    assert np.array_equal(run_decode(c, 0.5, window=13), run_decode(c, 0.5))
    c2, q, qs, ctx = _prefill_case(rng)
    a = oracle.prefill(q, "f64", c2["k"], c2["v"], "f64", c2["bt"], qs, ctx, True, 0.5, window=int(ctx.max()))
    b_ = oracle.prefill(q, "f64", c2["k"], c2["v"], "f64", c2["bt"], qs, ctx, True, 0.5)
    assert np.array_equal(a, b_)


def test_window_one_returns_the_own_value():
    rng = np.random.default_rng(31)
    c = random_paged(rng, ctx=(5, 8, 13))
    out = run_decode(c, 0.9, window=1)
    for b in range(3):
        v_last = gather(c["v"], c["bt"][b], c["ps"], int(c["ctx"][b]))[-1]
        for h in range(4):
            assert np.array_equal(out[b, h], v_last[h // 2])


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("window", [1, 3, 6])
def test_window_matches_sdpa_band_mask(window, causal):
    """A query at position pos sees the window's w keys pos-w+1 .. pos when causal; without
    the causal mask the window bounds only the lower side, so it sees pos-w+1 .. ctx-1."""
    rng = np.random.default_rng(32)
    c, q, qs, ctx = _prefill_case(rng)
    out = oracle.prefill(q, "f64", c["k"], c["v"], "f64", c["bt"], qs, ctx, causal, 0.35, window=window)
    Hq, Hkv = 4, 2
    for b in range(len(ctx)):
        n, L = int(qs[b + 1] - qs[b]), int(ctx[b])
        K = torch.from_numpy(gather(c["k"], c["bt"][b], c["ps"], L)).permute(1, 0, 2).repeat_interleave(2, 0)
        V = torch.from_numpy(gather(c["v"], c["bt"][b], c["ps"], L)).permute(1, 0, 2).repeat_interleave(2, 0)
        Q = torch.from_numpy(q[qs[b]:qs[b + 1]]).permute(1, 0, 2)
        pos = (L - n + torch.arange(n))[:, None]
        key = torch.arange(L)[None, :]
        mask = key > pos - window
        if causal:
            mask = mask & (key <= pos)
        ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask, scale=0.35)
        got = torch.from_numpy(out[qs[b]:qs[b + 1]]).permute(1, 0, 2)
        assert (got - ref).abs().max().item() < 1e-12
