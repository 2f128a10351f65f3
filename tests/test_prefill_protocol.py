"""Host model of the prefill kernel's mbarrier protocol (paged_kv_cache_380_b200/csrc/prefill.cu).

Each role of a CTA (K producer, V producer, MMA issuer, the softmax warps of the two query
tiles) is written as the sequence of waits and arrivals the kernel performs, with the
phase each one means.  Arrivals count toward a barrier's current phase, as on the GPU, so
an arrival that lands before the previous phase of its barrier has completed is reported
(it would complete the wrong phase), and so is a wait whose barrier is two phases ahead
(a parity wait could not tell them apart).  The roles are run under several scheduling
orders; every one must finish.  The model caught the K producer's final arrival ("no K
tile after the last one") landing in an earlier phase of its load-step barrier when short
units (local attention) let the V producer lag behind an epilogue's staging area."""
import random

import pytest

KST, VST, BM, BN = 3, 2, 128, 128


def roles_for(units, NT):
    def producer(is_k):
        g = uc = 0
        end_g = [-8, -8]
        nst = KST if is_k else VST
        if not is_k:
            yield ("arrive", ("kv_full", 0), 0)                       # step 0 carries no V tile
        for n_tiles in units:
            if is_k:
                if uc > 0:
                    gl = g - 1
                    yield ("wait", ("s_full", NT - 1, gl % KST), gl // KST)
                yield ("arrive", ("q_full",), uc)
            for _ in range(n_tiles):
                st = g % nst
                if g >= nst:
                    prev = g - nst
                    yield ("wait", ("s_full", NT - 1, st) if is_k else ("pv_done", st), prev // nst)
                    for e in range(2):
                        if not is_k and end_g[e] == prev:
                            ue = uc - 1 - ((uc - 1 - e) & 1)
                            yield ("wait", ("stage_free", ue & 1), ue >> 1)
                step = g if is_k else g + 1
                yield ("arrive", ("kv_full", step % KST), step // KST)
                g += 1
            end_g[uc & 1] = g - 1
            uc += 1
        if is_k:                                                      # the step after the last tile
            if g >= KST:
                yield ("wait", ("s_full", NT - 1, g % KST), (g - KST) // KST)
            yield ("arrive", ("kv_full", g % KST), g // KST)

    def issuer():
        g = uc = 0
        for n_tiles in units:
            g0 = g
            yield ("wait", ("q_full",), uc)
            if g0 == 0:
                yield ("wait", ("kv_full", 0), 0)
            for x in range(NT):
                yield ("arrive", ("s_full", x, g0 % KST), g0 // KST)
            for j in range(n_tiles):
                gg, more = g0 + j, j + 1 < n_tiles
                vs, ks1 = gg % VST, (gg + 1) % KST
                yield ("wait", ("kv_full", ks1), (gg + 1) // KST)
                if j == 0 and uc > 0:
                    yield ("wait", ("o_read", (uc - 1) & 1), (uc - 1) >> 1)
                for x in range(NT):
                    yield ("wait", ("p_half", x), gg)
                    yield ("wait", ("p_full", x), gg)
                    if x == NT - 1:
                        yield ("arrive", ("pv_done", vs), gg // VST)
                    if not more:
                        yield ("arrive", ("o_full", x), uc)
                    if more:
                        yield ("arrive", ("s_full", x, ks1), (gg + 1) // KST)
            g += n_tiles
            uc += 1

    def softmax(x):
        g = uc = 0
        pending = None

        def epilogue(e_uc):
            yield ("wait", ("o_full", NT - 1), e_uc)
            yield ("arrive", ("o_read", e_uc & 1), e_uc >> 1)
            yield ("arrive", ("stage_free", e_uc & 1), e_uc >> 1)

        for n_tiles in units:
            for j in range(n_tiles):
                yield ("wait", ("s_full", x, g % KST), g // KST)
                yield ("arrive", ("p_half", x), g)
                yield ("arrive", ("p_full", x), g)
                if j == 0 and pending is not None:
                    yield from epilogue(pending)
                    pending = None
                g += 1
            pending = uc
            uc += 1
        if pending is not None:
            yield from epilogue(pending)

    roles = {"K": producer(True), "V": producer(False), "MMA": issuer()}
    for x in range(NT):
        for w in range(4):
            roles[f"S{x}{w}"] = softmax(x)
    counts = {"q_full": 1, "kv_full": 2, "s_full": 1, "p_full": 4, "p_half": 4, "pv_done": 1, "o_full": 1,
              "o_read": 4 * NT, "stage_free": 4 * NT}
    return roles, counts


def run(units, NT, order):
    roles, counts = roles_for(units, NT)
    names = order(list(roles))
    done, pend = {}, {}
    cur = {r: next(roles[r], None) for r in names}
    progress = True
    while progress:
        progress = False
        for r in names:
            while cur[r] is not None:
                op, bar, idx = cur[r]
                c = done.get(bar, 0)
                if op == "wait":
                    assert c < idx + 2, f"{r} waits {bar} phase {idx}, {c} phases already done"
                    if c <= idx:
                        break
                else:
                    assert idx == c, f"{r}'s arrival on {bar} meant for phase {idx} lands in phase {c}"
                    pend[bar] = pend.get(bar, 0) + 1
                    if pend[bar] == counts[bar[0]]:
                        done[bar], pend[bar] = c + 1, 0
                cur[r] = next(roles[r], None)
                progress = True
    stuck = {r: v for r, v in cur.items() if v is not None}
    assert not stuck, f"deadlock: {stuck}"


ORDERS = {
    "producers first": lambda rs: ["K", "V", "MMA"] + [r for r in rs if r.startswith("S")],
    "K first, V last": lambda rs: ["K"] + [r for r in rs if r not in ("K", "V")] + ["V"],
    "softmax first": lambda rs: [r for r in rs if r.startswith("S")] + ["MMA", "K", "V"],
    "reversed": lambda rs: list(reversed(rs)),
}


def chunked_prefill_units(cta, grid=148, window=0, nseq=8, n=512, ctx=1536, Hq=32, NT=2):
    """Key-tile counts of the units a CTA walks for the chunked-prefill workload."""
    num_qt = (n + BM - 1) // BM
    out = []
    for u in range(cta, (Hq // NT) * nseq * num_qt, grid):
        qt = num_qt - 1 - (u // (Hq // NT)) // nseq
        r0 = qt * BM
        last_row = min(r0 + BM, n) - 1
        key_lo = max(0, ctx - n + r0 - window + 1) if window > 0 else 0
        out.append((ctx - n + last_row) // BN + 1 - key_lo // BN)
    return out


@pytest.mark.parametrize("order", list(ORDERS))
@pytest.mark.parametrize("window", [0, 512, 128])
def test_chunked_prefill_schedules(order, window):
    for cta in (0, 1, 67, 100, 147):
        run(chunked_prefill_units(cta, window=window), 2, ORDERS[order])


def test_random_unit_mixes():
    rng = random.Random(7)
    for _ in range(1500):
        units = [rng.randint(1, 6) for _ in range(rng.randint(1, 7))]
        run(units, rng.choice((1, 2)), ORDERS[rng.choice(list(ORDERS))])
