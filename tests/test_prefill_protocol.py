"""Host model of the prefill kernel's mbarrier protocol (paged_kv_cache_380_b200/csrc/prefill.cu).

Each role of a CTA (K producer, V producer, MMA issuer, the softmax warps of the two query
tiles) is written as the sequence of waits and arrivals the kernel performs, with the
phase each one means.  Arrivals count toward a barrier's current phase, as on the GPU, so
an arrival that lands before the previous phase of its barrier has completed is reported
(it would complete the wrong phase), and so is a wait whose barrier is two phases ahead
(a parity wait could not tell them apart).  Buffer reuse is checked too: before a K or V
stage or the Q buffers are refilled, every query tile's S or P.V that read them must have
been signalled, and a unit's epilogue (which stages its output in the V stage of the unit's
last key tile) needs every tile's last P.V; a role states such a need as a "require" event,
checked when the role reaches it.  A commit signals, with its barrier's phase, every MMA the
issuing thread issued before it (tcgen05 MMAs of one thread complete in issue order).  The
roles run under fixed orders (each role as far as it can go, in turn) and under random
schedules (one operation at a time of a role picked at random), so that any role may fall
far behind the others; every run must finish.  The model caught the K producer's final
arrival ("no K tile after the last one") landing in an earlier phase of its load-step
barrier when short units (local attention) let the V producer lag behind an epilogue's
staging area."""
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
                    yield ("require", [("S", x, gl) for x in range(NT)], None)
                yield ("arrive", ("q_full",), uc)
            for _ in range(n_tiles):
                st = g % nst
                if g >= nst:
                    prev = g - nst
                    # one issuer, in order: the last tile's S (PV) done means every tile's is
                    yield ("wait", ("s_full", NT - 1, st) if is_k else ("pv_done", st), prev // nst)
                    for e in range(2):
                        if not is_k and end_g[e] == prev:
                            ue = uc - 1 - ((uc - 1 - e) & 1)
                            yield ("wait", ("stage_free", ue & 1), ue >> 1)
                if g >= nst:
                    yield ("require", [("S" if is_k else "PV", x, g - nst) for x in range(NT)], None)
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
        # one thread issues both tiles' MMAs; they complete in issue order, so a commit's
        # barrier phase also signals every MMA issued before it
        g = uc = 0
        issued = []

        def commit(bar, phase, ev=None):
            evs = issued + ([ev] if ev else [])
            issued.clear()
            return ("arrive", bar, phase, evs)

        for n_tiles in units:
            g0 = g
            yield ("wait", ("q_full",), uc)
            if g0 == 0:
                yield ("wait", ("kv_full", 0), 0)
            for x in range(NT):
                yield commit(("s_full", x, g0 % KST), g0 // KST, ("S", x, g0))
            for j in range(n_tiles):
                gg, more = g0 + j, j + 1 < n_tiles
                vs, ks1 = gg % VST, (gg + 1) % KST
                yield ("wait", ("kv_full", ks1), (gg + 1) // KST)
                if j == 0 and uc > 0:
                    yield ("wait", ("o_read", (uc - 1) & 1), (uc - 1) >> 1)
                for x in range(NT):
                    yield ("wait", ("p_half", x), gg)
                    yield ("wait", ("p_full", x), gg)
                    issued.append(("PV", x, gg))
                    if x == NT - 1:
                        yield commit(("pv_done", vs), gg // VST)
                    if not more:
                        yield commit(("o_full", x), uc)
                    if more:
                        yield commit(("s_full", x, ks1), (gg + 1) // KST, ("S", x, gg + 1))
            g += n_tiles
            uc += 1

    def softmax(x):
        g = uc = 0
        pending = None

        def epilogue(e_uc, g_last):
            yield ("wait", ("o_full", NT - 1), e_uc)
            yield ("require", [("PV", y, g_last) for y in range(NT)], None)
            yield ("arrive", ("o_read", e_uc & 1), e_uc >> 1)
            yield ("arrive", ("stage_free", e_uc & 1), e_uc >> 1)

        for n_tiles in units:
            for j in range(n_tiles):
                yield ("wait", ("s_full", x, g % KST), g // KST)
                yield ("arrive", ("p_half", x), g)
                yield ("arrive", ("p_full", x), g)
                if j == 0 and pending is not None:
                    yield from epilogue(*pending)
                    pending = None
                g += 1
            pending = (uc, g - 1)
            uc += 1
        if pending is not None:
            yield from epilogue(*pending)

    roles = {"K": producer(True), "V": producer(False), "MMA": issuer()}
    for x in range(NT):
        for w in range(4):
            roles[f"S{x}{w}"] = softmax(x)
    counts = {"q_full": 1, "kv_full": 2, "s_full": 1, "p_full": 4, "p_half": 4, "pv_done": 1, "o_full": 1,
              "o_read": 4 * NT, "stage_free": 4 * NT}
    return roles, counts


def run(units, NT, order=None, rng=None):
    """Run the roles to the end: with `order`, each role in turn as far as it can go; with
    `rng`, one operation at a time of a role picked at random among those that can proceed
    (so any role may fall arbitrarily far behind the others)."""
    roles, counts = roles_for(units, NT)
    names = list(roles) if order is None else order(list(roles))
    done, pend = {}, {}
    signalled, pend_ev = set(), {}     # events ("S"/"PV", tile x, key tile) whose barrier phase completed
    cur = {r: next(roles[r], None) for r in names}

    def ready(r):
        op = cur[r]
        if op is None:
            return False
        if op[0] == "wait":
            assert done.get(op[1], 0) < op[2] + 2, f"{r} waits {op[1]} phase {op[2]}, {done.get(op[1], 0)} done"
            return done.get(op[1], 0) > op[2]
        return True

    def execute(r):
        op, bar, idx = cur[r][:3]
        if op == "require":
            missing = [ev for ev in bar if ev not in signalled]
            assert not missing, f"{r} reuses a buffer before {missing} were signalled"
        elif op == "arrive":
            c = done.get(bar, 0)
            assert idx == c, f"{r}'s arrival on {bar} meant for phase {idx} lands in phase {c}"
            if len(cur[r]) > 3:
                pend_ev.setdefault(bar, []).extend(cur[r][3])
            pend[bar] = pend.get(bar, 0) + 1
            if pend[bar] == counts[bar[0]]:
                done[bar], pend[bar] = c + 1, 0
                signalled.update(pend_ev.pop(bar, []))
        cur[r] = next(roles[r], None)

    if rng is None:
        progress = True
        while progress:
            progress = False
            for r in names:
                while ready(r):
                    execute(r)
                    progress = True
    else:
        while True:
            able = [r for r in names if ready(r)]
            if not able:
                break
            execute(rng.choice(able))
    stuck = {r: v for r, v in cur.items() if v is not None}
    assert not stuck, f"deadlock: {stuck}"


ORDERS = {
    "producers first": lambda rs: ["K", "V"] + [r for r in rs if r.startswith("M")] + [r for r in rs if r.startswith("S")],
    "K first, V last": lambda rs: ["K"] + [r for r in rs if r not in ("K", "V")] + ["V"],
    "softmax first": lambda rs: [r for r in rs if r.startswith("S")] + [r for r in rs if r.startswith("M")] + ["K", "V"],
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


@pytest.mark.parametrize("window", [0, 512, 128])
def test_random_schedules_chunked_prefill(window):
    rng = random.Random(11 + window)
    for cta in (0, 100, 147):
        units = chunked_prefill_units(cta, window=window)
        for _ in range(40):
            run(units, 2, rng=rng)


def test_random_schedules_random_units():
    rng = random.Random(5)
    for _ in range(400):
        units = [rng.randint(1, 5) for _ in range(rng.randint(1, 5))]
        run(units, rng.choice((1, 2)), rng=rng)
