"""A host-side model of the persistent 64-key pipeline's synchronisation.

The kernel's roles (TMA producer, expander, two MMA issuers, two softmax
warpgroups) wait on mbarrier phases by parity and pass the exp turn between
the two softmax warpgroups through named barriers. This model replays each
role's sequence of waits and arrivals exactly as the kernel orders them, for
1 to 5 pairs per CTA and 1 to 6 key tiles per pair, in random interleavings,
and checks that:
- every wait is eventually satisfied (no deadlock);
- no barrier runs two phases ahead of a waiter (a parity wait would then
  alias to the wrong phase);
- named-barrier arrivals and syncs balance, and no barrier is left with
  pending arrivals.
A planted parity mistake (the P.V completion barrier's phase for pairs with one
key tile) must be caught.
"""
import random

import pytest

KS, BS = 4, 4  # K/V and bias ring stages with a bias


def run(n_items, nkt, rescale, seed, bias=True, od_phase=None):
    rng = random.Random(seed)
    comp, pend, cnt = {}, {}, {}

    def init(b, c):
        comp[b], pend[b], cnt[b] = 0, 0, c

    for s in range(KS):
        init(("kv_full", s), 33)
        init(("kv_empty", s), 2)
    for i in range(BS * 2):
        init(("b_full", i), 1)
        init(("b_empty", i), 128)
    for i in range(4):
        init(("s_full", i), 2)
        init(("p_full", i), 128)
        init(("o_done", i), 1)
    for t in range(2):
        init(("q_ready", t), 128)
    named = {3: [0, 0], 4: [0, 0]}  # [arrive generations, sync generations]
    errors = []
    g_end = n_items * nkt
    od = od_phase or (lambda it: it if nkt >= 2 else it >> 1)

    def arrive(b, n=1):
        pend[b] += n
        assert pend[b] <= cnt[b], b
        if pend[b] == cnt[b]:
            comp[b] += 1
            pend[b] = 0

    def wait(b, k):  # the k-th completion (0-based), waited for by parity k & 1
        while comp[b] < k + 1:
            yield ("wait", b, k)
        if comp[b] > k + 1:
            errors.append(("phase alias", b, k, comp[b]))

    def tma():
        for it in range(n_items):
            for kt in range(nkt):
                g = it * nkt + kt
                s = g % KS
                if g >= KS:
                    yield from wait(("kv_empty", s), g // KS - 1)
                arrive(("kv_full", s))
                if bias:
                    for t2 in range(2):
                        i = (g % BS) * 2 + t2
                        if g >= BS:
                            yield from wait(("b_empty", i), g // BS - 1)
                        arrive(("b_full", i))
                yield ("step",)

    def expander():
        for g in range(g_end):
            s = g % KS
            if g >= KS:
                yield from wait(("kv_empty", s), g // KS - 1)
            arrive(("kv_full", s), 32)
            yield ("step",)

    def issuer(tt):
        def stage_ready(g):
            yield from wait(("kv_full", g % KS), g // KS)
            if bias:
                yield from wait(("b_full", (g % BS) * 2 + tt), g // BS)
            arrive(("s_full", tt * 2 + (g & 1)))

        for it in range(n_items):
            yield from wait(("q_ready", tt), it)
            g0 = it * nkt
            for kt in range(min(2, nkt)):
                yield from stage_ready(g0 + kt)
                arrive(("s_full", tt * 2 + ((g0 + kt) & 1)))  # the QK^T commit
            for kt in range(nkt):
                g = g0 + kt
                bf = g & 1
                yield from wait(("p_full", tt * 2 + bf), g >> 1)
                arrive(("kv_empty", g % KS))
                if kt + 2 < nkt:
                    yield from stage_ready(g + 2)
                    arrive(("s_full", tt * 2 + bf))
                else:
                    arrive(("o_done", tt * 2 + bf))
                yield ("step",)

    def named_sync(bid):
        k = named[bid][1]
        while named[bid][0] < k + 1:
            yield ("named", bid)
        named[bid][1] += 1

    def named_arrive(bid):
        if named[bid][0] >= named[bid][1] + 1:
            errors.append(("named barrier arrived twice", bid))
        named[bid][0] += 1

    def softmax(t):
        if t == 1 and n_items > 0:
            named_arrive(3)  # tile 0 takes the first exp turn
        for it in range(n_items):
            arrive(("q_ready", t), 128)
            for kt in range(nkt):
                g = it * nkt + kt
                bf = g & 1
                yield from wait(("s_full", t * 2 + bf), g >> 1)
                if kt > 0 and rescale(g):  # P.V of the previous tile, before O is rescaled
                    if kt + 1 < nkt:
                        yield from wait(("s_full", t * 2 + ((g + 1) & 1)), (g + 1) >> 1)
                    else:
                        yield from wait(("o_done", t * 2 + ((g - 1) & 1)), od(it))
                yield from named_sync(3 + t)
                if bias:
                    arrive(("b_empty", (g % BS) * 2 + t), 128)
                if not (t == 1 and g == g_end - 1):
                    named_arrive(4 - t)
                arrive(("p_full", t * 2 + bf), 128)
                yield ("step",)
            yield from wait(("o_done", t * 2 + ((it * nkt + nkt - 1) & 1)), od(it))

    roles = {"tma": tma(), "expander": expander(), "issuer0": issuer(0), "issuer1": issuer(1),
             "softmax0": softmax(0), "softmax1": softmax(1)}
    done, last, stuck = set(), {}, 0
    while len(done) < len(roles):
        names = [n for n in roles if n not in done]
        rng.shuffle(names)
        progressed = False
        for n in names:
            try:
                ev = next(roles[n])
            except StopIteration:
                done.add(n)
                progressed = True
                continue
            if ev[0] == "step" or last.get(n) != ev:
                progressed = True
            last[n] = ev if ev[0] != "step" else None
        stuck = 0 if progressed else stuck + 1
        if stuck > 50:
            return errors + [("deadlock", {n: last.get(n) for n in roles if n not in done})]
    if named[3][0] != named[3][1] or named[4][0] != named[4][1]:
        errors.append(("named barriers unbalanced", dict(named)))
    errors += [("pending arrivals", b, pend[b]) for b in comp if pend[b]]
    return errors


RESCALE = {"never": lambda g: False, "always": lambda g: True, "some": lambda g: g % 3 == 1}


@pytest.mark.parametrize("bias", [True, False])
@pytest.mark.parametrize("rescale", sorted(RESCALE))
def test_protocol_every_pair_and_tile_count(bias, rescale):
    for n_items in range(0, 6):
        for nkt in range(1, 7):
            for seed in range(4):
                assert run(n_items, nkt, RESCALE[rescale], seed, bias) == [], (n_items, nkt, seed)


def test_model_catches_a_wrong_phase():
    # with one key tile per pair, each pair alternates between the two P.V
    # completion barriers: waiting for phase `it` instead of `it >> 1` hangs
    errs = run(2, 1, RESCALE["never"], 0, True, od_phase=lambda it: it)
    assert errs and errs[-1][0] == "deadlock"
