"""CPU model of the forward helper kernel's barrier protocol (csrc/sa_fwd_sm100.cu,
sa_fwd_sm100_helper_kernel): one helper CTA walks its tile range in chunks; per chunk,
pass 1 runs the score MMA and the partial log-sums for every (slice, tile), pass 2 the
score MMA again, the A store and the accumulate MMA. Roles as coroutines: the X producer
(four stages, one tile per step), the P' producer (one buffer, one slice per (pass,
slice) group), the score-MMA and accumulate-MMA
issuers (one in-order tensor pipe), and the two softmax warpgroups (tile parity), of
which warpgroup 0 also runs every segment epilogue; a warpgroup hands its score buffer
back as soon as it has read the scores. TMA landings and pipe completions
come in random order; barriers follow mbarrier phase and parity semantics (a wait can
pass on a stale phase).

Checked on every run: no deadlock; every MMA reads the X stage, P' buffer, S buffer and A
tile of its own step; no TMA, MMA or A store overwrites a buffer in use; a token's running
lse2 is written by one warpgroup, slice after slice, and read in pass 2 only after all C
slices went in; each segment epilogue reads U after its run's last MMA and before the next
run resets it; per (user, slice) the first epilogue stores and the later ones add, all from
one warpgroup, and the runs cover every tile of the user in the range exactly once.
Planted mistakes, each caught: one parity-checked barrier for the single A buffer (a
stale phase lets a store pass), and epilogues run by the warpgroup that owned the run's
last tile (two threads would then read and write one workspace row without an order).
"""
import random

import pytest

from test_fwd_barrier_protocol import Bar, Violation, check
from test_stca_barrier_protocol import _engine


def run_helper(owner, ra, rb, C, chunk, seed, single_a_barrier=False, epilogue_by_last=False):
    """owner[g]: user of global tile g; the CTA's range is tiles [ra, rb)."""
    rnd = random.Random(seed)
    later, issue, run = _engine(rnd)
    NS = 4
    first_tile = {}
    for g, u in enumerate(owner):
        first_tile.setdefault(u, g)
    chunks = [(c0, min(chunk, rb - c0)) for c0 in range(ra, rb, chunk)]
    step_of = {}
    for ci, (c0, K) in enumerate(chunks):
        for ph in range(2):
            for s in range(C):
                for tl in range(K):
                    step_of[(ci, ph, s, tl)] = len(step_of)
    st = dict(x_full=[Bar(1) for _ in range(NS)], x_empty=[Bar(1) for _ in range(NS)],
              s_full=[Bar(1), Bar(1)], s_empty=[Bar(4), Bar(4)], p_full=Bar(1),
              p_empty=Bar(1), a_full=Bar(4), a_empty=[Bar(1) for _ in range(4)],
              u_full=Bar(1), u_empty=Bar(4), m2iss=[Bar(1) for _ in range(4)],
              xstage=[None] * NS, xuse=[0] * NS, pbuf=[None], puse=[0],
              S=[None, None], s_held=[False, False], A=[None], a_use=[0],
              U=dict(seg=None, done=False, read=True), L={}, out={})

    def last_of_run(g, tl, K):
        return tl == K - 1 or g == rb - 1 or owner[g + 1] != owner[g]

    def producer():
        i = 0
        for ci, (c0, K) in enumerate(chunks):
            for ph in range(2):
                for s in range(C):
                    for tl in range(K):
                        sg = i % NS
                        yield lambda: st["x_empty"][sg].passes(((i // NS) & 1) ^ 1)
                        st["x_full"][sg].arrive_expect_tx(1)

                        def land(i=i, sg=sg):
                            check(st["xuse"][sg] == 0, f"X load of step {i} overwrote stage {sg} in use")
                            st["xstage"][sg] = i
                            st["x_full"][sg].complete_tx(1)
                        later(land)
                        i += 1

    def p_producer():
        q = 0
        for ci, (c0, K) in enumerate(chunks):
            for ph in range(2):
                for s in range(C):
                    yield lambda: st["p_empty"].passes((q & 1) ^ 1)
                    st["p_full"].arrive_expect_tx(1)

                    def land_p(q=q):
                        check(st["puse"][0] == 0, f"P' load of group {q} overwrote the buffer in use")
                        st["pbuf"][0] = q
                        st["p_full"].complete_tx(1)
                    later(land_p)
                    q += 1

    def mma1():
        i = q = i2 = 0
        nb = [0, 0]
        for ci, (c0, K) in enumerate(chunks):
            for ph in range(2):
                for s in range(C):
                    pb = 0
                    yield lambda: st["p_full"].passes(q & 1)
                    for tl in range(K):
                        sg, sb = i % NS, tl & 1
                        nbs = nb[sb]
                        yield lambda: (
                            st["x_full"][sg].passes((i // NS) & 1)
                            and st["s_empty"][sb].passes((nbs & 1) ^ 1)
                            and (ph == 0 or i2 < 3 or st["m2iss"][(i2 - 3) & 3].passes(((i2 - 3) >> 2) & 1))
                            and (ph == 0 or i2 < 4 or st["a_empty"][(i2 - 4) & 3].passes(((i2 - 4) >> 2) & 1)))

                        def start(i=i, sg=sg, sb=sb, pb=pb, q=q):
                            check(st["xstage"][sg] == i, f"MMA1({i}) read X stage holding {st['xstage'][sg]}")
                            check(st["pbuf"][pb] == q, f"MMA1({i}) read P' buffer holding group {st['pbuf'][pb]}")
                            check(not st["s_held"][sb], f"MMA1({i}) overwrote S{sb} in use")
                            st["xuse"][sg] += 1
                            st["puse"][pb] += 1

                        def finish(i=i, sg=sg, sb=sb, pb=pb, ph=ph, lastp=(tl == K - 1)):
                            st["xuse"][sg] -= 1
                            st["puse"][pb] -= 1
                            st["S"][sb] = i
                            st["s_full"][sb].arrive()
                            if ph == 0:
                                st["x_empty"][sg].arrive()
                            if lastp:
                                st["p_empty"].arrive()
                        issue(start, finish)
                        nb[sb] += 1
                        i += 1
                        i2 += ph
                    q += 1

    def mma2():
        i = i2 = seg = 0
        for ci, (c0, K) in enumerate(chunks):
            i += C * K
            for s in range(C):
                prev_u = None
                for tl in range(K):
                    g = c0 + tl
                    u = owner[g]
                    first, last = tl == 0 or u != prev_u, last_of_run(g, tl, K)
                    prev_u = u
                    sg = i % NS
                    yield lambda: (st["a_full"].passes(i2 & 1) and
                                   (not first or st["u_empty"].passes((seg & 1) ^ 1)))

                    def start(i=i, i2=i2, sg=sg, first=first, seg=seg):
                        check(st["A"][0] == i2, f"MMA2({i2}) read A holding {st['A'][0]}")
                        check(st["xstage"][sg] == i, f"MMA2({i2}) read X stage holding {st['xstage'][sg]}")
                        if first:
                            check(st["U"]["read"], f"MMA2({i2}) reset U before its epilogue read it")
                            st["U"].update(seg=seg, done=False, read=False)
                        else:
                            check(st["U"]["seg"] == seg, f"MMA2({i2}) accumulated into another run")
                        st["a_use"][0] += 1
                        st["xuse"][sg] += 1

                    def finish(i2=i2, sg=sg, last=last):
                        st["a_use"][0] -= 1
                        st["xuse"][sg] -= 1
                        st["U"]["done"] |= last
                        st["x_empty"][sg].arrive()
                        st["a_empty"][0 if single_a_barrier else (i2 & 3)].arrive()
                        if last:
                            st["u_full"].arrive()
                    issue(start, finish)
                    st["m2iss"][i2 & 3].arrive()
                    seg += last
                    i += 1
                    i2 += 1

    def softmax(w):
        nbw = i2 = useg = 0
        run_g0 = None
        for ci, (c0, K) in enumerate(chunks):
            for ph in range(2):
                for s in range(C):
                    prev_u = None
                    for tl in range(K):
                        g = c0 + tl
                        u = owner[g]
                        sb = tl & 1
                        if ph == 1 and (tl == 0 or u != prev_u):
                            run_g0 = g
                        prev_u = u
                        if sb == w:
                            yield lambda: st["s_full"][sb].passes(nbw & 1)
                            nbw += 1
                            i = step_of[(ci, ph, s, tl)]
                            check(st["S"][sb] == i, f"WG{w} read S{sb} holding {st['S'][sb]} for step {i}")
                            st["s_empty"][sb].arrive(4)  # scores in registers: released at once
                            yield None  # the exponentials
                            if ph == 0:
                                if s == 0:
                                    st["L"][tl] = dict(ci=ci, n=1, w=w)
                                else:
                                    lv = st["L"][tl]
                                    check(lv == dict(ci=ci, n=s, w=w), f"lse2 of tile {tl}: {lv} at slice {s} by WG{w}")
                                    lv["n"] += 1
                            else:
                                lv = st["L"][tl]
                                check(lv == dict(ci=ci, n=C, w=w), f"pass 2 read lse2 of tile {tl}: {lv}")
                                if single_a_barrier:
                                    eb, epar = 0, (i2 & 1) ^ 1
                                else:
                                    eb, epar = (i2 - 1) & 3, ((i2 - 1) >> 2) & 1
                                yield lambda: st["a_empty"][eb].passes(epar)
                                check(st["a_use"][0] == 0, f"A({i2}) stored while MMA2 reads A")
                                st["A"][0] = i2
                                st["a_full"].arrive(4)
                        if ph == 1:
                            epi = (sb == w) if epilogue_by_last else (w == 0)
                            if epi and last_of_run(g, tl, K):
                                yield lambda: st["u_full"].passes(useg & 1)
                                check(st["U"]["done"] and not st["U"]["read"], f"epilogue at tile {g} saw U {st['U']}")
                                useg += 1
                                st["U"]["read"] = True
                                seg_first = run_g0 == ra or run_g0 == first_tile[u]
                                key = (u, s)
                                if seg_first:
                                    check(key not in st["out"], f"segment {key} stored twice")
                                    st["out"][key] = dict(w=w, tiles=g - run_g0 + 1)
                                else:
                                    check(key in st["out"], f"segment {key} added to before its store")
                                    check(st["out"][key]["w"] == w, f"segment {key} written by two warpgroups")
                                    st["out"][key]["tiles"] += g - run_g0 + 1
                                st["u_empty"].arrive(4)
                            i2 += 1

    run([producer(), p_producer(), mma1(), mma2(), softmax(0), softmax(1)])
    want = {}
    for g in range(ra, rb):
        for s in range(C):
            want[(owner[g], s)] = want.get((owner[g], s), 0) + 1
    check({k: v["tiles"] for k, v in st["out"].items()} == want, "runs do not cover the range")


def random_owner(rnd, T):
    owner, u = [], 0
    p_new = rnd.choice([0.05, 0.3, 0.8])
    for g in range(T):
        if g > 0 and rnd.random() < p_new:
            u += rnd.choice([1, 1, 2])  # a skipped user id: a user without tiles
        owner.append(u)
    return owner


@pytest.mark.parametrize("C,chunk", [(8, 4), (8, 5), (3, 3), (5, 2), (2, 1), (1, 3)])
def test_helper_protocol_random_schedules(C, chunk):
    rnd = random.Random(100 * C + chunk)
    for trial in range(60):
        T = rnd.randint(1, 30)
        owner = random_owner(rnd, T)
        ra = rnd.randint(0, T - 1)
        rb = rnd.randint(ra + 1, T)
        run_helper(owner, ra, rb, C, chunk, seed=trial)


def test_helper_protocol_kernel_chunk():
    # the kernel's 32-tile chunks over 70 tiles of three users (two chunks and a ragged one)
    owner = [0] * 20 + [1] * 45 + [3] * 5
    for seed in range(3):
        run_helper(owner, 3, 70, 8, 32, seed)


def test_model_catches_the_single_a_barrier_race():
    rnd = random.Random(11)
    found = 0
    for trial in range(300):
        T = rnd.randint(2, 24)
        owner = random_owner(rnd, T)
        try:
            run_helper(owner, 0, T, rnd.choice([2, 3, 8]), rnd.choice([1, 3, 4]), seed=trial,
                       single_a_barrier=True)
        except Violation:
            found += 1
    assert found > 0


def test_model_catches_epilogues_split_across_warpgroups():
    found = 0
    for trial in range(40):
        owner = [0] * 7 + [1] * 6
        try:
            run_helper(owner, 0, 13, 2, 4, seed=trial, epilogue_by_last=True)
        except Violation:
            found += 1
    assert found > 0
