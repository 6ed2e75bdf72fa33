"""CPU model of the single-pass backward kernel's barrier protocol (csrc/sa_bwd_fused.cu).

One cluster of C CTAs walks a tile range. Per CTA the model runs the kernel's roles as
coroutines: the TMA producer (X stages, and Gh and c whenever the user changes), the MMA
issuer (S and dA' of tile i + 1 ahead of dX_part and dPn of tile i when both tiles have
the same user, after them at a user boundary), the two elementwise warpgroups (pass 1,
the local combine of D's halves, the cluster exchange, pass 2 into the A and dS tiles)
and the dX epilogue. TMA landings, tensor-pipe completions (one in-order pipe per CTA)
and st.async deliveries complete in random order; barriers follow mbarrier phase and
parity semantics, so a wait can pass on a stale phase.

Checked on every run: no deadlock; every MMA reads the X stage, Gh, S/dA', A and dS of
its own tile (or user); no TMA, MMA or store overwrites a buffer still in use; both
warpgroups read c, S and dA' of their own tile; warpgroup 0 reads the other half's D of
its tile; every exchange slot read holds the right tile from every CTA and no partial
lands on an unread slot; the epilogue reads dX_part of its own tile. Two planted
variants must be caught: issuing the next tile's dA' MMA ahead of dX_part across a user
boundary (Gh would change under its reader), pass 2 storing A and dS without waiting
for the previous tile's dX_part and dPn MMAs, and the reduction issuer releasing a
staging buffer while its reduction may still read it. The dX staging ring (the epilogue
warps fill NB buffers, one thread issues the TMA reduce-adds and keeps NB - 1 reading)
is modelled with its own barriers.
"""
import heapq
import random

import pytest

from test_fwd_barrier_protocol import Bar, Violation, check, random_tiles


def run_cluster(tiles, C, NS, NX, seed, reorder_across_users=False, tiles_free_wait=True,
                NB=3, chunks=8, inflight=None):
    """NB staging buffers of dX chunks (chunks per tile); the reduction issuer keeps up to
    `inflight` reductions reading (NB - 1 in the kernel)."""
    inflight = NB - 1 if inflight is None else inflight
    rnd = random.Random(seed)
    T = len(tiles)
    seg_of = []
    s = -1
    for (_, first, _) in tiles:
        s += first
        seg_of.append(s)
    events, clock, seq = [], [0], [0]

    def later(fn, lo=1, hi=60):
        seq[0] += 1
        heapq.heappush(events, (clock[0] + rnd.randint(lo, hi), seq[0], fn))

    ctas = [dict(
        x_full=[Bar(1) for _ in range(NS)], x_empty=[Bar(1) for _ in range(NS)],
        p_full=Bar(1), g_full=Bar(1), g_empty=Bar(1),
        s_full=Bar(1), ds_full=Bar(8), dhalf=Bar(4), tiles_free=Bar(1),
        dx_full=Bar(1), dx_empty=Bar(4),
        xch=[Bar(1) for _ in range(NX)],
        slot=[[None] * C for _ in range(NX)], read=[[True] * C for _ in range(NX)],
        xstage=[None] * NS, xuse=[0] * NS, gh=None, gh_use=0, c_seg=None, c_readers=0,
        SG=None, sg_readers=0, AD=None, ad_use=0, dX=None, dx_held=False, dloc=None,
        stg_full=[Bar(4) for _ in range(NB)], stg_free=[Bar(1) for _ in range(NB)],
        stg=[None] * NB, stg_reading=[False] * NB, reads=[], red_done=[],
        pipe=[], busy=[False]) for _ in range(C)]

    def kick(cs):
        if cs["busy"][0] or not cs["pipe"]:
            return
        start, finish = cs["pipe"].pop(0)
        cs["busy"][0] = True
        start()

        def done():
            finish()
            cs["busy"][0] = False
            kick(cs)
        later(done, 1, 30)

    def producer(c):
        cs = ctas[c]
        seg = -1
        for i in range(T):
            if tiles[i][1]:
                seg += 1
                yield lambda: cs["g_empty"].passes((seg & 1) ^ 1)
                cs["g_full"].arrive_expect_tx(1)

                def land_g(seg=seg):
                    check(cs["gh_use"] == 0 and cs["c_readers"] == 0,
                          f"Gh/c of segment {seg} landed while segment {cs['gh']} is read")
                    cs["gh"], cs["c_seg"] = seg, seg
                    cs["g_full"].complete_tx(1)
                later(land_g)
            st = i % NS
            yield lambda: cs["x_empty"][st].passes(((i // NS) & 1) ^ 1)
            cs["x_full"][st].arrive_expect_tx(1)

            def land(i=i, st=st):
                check(cs["xuse"][st] == 0, f"TMA of tile {i} overwrote X stage {st} in use")
                cs["xstage"][st] = i
                cs["x_full"][st].complete_tx(1)
            later(land)

    def mma(c):
        cs = ctas[c]

        def sg(j):
            st = j % NS

            def start(j=j, st=st):
                check(cs["xstage"][st] == j, f"S({j}) read X stage holding {cs['xstage'][st]}")
                check(cs["gh"] == seg_of[j], f"dA'({j}) read Gh of segment {cs['gh']}")
                check(cs["sg_readers"] == 0, f"S({j}) overwrote S/dA' of tile {cs['SG']} in use")
                cs["xuse"][st] += 1
                cs["gh_use"] += 1

            def finish(j=j, st=st):
                cs["xuse"][st] -= 1
                cs["gh_use"] -= 1
                cs["SG"] = j
                cs["s_full"].arrive()
            cs["pipe"].append((start, finish))
            kick(cs)

        yield lambda: cs["x_full"][0].passes(0) and cs["g_full"].passes(0)
        sg(0)
        seg = 0
        for i in range(T):
            st, last = i % NS, tiles[i][2]
            more = i + 1 < T
            same = more and (not last or reorder_across_users)
            s1 = (i + 1) % NS
            yield lambda: cs["ds_full"].passes(i & 1)
            if same:
                yield lambda: cs["x_full"][s1].passes(((i + 1) // NS) & 1)
                sg(i + 1)
            yield lambda: cs["dx_empty"].passes((i & 1) ^ 1)

            def start_dx(i=i, st=st):
                check(cs["AD"] == i, f"dX_part({i}) read A/dS of tile {cs['AD']}")
                check(cs["gh"] == seg_of[i], f"dX_part({i}) read Gh of segment {cs['gh']}")
                check(not cs["dx_held"], f"dX_part({i}) overwrote dX_part({cs['dX']}) in use")
                cs["ad_use"] += 1
                cs["gh_use"] += 1

            def finish_dx(i=i):
                cs["ad_use"] -= 1
                cs["gh_use"] -= 1
                cs["dX"] = i
                cs["dx_full"].arrive()

            def start_dp(i=i, st=st):
                check(cs["AD"] == i and cs["xstage"][st] == i, f"dPn({i}) read the wrong dS or X")
                cs["ad_use"] += 1
                cs["xuse"][st] += 1

            def finish_dp(i=i, st=st, last=last):
                cs["ad_use"] -= 1
                cs["xuse"][st] -= 1
                cs["x_empty"][st].arrive()
                cs["tiles_free"].arrive()
                if last:
                    cs["g_empty"].arrive()
            cs["pipe"].append((start_dx, finish_dx))
            cs["pipe"].append((start_dp, finish_dp))
            kick(cs)
            if more and not same:
                seg += 1
                yield lambda: (cs["x_full"][s1].passes(((i + 1) // NS) & 1) and
                               cs["g_full"].passes(seg & 1))
                sg(i + 1)

    def elementwise(c, hh):
        cs = ctas[c]
        seg = -1
        for i in range(T):
            if tiles[i][1]:
                seg += 1
            yield lambda: cs["s_full"].passes(i & 1) and (not tiles[i][1] or cs["g_full"].passes(seg & 1))
            check(cs["SG"] == i, f"WG{hh} pass 1 of tile {i} read S/dA' of tile {cs['SG']}")
            check(cs["c_seg"] == seg, f"WG{hh} read c of segment {cs['c_seg']} for tile {i}")
            cs["sg_readers"] += 1
            cs["c_readers"] += 1
            yield None  # pass 1
            q = i % NX
            if hh == 1:
                cs["dloc"] = i
                cs["dhalf"].arrive(4)
            else:
                yield lambda: cs["dhalf"].passes(i & 1)
                check(cs["dloc"] == i, f"WG0 read the other half's D of tile {cs['dloc']} for {i}")
                for p in range(C):
                    def deliver(p=p, i=i, q=q):
                        peer = ctas[p]
                        check(peer["read"][q][c], f"tile {i} partial overwrote an unread slot {q} of CTA {p}")
                        peer["slot"][q][c], peer["read"][q][c] = i, False
                        peer["xch"][q].complete_tx(1)
                    later(deliver, 1, 80)
                cs["xch"][q].arrive_expect_tx(C)
            yield lambda: cs["xch"][q].passes((i // NX) & 1)
            for src in range(C):
                check(cs["slot"][q][src] == i, f"slot {q} from CTA {src} holds tile {cs['slot'][q][src]}, not {i}")
            cs.setdefault("slot_reads", {}).setdefault((q, i), 0)
            cs["slot_reads"][(q, i)] += 1
            if cs["slot_reads"][(q, i)] == 2:  # both warpgroups have read it
                for src in range(C):
                    cs["read"][q][src] = True
            if i > 0 and tiles_free_wait:
                yield lambda: cs["tiles_free"].passes((i - 1) & 1)
            check(cs["ad_use"] == 0, f"pass 2 of tile {i} stored A/dS while an MMA reads them")
            check(cs["SG"] == i, f"WG{hh} pass 2 of tile {i} read S/dA' of tile {cs['SG']}")
            yield None  # pass 2
            cs["AD"] = i
            cs["sg_readers"] -= 1
            cs["c_readers"] -= 1
            cs["ds_full"].arrive(4)

    def epilogue(c):
        cs = ctas[c]
        n = 0
        for i in range(T):
            yield lambda: cs["dx_full"].passes(i & 1)
            check(cs["dX"] == i, f"epilogue of tile {i} read dX_part({cs['dX']})")
            cs["dx_held"] = True
            for ch in range(chunks):
                if ch == chunks - 1:  # the last TMEM load of the tile
                    cs["dx_held"] = False
                    cs["dx_empty"].arrive(4)
                b = n % NB
                if n >= NB:
                    yield lambda: cs["stg_free"][b].passes((n // NB - 1) & 1)
                check(not cs["stg_reading"][b], f"chunk {n} overwrote staging {b} while a reduction reads it")
                cs["stg"][b] = (i, ch)
                cs["stg_full"][b].arrive(4)
                n += 1

    def issuer(c):
        cs = ctas[c]
        n = 0
        for i in range(T):
            for ch in range(chunks):
                b = n % NB
                yield lambda: cs["stg_full"][b].passes((n // NB) & 1)
                check(cs["stg"][b] == (i, ch), f"reduction of chunk {(i, ch)} read staging holding {cs['stg'][b]}")
                cs["stg_reading"][b] = True
                cs["reads"].append(n)

                def read_done(b=b, n=n):
                    cs["stg_reading"][b] = False
                    cs["red_done"].append(n)
                later(read_done, 1, 90)
                # wait_group.read: all but the newest `inflight` reductions have read
                yield lambda: all(m in cs["red_done"] for m in cs["reads"][:max(0, len(cs["reads"]) - inflight)])
                if n >= inflight:
                    cs["stg_free"][(n - inflight) % NB].arrive()
                n += 1

    agents = []
    for c in range(C):
        agents += [producer(c), mma(c), elementwise(c, 0), elementwise(c, 1), epilogue(c), issuer(c)]
    waiting, alive = [None] * len(agents), [True] * len(agents)
    for k, a in enumerate(agents):
        try:
            waiting[k] = next(a)
        except StopIteration:
            alive[k] = False
    while True:
        ready = [k for k in range(len(agents)) if alive[k] and (waiting[k] is None or waiting[k]())]
        if ready and (not events or rnd.random() < 0.6):
            k = rnd.choice(ready)
            try:
                waiting[k] = agents[k].send(None)
            except StopIteration:
                alive[k] = False
        elif events:
            t, _, fn = heapq.heappop(events)
            clock[0] = max(clock[0], t)
            fn()
        elif any(alive):
            raise Violation(f"deadlock: roles {[k % 6 for k in range(len(agents)) if alive[k]]} waiting")
        else:
            return


# the kernel's instantiations: 2 X stages, 2 exchange slots, 3 staging buffers up to
# clusters of 8 and 2 beyond; 8 chunks per tile at d = 128, 4 at d = 64
@pytest.mark.parametrize("C,NB,chunks", [(1, 3, 8), (2, 3, 4), (8, 3, 8), (16, 2, 8)])
def test_protocol_random_schedules(C, NB, chunks):
    rnd = random.Random(500 + C)
    for trial in range(40 if C <= 8 else 12):
        run_cluster(random_tiles(rnd), C, 2, 2, seed=trial, NB=NB, chunks=chunks)


def test_model_catches_reordering_across_a_user_boundary():
    rnd = random.Random(9)
    found = 0
    for trial in range(200):
        tiles = random_tiles(rnd)
        try:
            run_cluster(tiles, 4, 2, 2, seed=trial, reorder_across_users=True)
        except Violation:
            found += 1
    assert found > 0


def test_model_catches_pass2_without_tiles_free():
    rnd = random.Random(11)
    found = 0
    for trial in range(200):
        try:
            run_cluster(random_tiles(rnd), 2, 2, 2, seed=trial, tiles_free_wait=False)
        except Violation:
            found += 1
    assert found > 0


def test_model_catches_releasing_staging_before_its_reduction_read_it():
    rnd = random.Random(13)
    found = 0
    for trial in range(150):
        try:
            run_cluster(random_tiles(rnd), 1, 2, 2, seed=trial, NB=3, chunks=8, inflight=3)
        except Violation:
            found += 1
    assert found > 0
