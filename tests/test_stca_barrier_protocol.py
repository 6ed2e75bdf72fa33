"""CPU models of the barrier protocols of the two cross-attention kernels
(csrc/sa_stca_keys.cu: the flash forward; csrc/sa_stca_keys_bwd.cu: the backward), in the
style of the Sketch Attention kernels' models: each role of one CTA runs as a coroutine,
TMA landings and tensor-pipe completions (one in-order pipe) complete in random order, and
barriers follow mbarrier phase and parity semantics, so a wait can pass on a stale phase.

Forward (per candidate tile, nkt key tiles): the producer fills a ring of key stages; the
MMA thread issues Z(j) into score buffer j mod 2 and, once P(j) is stored, O'_(j mod 2) +=
P(j) Kx_j, Z(j + 1) ahead of O'(j); softmax warpgroup w takes the tiles j = w mod 2, reads
Z(j), rescales O'_w when its running maximum rises (after P(j - 2) was read, which also
means O'_w holds every earlier tile of w), stores P(j); at the end warpgroup 1 hands its
state to warpgroup 0, which reads both accumulators. Checked: no deadlock, every MMA reads
the key stage and P of its own tile, no TMA or store overwrites a buffer in use, the
rescale and the final read see O'_w with no MMA pending on it, and O'_w accumulates
exactly the tiles of w.

Backward: the MMA thread issues S(j) after the elementwise step released S(j - 1), dP(j)
after it moved the packed dz / a of tile j - 1 out of the dP columns, then G1 and dKx of
tile j - 1; the elementwise step reads S(j) and dP(j), parks the packed values in the dP
columns, releases S, waits for the previous tile's G1 and dKx MMAs to have read the shared
dz / a tiles, moves the packed values there and releases dP; the epilogue drains dKx(j).
Checked likewise, plus: G1 accumulates every tile once and is read only after the last.
In the forward, one thread's MMAs complete in order and each commit covers every earlier
MMA, so seeing Z(j) already implies that O'(j - 2) has read P(j - 2) and that P(j - 2)
was stored after Z(j - 2) was read: the kernel's explicit waits on the P buffer and on the
score buffer's release are cheap insurance there, and the model shows them redundant.
Planted races (each must be caught): the forward issuing score MMAs two tiles ahead
without the score buffer's release, the forward's merge not waiting for the last
accumulate MMA; the backward's dP issued without the packed values' release, dz / a
stored without the previous MMAs' release, dKx overwritten before the epilogue drained
it.
"""
import heapq
import random

import pytest

from test_fwd_barrier_protocol import Bar, Violation, check


def _engine(rnd):
    events, clock, seq = [], [0], [0]

    def later(fn, lo=1, hi=60):
        seq[0] += 1
        heapq.heappush(events, (clock[0] + rnd.randint(lo, hi), seq[0], fn))

    pipe, busy = [], [False]

    def kick():
        if busy[0] or not pipe:
            return
        start, finish = pipe.pop(0)
        busy[0] = True
        start()

        def done():
            finish()
            busy[0] = False
            kick()
        later(done, 1, 30)

    def issue(start, finish):
        pipe.append((start, finish))
        kick()

    def run(agents):
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
                raise Violation(f"deadlock: agents {[k for k in range(len(agents)) if alive[k]]} waiting")
            else:
                return
    return later, issue, run


def run_forward(nkt, NK, seed, raises=None, z_ahead=1, z_waits=True, final_wait=True):
    """raises[j]: whether warpgroup j mod 2 raises its running maximum at tile j; z_ahead:
    how many score MMAs the MMA thread issues ahead of O'(j) (1 in the kernel)."""
    rnd = random.Random(seed)
    raises = raises or [rnd.random() < 0.4 for _ in range(nkt)]
    later, issue, run = _engine(rnd)
    st = dict(k_full=[Bar(1) for _ in range(NK)], k_empty=[Bar(1) for _ in range(NK)],
              z_full=[Bar(1), Bar(1)], z_empty=[Bar(4), Bar(4)], p_full=[Bar(4), Bar(4)],
              p_empty=[Bar(1), Bar(1)], q_full=Bar(1), merge=Bar(4),
              kst=[None] * NK, kuse=[0] * NK, Z=[None, None], zread=[0, 0],
              P=[None, None], puse=[0, 0], O=[[], []], opend=[0, 0])

    def producer():
        if nkt == 0:  # the kernel's producer and MMA roles do nothing for a user without keys
            return
            yield
        st["q_full"].arrive_expect_tx(1)
        later(lambda: st["q_full"].complete_tx(1))
        for j in range(nkt):
            s = j % NK
            yield lambda: st["k_empty"][s].passes(((j // NK) & 1) ^ 1)
            st["k_full"][s].arrive_expect_tx(1)

            def land(j=j, s=s):
                check(st["kuse"][s] == 0, f"key tile {j} overwrote stage {s} in use")
                st["kst"][s] = j
                st["k_full"][s].complete_tx(1)
            later(land)

    def mma():
        if nkt == 0:
            return
        yield lambda: st["q_full"].passes(0)

        def issue_z(j):
            s, zb = j % NK, j & 1
            yield lambda: st["k_full"][s].passes((j // NK) & 1)
            if z_waits:
                yield lambda: st["z_empty"][zb].passes(((j >> 1) & 1) ^ 1)

            def start(j=j, s=s, zb=zb):
                check(st["kst"][s] == j, f"Z({j}) read key stage holding {st['kst'][s]}")
                check(st["zread"][zb] == 0, f"Z({j}) overwrote score buffer {zb} while read")
                st["kuse"][s] += 1

            def finish(j=j, s=s, zb=zb):
                st["kuse"][s] -= 1
                st["Z"][zb] = j
                st["z_full"][zb].arrive()
            issue(start, finish)

        for j in range(min(z_ahead, nkt)):
            yield from issue_z(j)
        for j in range(nkt):
            if j + z_ahead < nkt:
                yield from issue_z(j + z_ahead)
            s, pb = j % NK, j & 1
            yield lambda: st["p_full"][pb].passes((j >> 1) & 1)
            st["opend"][pb] += 1

            def start(j=j, s=s, pb=pb):
                check(st["kst"][s] == j, f"O'({j}) read key stage holding {st['kst'][s]}")
                check(st["P"][pb] == j, f"O'({j}) read P buffer holding {st['P'][pb]}")
                st["kuse"][s] += 1
                st["puse"][pb] += 1

            def finish(j=j, s=s, pb=pb):
                st["kuse"][s] -= 1
                st["puse"][pb] -= 1
                st["O"][pb].append(j)
                st["opend"][pb] -= 1
                st["k_empty"][s].arrive()
                st["p_empty"][pb].arrive()
            issue(start, finish)

    def softmax(w):
        last = -1
        for j in range(w, nkt, 2):
            yield lambda: st["z_full"][w].passes((j >> 1) & 1)
            check(st["Z"][w] == j, f"softmax of tile {j} read score buffer holding {st['Z'][w]}")
            st["zread"][w] += 1
            yield None  # the row maximum of the tile
            yield lambda: st["p_empty"][w].passes(((j >> 1) & 1) ^ 1)
            if raises[j] and j >= 2:
                check(st["opend"][w] == 0, f"rescale at tile {j} while O'_{w} has an MMA pending")
                check(st["O"][w] == list(range(w, j, 2)), f"rescale at tile {j}: O'_{w} holds {st['O'][w]}")
            check(st["puse"][w] == 0, f"P({j}) stored while an MMA reads P buffer {w}")
            st["P"][w] = j
            st["zread"][w] -= 1
            st["z_empty"][w].arrive(4)
            st["p_full"][w].arrive(4)
            last = j
        if last >= 0 and final_wait:
            yield lambda: st["p_empty"][w].passes((last >> 1) & 1)
        if w == 1:
            st["merge"].arrive(4)
        else:
            yield lambda: st["merge"].passes(0)
            for v in (0, 1):
                check(st["opend"][v] == 0, f"merge read O'_{v} with an MMA pending")
                check(st["O"][v] == list(range(v, nkt, 2)), f"merge read O'_{v} holding {st['O'][v]}")

    run([producer(), mma(), softmax(0), softmax(1)])


@pytest.mark.parametrize("NK", [2, 3])
def test_forward_protocol_random_schedules(NK):
    rnd = random.Random(700 + NK)
    for trial in range(120):
        run_forward(rnd.randint(0, 12), NK, seed=trial)


def test_forward_model_catches_score_mmas_two_ahead_without_the_buffer_release():
    found = 0
    for trial in range(200):
        try:
            run_forward(8, 3, seed=trial, z_ahead=2, z_waits=False)
        except Violation:
            found += 1
    assert found > 0


def test_forward_model_catches_a_merge_before_the_last_accumulate():
    found = 0
    for trial in range(200):
        try:
            run_forward(7, 3, seed=trial, final_wait=False)
        except Violation:
            found += 1
    assert found > 0


def run_backward(nkt, NK, seed, p_waits=True, ew_waits=True, dk_waits=True):
    rnd = random.Random(seed)
    later, issue, run = _engine(rnd)
    st = dict(k_full=[Bar(1) for _ in range(NK)], k_empty=[Bar(1) for _ in range(NK)],
              q_full=Bar(1), sd_full=Bar(1), s_empty=Bar(8), p_empty=Bar(8), ew_full=Bar(8),
              ew_empty=Bar(1), dk_full=Bar(1), dk_empty=Bar(4),
              kst=[None] * NK, kuse=[0] * NK, S=None, sread=0, dP=None, packed=[None, None],
              dz=None, dzuse=0, G1=[], g1pend=0, dK=None, dkread=False, dk_drained=[])

    def producer():
        if nkt == 0:  # the kernel's producer and MMA roles do nothing for a user without keys
            return
            yield
        st["q_full"].arrive_expect_tx(1)
        later(lambda: st["q_full"].complete_tx(1))
        for j in range(nkt):
            s = j % NK
            yield lambda: st["k_empty"][s].passes(((j // NK) & 1) ^ 1)
            st["k_full"][s].arrive_expect_tx(1)

            def land(j=j, s=s):
                check(st["kuse"][s] == 0, f"key tile {j} overwrote stage {s} in use")
                st["kst"][s] = j
                st["k_full"][s].complete_tx(1)
            later(land)

    def mma():
        if nkt == 0:
            return
        yield lambda: st["q_full"].passes(0)

        def back(i):
            s = i % NK
            yield lambda: st["ew_full"].passes(i & 1)
            st["g1pend"] += 1

            def g_start(i=i, s=s):
                check(st["dz"] == i, f"G1({i}) read dz holding {st['dz']}")
                check(st["kst"][s] == i, f"G1({i}) read key stage holding {st['kst'][s]}")
                st["dzuse"] += 1
                st["kuse"][s] += 1

            def g_finish(i=i, s=s):
                st["dzuse"] -= 1
                st["kuse"][s] -= 1
                st["G1"].append(i)
                st["g1pend"] -= 1
                st["k_empty"][s].arrive()
            issue(g_start, g_finish)
            if dk_waits:
                yield lambda: st["dk_empty"].passes((i & 1) ^ 1)

            def k_start(i=i):
                check(st["dz"] == i, f"dKx({i}) read dz / a holding {st['dz']}")
                check(not st["dkread"], f"dKx({i}) overwrote dKx of tile {st['dK']} while drained")
                check(st["dK"] is None or st["dK"] in st["dk_drained"],
                      f"dKx({i}) overwrote dKx of tile {st['dK']} before it was drained")
                st["dzuse"] += 1

            def k_finish(i=i):
                st["dzuse"] -= 1
                st["dK"] = i
                st["dk_full"].arrive()
                st["ew_empty"].arrive()
            issue(k_start, k_finish)

        for j in range(nkt):
            s = j % NK
            yield lambda: st["k_full"][s].passes((j // NK) & 1)
            if j > 0:
                yield lambda: st["s_empty"].passes((j - 1) & 1)

            def s_start(j=j, s=s):
                check(st["kst"][s] == j, f"S({j}) read key stage holding {st['kst'][s]}")
                check(st["sread"] == 0, f"S({j}) overwrote S of tile {st['S']} while read")
                st["kuse"][s] += 1

            def s_finish(j=j, s=s):
                st["kuse"][s] -= 1
                st["S"] = j
            issue(s_start, s_finish)
            if j > 0 and p_waits:
                yield lambda: st["p_empty"].passes((j - 1) & 1)

            def p_start(j=j, s=s):
                check(st["kst"][s] == j, f"dP({j}) read key stage holding {st['kst'][s]}")
                check(st["packed"] == [None, None], f"dP({j}) overwrote the parked dz / a {st['packed']}")
                st["kuse"][s] += 1

            def p_finish(j=j, s=s):
                st["kuse"][s] -= 1
                st["dP"] = j
                st["sd_full"].arrive()
            issue(p_start, p_finish)
            if j > 0:
                yield from back(j - 1)
        if nkt > 0:
            yield from back(nkt - 1)

    def elementwise(w):
        for j in range(nkt):
            yield lambda: st["sd_full"].passes(j & 1)
            check(st["S"] == j and st["dP"] == j, f"elementwise {j} read S {st['S']} / dP {st['dP']}")
            st["packed"][w] = j  # this warpgroup's half, parked in the dP columns it read
            st["s_empty"].arrive(4)
            if ew_waits:
                yield lambda: st["ew_empty"].passes((j & 1) ^ 1)
            check(st["packed"][w] == j, f"elementwise {j}: parked values replaced by {st['packed'][w]}")
            check(st["dzuse"] == 0, f"dz / a of tile {j} stored while an MMA reads them")
            st["dz"] = j
            yield None
            st["packed"][w] = None
            st["p_empty"].arrive(4)
            st["ew_full"].arrive(4)
        if nkt > 0:
            yield lambda: st["ew_empty"].passes((nkt - 1) & 1)
            check(st["g1pend"] == 0 and st["G1"] == list(range(nkt)), f"G1 read holding {st['G1']}")

    def epilogue():
        for j in range(nkt):
            yield lambda: st["dk_full"].passes(j & 1)
            check(st["dK"] == j, f"epilogue {j} read dKx of tile {st['dK']}")
            st["dkread"] = True
            yield None
            st["dkread"] = False
            st["dk_drained"].append(j)
            st["dk_empty"].arrive(4)

    run([producer(), mma(), elementwise(0), elementwise(1), epilogue()])


@pytest.mark.parametrize("NK", [2, 3])
def test_backward_protocol_random_schedules(NK):
    rnd = random.Random(800 + NK)
    for trial in range(120):
        run_backward(rnd.randint(0, 12), NK, seed=trial)


@pytest.mark.parametrize("planted", ["p_waits", "ew_waits", "dk_waits"])
def test_backward_model_catches_planted_races(planted):
    found = 0
    for trial in range(200):
        try:
            run_backward(8, 2, seed=trial, **{planted: False})
        except Violation:
            found += 1
    assert found > 0, planted
