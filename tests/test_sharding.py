"""Multi-GPU sharding, host side: the user planner, and world_size-2 gloo runs of the
sharded forward and backward with the fp64 oracle standing in for each rank's GPU.

The sharded result must equal the oracle on the whole batch: a cut user's parts add
up (xsketch and mass are sums over tokens) and the gradients of dP, dW_k, dW_v add
over ranks."""
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from prototype_sketch_attention_b200 import inputs
from prototype_sketch_attention_b200.sharding import plan_shards, sharded_backward, sharded_forward


# ---------------------------------------------------------------- planner
@pytest.mark.parametrize("lengths,world,cap", [
    ([100000], 2, None), ([5, 0, 7], 4, None), ([37, 0, 260, 91], 2, 100),
    (list(np.random.default_rng(0).integers(10000, 100001, 40)), 8, None),
    (list(np.random.default_rng(1).integers(1, 5000, 300)), 3, None), ([3, 4], 5, None)])
def test_plan_covers_every_token_once(lengths, world, cap):
    plan = plan_shards(lengths, world, cap)
    for u, n in enumerate(lengths):
        ps = sorted((p for p in plan.parts if p.user == u), key=lambda p: p.start)
        assert ps, f"user {u} has no part"
        assert ps[0].start == 0 and ps[-1].stop == n
        for a, b in zip(ps, ps[1:]):
            assert a.stop == b.start
        if n > 0:
            assert all(p.n > 0 for p in ps)
    rows = np.concatenate([plan.local_rows(r) for r in range(world)])
    assert np.array_equal(np.sort(rows), np.arange(sum(lengths)))
    assert sum(plan.loads()) == sum(lengths)
    assert all(plan.owner(u) in range(world) for u in range(len(lengths)))
    assert sorted(sum((plan.owned_users(r) for r in range(world)), [])) == list(range(len(lengths)))


def test_plan_cap_and_balance():
    rng = np.random.default_rng(2)
    lengths = list(rng.integers(1, 100000, 57)) + [900000]
    world = 8
    plan = plan_shards(lengths, world)
    cap = -(-sum(lengths) // world)
    assert max(p.n for p in plan.parts) <= cap
    # LPT: the most loaded rank exceeds the mean by at most the largest piece
    assert max(plan.loads()) <= sum(lengths) / world + max(p.n for p in plan.parts)
    assert plan.split_users() == [len(lengths) - 1]
    assert plan == plan_shards(lengths, world)  # deterministic


def test_plan_rejects_bad_arguments():
    with pytest.raises(ValueError):
        plan_shards([1, 2], 0)
    with pytest.raises(ValueError):
        plan_shards([1, -2], 2)
    with pytest.raises(ValueError):
        plan_shards([1, 2], 2, max_part_tokens=0)


# ---------------------------------------------------------------- gloo runs
def _oracle_forward(X, offs, P, Wk, Wv):
    r = oracle.forward(X.numpy(), offs.numpy(), P.numpy(), Wk.numpy(), Wv.numpy(), nthreads=1)
    return {k: torch.from_numpy(v) for k, v in r.items()}


def _combine(U, M, Wv):
    # sketch = (U Wv) / mass, mass = 0 -> 0 (the sketch's definition; test-side helper)
    S = torch.einsum("rkc,ce->rke", U, Wv)
    inv = torch.where(M > 0, 1.0 / torch.where(M > 0, M, torch.ones_like(M)), torch.zeros_like(M))
    return S * inv[..., None]


def _oracle_backward(X, offs, P, Wk, Wv, fwd, G, Gm):
    r = oracle.backward(X.numpy(), offs.numpy(), P.numpy(), Wk.numpy(), Wv.numpy(), G.numpy(),
                        Gm.numpy(), nthreads=1)
    return {k: torch.from_numpy(v) for k, v in r.items()}


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _workload(case):
    lengths, k, d, cap = case
    w = inputs.make_workload(lengths, d, k, "f32", seed=321, with_grad=True)
    return w, w.to_f64()


def _worker(rank, world, port, case, outdir, mode):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        w, f = _workload(case)
        plan = plan_shards(case[0], world, case[3])
        t = {n: torch.from_numpy(np.ascontiguousarray(f[n])) for n in ("X", "P", "Wk", "Wv")}
        Xl = t["X"][torch.from_numpy(plan.local_rows(rank))].contiguous()
        fwd = sharded_forward(plan, rank, Xl, t["P"], t["Wk"], t["Wv"],
                              forward_fn=_oracle_forward, combine_fn=_combine)
        res = {"users": np.array(fwd["users"], dtype=np.int64), "sketch": fwd["sketch"].numpy(),
               "mass": fwd["mass"].numpy(), "xsketch": fwd["xsketch"].numpy(),
               "lse": fwd["lse"].numpy(), "rows": plan.local_rows(rank)}
        G = torch.from_numpy(w.G.numpy().astype(np.float64))
        Gm = torch.from_numpy(np.random.default_rng(9).standard_normal((len(plan.lengths), case[1])))
        own = torch.tensor(fwd["users"], dtype=torch.int64)
        if mode == "grad":
            b = sharded_backward(plan, rank, Xl, t["P"], t["Wk"], t["Wv"], fwd, G[own], Gm[own],
                                 backward_fn=_oracle_backward)
            res.update({n: b[n].numpy() for n in ("dX", "dP", "dWk", "dWv")})
        elif mode == "plumbing":
            seen = {}

            def fake_backward(X, offs, P, Wk, Wv, f_, G_, Gm_):
                seen.update(sketch=f_["sketch"].numpy(), mass=f_["mass"].numpy(),
                            xsketch=f_["xsketch"].numpy(), G=G_.numpy(), Gm=Gm_.numpy())
                k_, d_ = P.shape
                return {"dX": torch.zeros(X.shape[0], d_, dtype=torch.float64),
                        "dP": torch.full((k_, d_), rank + 1.0, dtype=torch.float64),
                        "dWk": torch.full((d_, d_), 10.0 * (rank + 1), dtype=torch.float64),
                        "dWv": torch.zeros(d_, d_, dtype=torch.float64)}
            b = sharded_backward(plan, rank, Xl, t["P"], t["Wk"], t["Wv"], fwd, G[own], Gm[own],
                                 backward_fn=fake_backward)
            res.update({"seen_" + n: v for n, v in seen.items()})
            res.update({n: b[n].numpy() for n in ("dP", "dWk")})
            res["part_users"] = np.array([p.user for p in plan.parts_of(rank)], dtype=np.int64)
            res["part_xsketch"] = fwd["part"]["xsketch"].numpy()
        np.savez(os.path.join(outdir, f"rank{rank}.npz"), **res)
    finally:
        dist.destroy_process_group()


def _run(case, mode, world=2):
    with tempfile.TemporaryDirectory() as outdir:
        mp.spawn(_worker, args=(world, _free_port(), case, outdir, mode), nprocs=world, join=True)
        return [dict(np.load(os.path.join(outdir, f"rank{r}.npz"))) for r in range(world)]


CUT = ([37, 0, 260, 91, 5], 6, 8, 100)     # user 2 is cut into three parts
WHOLE = ([37, 0, 160, 91, 5], 6, 8, 1000)  # no user is cut


@pytest.mark.parametrize("case", [CUT, WHOLE])
def test_sharded_forward_matches_whole_batch(case):
    outs = _run(case, "fwd")
    w, f = _workload(case)
    ref = oracle.forward(f["X"], f["offsets"], f["P"], f["Wk"], f["Wv"], nthreads=1)
    seen = []
    for o in outs:
        for i, u in enumerate(o["users"]):
            seen.append(u)
            for n in ("sketch", "mass", "xsketch"):
                np.testing.assert_allclose(o[n][i], ref[n][u], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(o["lse"], ref["lse"][o["rows"]], rtol=1e-12, atol=1e-12)
    assert sorted(seen) == list(range(len(case[0])))


def test_sharded_backward_matches_whole_batch():
    outs = _run(WHOLE, "grad")
    w, f = _workload(WHOLE)
    G = w.G.numpy().astype(np.float64)
    Gm = np.random.default_rng(9).standard_normal((len(WHOLE[0]), WHOLE[1]))
    ref = oracle.backward(f["X"], f["offsets"], f["P"], f["Wk"], f["Wv"], G, Gm, nthreads=1)
    for o in outs:
        for n in ("dP", "dWk", "dWv"):  # all-reduced: the whole batch's sums on every rank
            np.testing.assert_allclose(o[n], ref[n], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(o["dX"], ref["dX"][o["rows"]], rtol=1e-10, atol=1e-12)


def test_sharded_backward_feeds_cut_users_whole_statistics():
    outs = _run(CUT, "plumbing")
    w, f = _workload(CUT)
    ref = oracle.forward(f["X"], f["offsets"], f["P"], f["Wk"], f["Wv"], nthreads=1)
    G = w.G.numpy().astype(np.float64)
    Gm = np.random.default_rng(9).standard_normal((len(CUT[0]), CUT[1]))
    for o in outs:
        for i, u in enumerate(o["part_users"]):
            # the whole user's sketch, mass and gradients, but the part's own xsketch
            np.testing.assert_allclose(o["seen_sketch"][i], ref["sketch"][u], rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(o["seen_mass"][i], ref["mass"][u], rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(o["seen_G"][i], G[u], rtol=0, atol=0)
            np.testing.assert_allclose(o["seen_Gm"][i], Gm[u], rtol=0, atol=0)
            np.testing.assert_array_equal(o["seen_xsketch"][i], o["part_xsketch"][i])
        np.testing.assert_allclose(o["dP"], 3.0)    # 1 + 2 over the two ranks
        np.testing.assert_allclose(o["dWk"], 30.0)
    # the parts' own xsketch add up to the user's
    tot = sum(o["part_xsketch"][o["part_users"] == 2].sum(0) for o in outs)
    np.testing.assert_allclose(tot, ref["xsketch"][2], rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- failure detection
def _absent_rank_worker(rank, world, port, outdir):
    """Rank 1 fails before the forward (it never joins the cut user's all-reduce); rank 0
    must leave the collective with an error once the process group's timeout runs out,
    instead of waiting for ever. Rank 1 stays alive (holding its connection) until rank 0
    has reported, so the error rank 0 sees is the timeout, not a closed socket."""
    import datetime
    import time
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=3))
    flag = os.path.join(outdir, "rank0_done")
    try:
        if rank == 1:
            deadline = time.monotonic() + 60.0
            while not os.path.exists(flag) and time.monotonic() < deadline:
                time.sleep(0.05)
            return
        w, f = _workload(CUT)
        plan = plan_shards(CUT[0], world, CUT[3])
        t = {n: torch.from_numpy(np.ascontiguousarray(f[n])) for n in ("X", "P", "Wk", "Wv")}
        Xl = t["X"][torch.from_numpy(plan.local_rows(rank))].contiguous()
        t0 = time.monotonic()
        try:
            sharded_forward(plan, rank, Xl, t["P"], t["Wk"], t["Wv"],
                            forward_fn=_oracle_forward, combine_fn=_combine)
            status = "no error"
        except RuntimeError as e:
            status = "error: " + str(e)[:200]
        with open(os.path.join(outdir, "rank0.txt"), "w") as fh:
            fh.write(f"{time.monotonic() - t0:.3f}\n{status}\n")
        open(flag, "w").close()
    finally:
        dist.destroy_process_group()


def test_absent_rank_ends_the_collective_with_an_error():
    assert plan_shards(CUT[0], 2, CUT[3]).split_users(), "the case must need an all-reduce"
    with tempfile.TemporaryDirectory() as outdir:
        mp.spawn(_absent_rank_worker, args=(2, _free_port(), outdir), nprocs=2, join=True)
        secs, status = open(os.path.join(outdir, "rank0.txt")).read().splitlines()[:2]
    assert status.startswith("error"), status
    assert float(secs) < 30.0, secs
