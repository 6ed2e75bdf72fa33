"""Data-parallel sharding of Sketch Attention over GPUs, one process per GPU.

A user's sketch depends on that user's history tokens only (each sketch row is a
mass-weighted mean over the user's own tokens; blog "100,000 videos in your pocket",
section "1. Sketch Attention compresses the history"), and the pages batch users
(R = 40 in training, R = 300 in serving; same blog, section "Training and serving").
So users are the unit of work:

* ``plan_shards`` assigns users to ranks by longest-processing-time first on their
  token counts. A user longer than the per-rank share (or than ``max_part_tokens``)
  is cut into contiguous token ranges, "parts", placed like any other piece.
* ``sharded_forward`` runs the forward on the rank's parts. Users in one piece need no
  communication. For a user cut into parts, the forward's per-prototype sums
  (xsketch = sum_t A_jt X_t and mass_j = sum_t A_jt) add over parts, so one all-reduce
  of k x (d + 1) floats per such user, then ``sa_sketch_combine`` (U Wv / mass),
  finishes it on every rank.
* ``sharded_backward`` runs the backward on the rank's parts with the whole user's
  sketch and mass, the part's own xsketch (dWv is linear in it, so the parts' terms add
  up to the user's), and the whole user's dL/dsketch (all-reduced from its owner for
  cut users). dP, dWk and dWv are then summed over ranks with one all-reduce, as in
  ordinary data parallelism.

Every rank calls the same collectives in the same order: the forward's all-reduce
happens only when the plan cuts some user, on every rank; the backward's first
all-reduce likewise, and its gradient all-reduce whenever world_size > 1.

The per-rank compute defaults to the CUDA library (``binding.forward``,
``binding.backward``, ``binding.combine``); the ``*_fn`` arguments exist so that the
host logic can be exercised on CPU processes.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Callable, Sequence

import numpy as np
import torch
import torch.distributed as dist


@dataclass(frozen=True)
class Part:
    """Tokens [start, stop) of user `user` (positions within that user), run on `rank`."""
    user: int
    start: int
    stop: int
    rank: int

    @property
    def n(self) -> int:
        return self.stop - self.start


@dataclass(frozen=True)
class ShardPlan:
    world_size: int
    lengths: tuple[int, ...]
    parts: tuple[Part, ...]  # ordered by (rank, user, start)

    def parts_of(self, rank: int) -> list[Part]:
        return [p for p in self.parts if p.rank == rank]

    def split_users(self) -> list[int]:
        """Users cut into more than one part (ascending)."""
        count: dict[int, int] = {}
        for p in self.parts:
            count[p.user] = count.get(p.user, 0) + 1
        return sorted(u for u, c in count.items() if c > 1)

    def owner(self, user: int) -> int:
        """The rank that reports the user: the rank of its first part."""
        return min((p for p in self.parts if p.user == user), key=lambda p: p.start).rank

    def owned_users(self, rank: int) -> list[int]:
        return sorted(u for u in range(len(self.lengths)) if self.owner(u) == rank)

    def loads(self) -> list[int]:
        load = [0] * self.world_size
        for p in self.parts:
            load[p.rank] += p.n
        return load

    def local_offsets(self, rank: int) -> np.ndarray:
        """Offsets array of the rank's parts taken as the users of one forward call."""
        sizes = [p.n for p in self.parts_of(rank)]
        return np.concatenate([[0], np.cumsum(sizes, dtype=np.int64)]).astype(np.int64)

    def local_rows(self, rank: int) -> np.ndarray:
        """Row indices, into the global token array, of the rank's tokens in its order."""
        starts = np.concatenate([[0], np.cumsum(self.lengths, dtype=np.int64)])
        rows = [np.arange(starts[p.user] + p.start, starts[p.user] + p.stop, dtype=np.int64)
                for p in self.parts_of(rank)]
        return np.concatenate(rows) if rows else np.zeros(0, dtype=np.int64)


def plan_shards(lengths: Sequence[int], world_size: int,
                max_part_tokens: int | None = None) -> ShardPlan:
    """Longest-processing-time assignment of users (cut where too long) to ranks.

    The part cap is ``max_part_tokens`` or, by default, ceil(total / world_size): a
    user longer than one rank's fair share is cut into ceil(n / cap) near-equal
    contiguous parts. Pieces are placed largest first on the least-loaded rank (lowest
    rank on ties), so no rank exceeds the mean load by more than the largest piece.
    Users with no tokens get one empty part (their outputs are zero). Deterministic.
    """
    if world_size < 1:
        raise ValueError("world_size must be >= 1")
    lengths = tuple(int(n) for n in lengths)
    if any(n < 0 for n in lengths):
        raise ValueError("negative user length")
    total = sum(lengths)
    cap = max_part_tokens if max_part_tokens is not None else max(1, math.ceil(total / world_size))
    if cap < 1:
        raise ValueError("max_part_tokens must be >= 1")
    pieces: list[tuple[int, int, int]] = []  # (user, start, stop)
    for u, n in enumerate(lengths):
        q = max(1, math.ceil(n / cap))
        base, extra = divmod(n, q)
        s = 0
        for i in range(q):
            size = base + (1 if i < extra else 0)
            pieces.append((u, s, s + size))
            s += size
    pieces.sort(key=lambda t: (-(t[2] - t[1]), t[0], t[1]))
    load = [0] * world_size
    parts = []
    for u, s, e in pieces:
        r = min(range(world_size), key=lambda i: (load[i], i))
        load[r] += e - s
        parts.append(Part(u, s, e, r))
    parts.sort(key=lambda p: (p.rank, p.user, p.start))
    return ShardPlan(world_size, lengths, tuple(parts))


def _default(fn, name):
    if fn is not None:
        return fn
    from . import binding  # the CUDA library; raises if it is not built
    return getattr(binding, name)


def sharded_forward(plan: ShardPlan, rank: int, X_local: torch.Tensor, P: torch.Tensor,
                    Wk: torch.Tensor, Wv: torch.Tensor, *, group=None,
                    forward_fn: Callable | None = None,
                    combine_fn: Callable | None = None) -> dict:
    """Forward for this rank's share of the plan.

    X_local: the rank's tokens, its parts concatenated in ``plan.parts_of(rank)`` order
    (``X[plan.local_rows(rank)]``). Returns
      users    global ids of the users this rank reports (its owned users, ascending)
      sketch   [len(users), k, d]; mass [len(users), k]; xsketch [len(users), k, d]
      lse      [n_local] per-token log-sum-exp of the rank's tokens
      part     the forward's raw per-part outputs (kept for the backward)
      split    {user: (sketch, mass)} for every cut user (same on all ranks)
    """
    forward_fn = _default(forward_fn, "forward")
    combine_fn = _default(combine_fn, "combine")
    parts = plan.parts_of(rank)
    k, d = P.shape
    dev = X_local.device
    offs = torch.as_tensor(plan.local_offsets(rank), dtype=torch.int64, device=dev)
    if parts:
        out = forward_fn(X_local, offs, P, Wk, Wv)
    else:  # more ranks than pieces: nothing to run, but still join the collectives
        out = {"sketch": torch.zeros(0, k, d, device=dev), "mass": torch.zeros(0, k, device=dev),
               "xsketch": torch.zeros(0, k, d, device=dev), "lse": torch.zeros(0, device=dev)}
    split = plan.split_users()
    combined: dict[int, tuple] = {}
    if split:
        idx = {u: i for i, u in enumerate(split)}
        buf = torch.zeros(len(split), k * d + k, dtype=out["xsketch"].dtype, device=dev)
        for pi, p in enumerate(parts):
            if p.user in idx:
                buf[idx[p.user], :k * d] += out["xsketch"][pi].reshape(-1)
                buf[idx[p.user], k * d:] += out["mass"][pi]
        if plan.world_size > 1:
            dist.all_reduce(buf, op=dist.ReduceOp.SUM, group=group)
        U = buf[:, :k * d].reshape(len(split), k, d).contiguous()
        M = buf[:, k * d:].contiguous()
        S = combine_fn(U, M, Wv)
        combined = {u: (S[i], M[i], U[i]) for u, i in idx.items()}
    users = plan.owned_users(rank)
    part_of = {p.user: pi for pi, p in enumerate(parts)}
    sk, ms, xs = [], [], []
    for u in users:
        if u in combined:
            s_, m_, x_ = combined[u]
        else:
            pi = part_of[u]
            s_, m_, x_ = out["sketch"][pi], out["mass"][pi], out["xsketch"][pi]
        sk.append(s_)
        ms.append(m_)
        xs.append(x_)

    def stack(v, shape):
        return torch.stack(v) if v else torch.zeros(shape, dtype=torch.float32, device=dev)

    return {"users": users, "sketch": stack(sk, (0, k, d)), "mass": stack(ms, (0, k)),
            "xsketch": stack(xs, (0, k, d)), "lse": out.get("lse"), "part": out,
            "split": {u: (v[0], v[1]) for u, v in combined.items()}}


def sharded_backward(plan: ShardPlan, rank: int, X_local: torch.Tensor, P: torch.Tensor,
                     Wk: torch.Tensor, Wv: torch.Tensor, fwd: dict, dsketch: torch.Tensor,
                     dmass: torch.Tensor | None = None, *, group=None,
                     backward_fn: Callable | None = None) -> dict:
    """Backward for this rank's share. dsketch [len(fwd['users']), k, d] (and optional
    dmass [len(fwd['users']), k]) are dL/dsketch and dL/dmass of the users this rank
    reports. Returns dX for the rank's tokens and dP, dWk, dWv summed over all ranks."""
    backward_fn = _default(backward_fn, "backward")
    parts = plan.parts_of(rank)
    k, d = P.shape
    dev = X_local.device
    pos = {u: i for i, u in enumerate(fwd["users"])}
    split = plan.split_users()
    g_split: dict[int, tuple] = {}
    if split:
        buf = torch.zeros(len(split), k * d + k, dtype=dsketch.dtype, device=dev)
        for i, u in enumerate(split):
            if u in pos:
                buf[i, :k * d] = dsketch[pos[u]].reshape(-1)
                if dmass is not None:
                    buf[i, k * d:] = dmass[pos[u]]
        if plan.world_size > 1:
            dist.all_reduce(buf, op=dist.ReduceOp.SUM, group=group)
        for i, u in enumerate(split):
            g_split[u] = (buf[i, :k * d].reshape(k, d), buf[i, k * d:])
    part = fwd["part"]
    sk, ms, ds, dm = [], [], [], []
    for pi, p in enumerate(parts):
        if p.user in g_split:
            s_, m_ = fwd["split"][p.user]
            g_, gm_ = g_split[p.user]
        else:
            s_, m_ = part["sketch"][pi], part["mass"][pi]
            g_ = dsketch[pos[p.user]]
            gm_ = (dmass[pos[p.user]] if dmass is not None
                   else torch.zeros(k, dtype=dsketch.dtype, device=dev))
        sk.append(s_)
        ms.append(m_)
        ds.append(g_)
        dm.append(gm_)
    n = len(parts)
    f = {"sketch": torch.stack(sk).contiguous() if n else torch.zeros(0, k, d, device=dev),
         "mass": torch.stack(ms).contiguous() if n else torch.zeros(0, k, device=dev),
         "xsketch": part["xsketch"], "lse": part.get("lse")}
    G = torch.stack(ds).contiguous() if n else torch.zeros(0, k, d, device=dev)
    Gm = torch.stack(dm).contiguous() if n else torch.zeros(0, k, device=dev)
    offs = torch.as_tensor(plan.local_offsets(rank), dtype=torch.int64, device=dev)
    if n:
        res = backward_fn(X_local, offs, P, Wk, Wv, f, G, Gm)
    else:
        z = dict(dtype=dsketch.dtype, device=dev)
        res = {"dX": torch.zeros(0, d, **z), "dP": torch.zeros(k, d, **z),
               "dWk": torch.zeros(d, d, **z), "dWv": torch.zeros(d, d, **z)}
    flat = torch.cat([res["dP"].reshape(-1), res["dWk"].reshape(-1), res["dWv"].reshape(-1)])
    flat = flat.contiguous()
    if plan.world_size > 1:
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    dP = flat[:k * d].reshape(k, d)
    dWk = flat[k * d:k * d + d * d].reshape(d, d)
    dWv = flat[k * d + d * d:].reshape(d, d)
    return {"dX": res["dX"], "dP": dP, "dWk": dWk, "dWv": dWv}
