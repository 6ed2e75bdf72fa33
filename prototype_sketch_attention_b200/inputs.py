"""Seeded synthetic inputs shaped like the pages' workloads.

This module only draws random numbers; it holds none of Sketch Attention's
arithmetic. Both the CUDA path and the fp64 oracle are fed from it.

The paper's Douyin histories are proprietary; these stand in for them with the
shapes the pages give: histories up to 100K interactions, k from several hundred
to several thousand prototypes, the deployed 1K x 128 sketch, and user-level
batches of R=40 (training) and R=300 (serving) (evolve.pub review "Summary";
blog "1. Sketch Attention compresses the history" and "3. The system makes it
cheap enough to matter").

Recipe: one CPU ``torch.Generator`` seeded with ``1000 + config``; draw order is
lengths, X, P, W_k, W_v, G. X ~ N(0,1) item embeddings, P ~ N(0,1),
W_k, W_v ~ N(0, 1/d), G ~ N(0,1). bf16 values are fp32 draws rounded to nearest
even; the oracle widens exactly those bf16 values to fp64.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

# The five workloads: (R, d, k, dtype, length rule, backward).
CONFIGS = {
    1: dict(R=1, d=64, k=64, dtype="f32", lengths="fixed:2048", backward=False,
            desc="1 user, n=2048, d=64, k=64, fp32, forward"),
    2: dict(R=1, d=128, k=1024, dtype="bf16", lengths="fixed:100000", backward=False,
            desc="1 user, n=100000, d=128, k=1024, bf16, forward"),
    3: dict(R=40, d=128, k=1024, dtype="bf16", lengths="uniform:10000:100000", backward=False,
            desc="R=40 users, n~U[10000,100000], d=128, k=1024, bf16, forward"),
    4: dict(R=300, d=128, k=1024, dtype="bf16", lengths="loguniform:1000:100000", backward=False,
            desc="R=300 users, n~logU[1000,100000], d=128, k in {256,512,1024,2048}, bf16, forward"),
    5: dict(R=40, d=128, k=1024, dtype="bf16", lengths="fixed:100000", backward=True,
            desc="R=40 users x n=100000, d=128, k=1024, bf16, forward+backward"),
}


@dataclass
class Workload:
    name: str
    R: int
    d: int
    k: int
    dtype: str                 # "f32" or "bf16"
    lengths: np.ndarray        # int64 [R]
    offsets: torch.Tensor      # int64 [R+1], CPU
    X: torch.Tensor            # [n_total, d] CPU, dtype per `dtype`
    P: torch.Tensor            # [k, d]
    Wk: torch.Tensor           # [d, d]
    Wv: torch.Tensor           # [d, d]
    G: torch.Tensor | None = None   # [R, k, d] fp32 upstream gradient
    meta: dict = field(default_factory=dict)

    @property
    def n_total(self) -> int:
        return int(self.offsets[-1])

    def to_f64(self, users=None) -> dict:
        """fp64 numpy copies of exactly the values the GPU sees (optionally a user subset)."""
        if users is None:
            users = range(self.R)
        users = list(users)
        off = self.offsets.numpy()
        rows = [np.arange(off[u], off[u + 1]) for u in users]
        idx = np.concatenate(rows) if rows else np.zeros(0, dtype=np.int64)
        lens = np.array([off[u + 1] - off[u] for u in users], dtype=np.int64)
        sub_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
        X = self.X[torch.from_numpy(idx)].double().numpy() if len(idx) else np.zeros((0, self.d))
        out = dict(X=X, offsets=sub_off, P=self.P.double().numpy(), Wk=self.Wk.double().numpy(),
                   Wv=self.Wv.double().numpy(), rows=idx)
        if self.G is not None:
            out["G"] = self.G[users].double().numpy()
        return out


def _torch_dtype(dtype: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]


def draw_lengths(rule: str, R: int, gen: torch.Generator) -> np.ndarray:
    kind, *args = rule.split(":")
    if kind == "fixed":
        return np.full(R, int(args[0]), dtype=np.int64)
    if kind == "uniform":
        lo, hi = int(args[0]), int(args[1])
        return torch.randint(lo, hi + 1, (R,), generator=gen).numpy().astype(np.int64)
    if kind == "loguniform":
        lo, hi = math.log(float(args[0])), math.log(float(args[1]))
        u = torch.rand(R, generator=gen, dtype=torch.float64)
        return torch.round(torch.exp(lo + (hi - lo) * u)).numpy().astype(np.int64)
    raise ValueError(f"unknown length rule {rule!r}")


def make_workload(lengths, d: int, k: int, dtype: str, seed: int, with_grad: bool = False,
                  name: str = "custom", x_std: float = 1.0, p_std: float = 1.0,
                  w_std: float | None = None, gen: torch.Generator | None = None) -> Workload:
    """Draw X, P, W_k, W_v (and G) for the given per-user lengths."""
    if gen is None:
        gen = torch.Generator().manual_seed(seed)
    lengths = np.asarray(lengths, dtype=np.int64)
    R = len(lengths)
    offsets = torch.from_numpy(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64))
    n_total = int(offsets[-1])
    td = _torch_dtype(dtype)
    w_std = (1.0 / math.sqrt(d)) if w_std is None else w_std
    X = (torch.randn(n_total, d, generator=gen) * x_std).to(td)
    P = (torch.randn(k, d, generator=gen) * p_std).to(td)
    Wk = (torch.randn(d, d, generator=gen) * w_std).to(td)
    Wv = (torch.randn(d, d, generator=gen) * w_std).to(td)
    G = torch.randn(R, k, d, generator=gen) if with_grad else None
    return Workload(name=name, R=R, d=d, k=k, dtype=dtype, lengths=lengths, offsets=offsets,
                    X=X, P=P, Wk=Wk, Wv=Wv, G=G, meta=dict(seed=seed))


def make_config(idx: int, k: int | None = None, with_grad: bool | None = None) -> Workload:
    """The numbered workload, drawn from seed 1000 + idx (k overrides config 4's sweep)."""
    c = CONFIGS[idx]
    kk = c["k"] if k is None else int(k)
    gen = torch.Generator().manual_seed(1000 + idx)
    lengths = draw_lengths(c["lengths"], c["R"], gen)
    wg = c["backward"] if with_grad is None else with_grad
    name = f"config{idx}" + (f"_k{kk}" if k is not None else "")
    w = make_workload(lengths, c["d"], kk, c["dtype"], seed=1000 + idx, with_grad=wg,
                      name=name, gen=gen)
    w.meta["desc"] = c["desc"]
    return w


@dataclass
class CrossWorkload:
    """Inputs of the candidate-to-sketch cross attention (CPU tensors)."""
    R: int
    k: int
    d: int
    counts: np.ndarray          # candidates per user
    cand_offsets: torch.Tensor  # int64 [R+1]
    Q: torch.Tensor             # bf16 [n_cand, d]
    S: torch.Tensor             # fp32 [R, k, d]
    Wq: torch.Tensor            # bf16 [d, d]
    WK: torch.Tensor
    WV: torch.Tensor

    def to_f64(self) -> dict:
        return dict(Q=self.Q.double().numpy(), cand_offsets=self.cand_offsets.numpy(),
                    S=self.S.double().numpy(), Wq=self.Wq.double().numpy(),
                    WK=self.WK.double().numpy(), WV=self.WV.double().numpy())


def make_cross_workload(counts, k: int, d: int, seed: int, s_std: float = 1.0,
                        S: torch.Tensor | None = None) -> CrossWorkload:
    """Draw candidates Q ~ N(0, 1) (bf16), weights ~ N(0, 1/d) (bf16) and, unless given,
    sketches S ~ N(0, s_std^2) (fp32) for the given candidate counts per user."""
    gen = torch.Generator().manual_seed(seed)
    counts = np.asarray(counts, dtype=np.int64)
    R = len(counts)
    off = torch.from_numpy(np.concatenate([[0], np.cumsum(counts)]).astype(np.int64))
    n = int(off[-1])
    Q = torch.randn(n, d, generator=gen).to(torch.bfloat16)
    Wq, WK, WV = ((torch.randn(d, d, generator=gen) / math.sqrt(d)).to(torch.bfloat16)
                  for _ in range(3))
    if S is None:
        S = torch.randn(R, k, d, generator=gen) * s_std
    return CrossWorkload(R=R, k=k, d=d, counts=counts, cand_offsets=off, Q=Q, S=S.float(),
                         Wq=Wq, WK=WK, WV=WV)


@dataclass
class RecentWorkload:
    """Inputs of the recent branch: candidates attending over each user's last L history
    rows (CPU tensors)."""
    R: int
    d: int
    L: int
    lengths: np.ndarray         # history rows per user
    offsets: torch.Tensor       # int64 [R+1], the history layout
    X: torch.Tensor             # bf16 [n_total, d], the history (the keys, read in place)
    counts: np.ndarray          # candidates per user
    cand_offsets: torch.Tensor  # int64 [R+1]
    Q: torch.Tensor             # bf16 [n_cand, d]
    Wq: torch.Tensor            # bf16 [d, d]
    WK: torch.Tensor
    WV: torch.Tensor

    def suffix_rows(self) -> np.ndarray:
        """History row indices of every user's last min(n_u, L) rows, users in order."""
        off = self.offsets.numpy()
        rows = [np.arange(max(off[u], off[u + 1] - self.L), off[u + 1]) for u in range(self.R)]
        return np.concatenate(rows).astype(np.int64) if rows else np.zeros(0, dtype=np.int64)


def make_recent_workload(lengths, counts, d: int, L: int, seed: int,
                         q_std: float = 1.0) -> RecentWorkload:
    """Draw the history X ~ N(0, 1), candidates Q ~ N(0, q_std^2) and Wq, WK, WV ~ N(0, 1/d),
    all bf16, in that order, for the given history lengths and candidate counts per user."""
    gen = torch.Generator().manual_seed(seed)
    lengths = np.asarray(lengths, dtype=np.int64)
    counts = np.asarray(counts, dtype=np.int64)
    assert len(lengths) == len(counts)
    R = len(lengths)
    off = torch.from_numpy(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64))
    coff = torch.from_numpy(np.concatenate([[0], np.cumsum(counts)]).astype(np.int64))
    X = torch.randn(int(off[-1]), d, generator=gen).to(torch.bfloat16)
    Q = (torch.randn(int(coff[-1]), d, generator=gen) * q_std).to(torch.bfloat16)
    Wq, WK, WV = ((torch.randn(d, d, generator=gen) / math.sqrt(d)).to(torch.bfloat16)
                  for _ in range(3))
    return RecentWorkload(R=R, d=d, L=int(L), lengths=lengths, offsets=off, X=X, counts=counts,
                          cand_offsets=coff, Q=Q, Wq=Wq, WK=WK, WV=WV)
