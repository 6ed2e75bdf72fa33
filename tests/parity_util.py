"""Helpers for GPU-vs-oracle parity tests.

Tolerances (written here once, used by every parity test):
  fp32 path:  relative L2 <= 1e-5 on sketch, mass, xsketch and lse (forward) and on the
              backward's gradients, as the stated fp32 tolerance.
  bf16 path:  per user, relative L2 <= 1e-2 and max |error| <= 5e-2 on the sketch (its
              values are O(1)); per user, relative L2 <= 1e-2 on mass and xsketch, with
              max |error| <= 5e-2 * max |reference| (they are sums over the user's n
              tokens, so an absolute bound would tighten with n); max |error| <= 5e-2 on
              lse. Gradients: dX per user relative L2 <= 1e-2 and max |error|
              <= 5e-2 * max(1, max |reference of that user|) (absolute for O(1) entries;
              a user with few tokens has a small mass and gradients far above 1); dP,
              dW_k, dW_v (sums over every user's tokens) relative L2 <= 1e-2 and
              max |error| <= 5e-2 * max |reference|.
"""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle

FP32_FWD = 1e-5
FP32_BWD = 1e-5
BF16_REL = 1e-2
BF16_ABS = 5e-2


def rel_l2(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(got - ref)
    if den == 0.0:
        return float(num)
    return float(num / den)


def nthreads() -> int:
    return os.cpu_count() or 1


def to_gpu(w, device="cuda"):
    g = {"X": w.X.to(device), "offsets": w.offsets.to(device), "P": w.P.to(device),
         "Wk": w.Wk.to(device), "Wv": w.Wv.to(device)}
    if w.G is not None:
        g["G"] = w.G.to(device)
    return g


def gpu_forward(w, device="cuda"):
    from prototype_sketch_attention_b200 import binding
    g = to_gpu(w, device)
    out = binding.forward(g["X"], g["offsets"], g["P"], g["Wk"], g["Wv"])
    st = binding.device_status(out["_ws"])
    assert st == 0, binding.sa_status_string(st)
    return g, out


def check_forward(w, out, users=None):
    """Compares the GPU forward with the oracle on the given users (default: all)."""
    users = list(range(w.R)) if users is None else list(users)
    sub = w.to_f64(users)
    ref = oracle.forward(sub["X"], sub["offsets"], sub["P"], sub["Wk"], sub["Wv"],
                         nthreads=nthreads())
    sk = out["sketch"].cpu().double().numpy()[users]
    ms = out["mass"].cpu().double().numpy()[users]
    xs = out["xsketch"].cpu().double().numpy()[users] if "xsketch" in out else None
    lse = out["lse"].cpu().double().numpy()[sub["rows"]] if "lse" in out else None
    fp32 = w.dtype == "f32"
    for i, u in enumerate(users):
        n_u = sub["offsets"][i + 1] - sub["offsets"][i]
        if n_u == 0:
            assert not sk[i].any() and not ms[i].any(), f"user {u}: empty user must give zeros"
            continue
        e_s = rel_l2(sk[i], ref["sketch"][i])
        e_m = rel_l2(ms[i], ref["mass"][i])
        if fp32:
            assert e_s <= FP32_FWD, (u, "sketch", e_s)
            assert e_m <= FP32_FWD, (u, "mass", e_m)
        else:
            assert e_s <= BF16_REL, (u, "sketch", e_s)
            assert np.abs(sk[i] - ref["sketch"][i]).max() <= BF16_ABS, (u, "sketch max-abs")
            assert e_m <= BF16_REL, (u, "mass", e_m)
            # mass and xsketch are sums over the user's tokens: their max-abs bound scales
            # with the user's largest entry, as for the gradients
            assert np.abs(ms[i] - ref["mass"][i]).max() <= BF16_ABS * np.abs(ref["mass"][i]).max(), \
                (u, "mass max-abs")
        if xs is not None:
            e_x = rel_l2(xs[i], ref["xsketch"][i])
            assert e_x <= (FP32_FWD if fp32 else BF16_REL), (u, "xsketch", e_x)
            if not fp32:
                assert (np.abs(xs[i] - ref["xsketch"][i]).max()
                        <= BF16_ABS * np.abs(ref["xsketch"][i]).max()), (u, "xsketch max-abs")
    if lse is not None and len(lse):
        if fp32:
            assert rel_l2(lse, ref["lse"]) <= FP32_FWD, ("lse", rel_l2(lse, ref["lse"]))
        else:
            assert np.abs(lse - ref["lse"]).max() <= BF16_ABS, ("lse", np.abs(lse - ref["lse"]).max())
    return ref


def check_grads(got: dict, ref: dict, fp32: bool, keys=("dX", "dP", "dWk", "dWv"),
                offsets=None):
    """offsets (host int64 [R + 1], the rows of dX): dX is also checked user by user."""
    for key in keys:
        g = got[key]
        r = ref[key]
        e = rel_l2(g, r)
        if fp32:
            assert e <= FP32_BWD, (key, e)
        else:
            assert e <= BF16_REL, (key, e)
            scale = max(np.abs(r).max(), 1e-30)
            assert np.abs(g - r).max() <= BF16_ABS * scale, (key, "max-abs")
    if "dX" in keys and offsets is not None:
        off = np.asarray(offsets)
        for u in range(len(off) - 1):
            a, b = int(off[u]), int(off[u + 1])
            if a == b:
                continue
            gu, ru = got["dX"][a:b], ref["dX"][a:b]
            e = rel_l2(gu, ru)
            if fp32:
                assert e <= FP32_BWD, (u, "dX", e)
            else:
                assert e <= BF16_REL, (u, "dX", e)
                bound = BF16_ABS * max(1.0, np.abs(ru).max())
                assert np.abs(gu - ru).max() <= bound, (u, "dX max-abs")
