"""CPU model of the launch sequences in csrc/sa_stca.cu, checked against the oracle.

Each step below restates what one launch computes, from the contracts in
csrc/sa_internal.h (launch_fold: Pf = scale * P Wk^T, rounded to bf16 when asked; the
GEMM's kEpiLse / kEpiAExp / kEpiStoreF32 epilogues) and the kernels of sa_stca.cu and
sa_stca_keys.cu, including every rounding to bf16. If the composition's algebra were
wrong (a fold with its operands swapped, a missing log2(e), the sketch used
untransposed, W_V applied on the wrong side), this model would miss the oracle by far
more than the bf16 tolerance. It needs no GPU and shares nothing with the oracle.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from prototype_sketch_attention_b200 import inputs


def bf16(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).bfloat16().float().numpy().astype(np.float64)


def fold(P, Wk, scale, to_bf16):
    out = scale * (np.asarray(P, np.float64) @ np.asarray(Wk, np.float64).T)
    return bf16(out) if to_bf16 else out.astype(np.float32).astype(np.float64)


def model_forward(cw):
    """The forward: the flash kernel of sa_stca_keys.cu over the bf16 sketch rows. The
    kernel's running maximum stays within 8 (log2 units) of the row maximum and only
    scales the bf16 weights' exponent, so the model uses the row maximum."""
    Q = cw.Q.float().numpy().astype(np.float64)
    S = cw.S.numpy().astype(np.float64)
    Wq, WK, WV = (t.float().numpy().astype(np.float64) for t in (cw.Wq, cw.WK, cw.WV))
    R, k, d = S.shape
    coff = cw.cand_offsets.numpy()
    Sb = bf16(S)                                               # stca_sketch_bf16_kernel
    M = fold(Wq, WK, 1.0, False)                               # keys_mfold: W_q W_K^T, fp32
    Qp = fold(Q, M.T, math.log2(math.e) / math.sqrt(d), False)  # keys_qfold: Q M ..., fp32
    hi_q = bf16(Qp)
    lo_q = bf16(Qp - hi_q)
    out = np.zeros((Q.shape[0], d))
    lse = np.zeros(Q.shape[0])
    for u in range(R):
        a, b = int(coff[u]), int(coff[u + 1])
        if a == b:
            continue
        z = (hi_q[a:b] + lo_q[a:b]) @ Sb[u].T                  # two score MMAs, log2 units
        m = z.max(axis=1, keepdims=True)
        e = np.exp2(z - m)
        l = e.sum(axis=1, keepdims=True)
        O = (bf16(e) @ Sb[u] / l).astype(np.float32).astype(np.float64)  # bf16 P, fp32 O'
        hi = bf16(O)
        lo = bf16(O - hi)
        out[a:b] = hi @ bf16(WV) + lo @ bf16(WV)               # two GEMM phases
        lse[a:b] = (m[:, 0] + np.log2(l[:, 0])) * math.log(2.0)
    return out, lse


@pytest.mark.parametrize("counts,k,d", [([300, 0, 1, 129], 1024, 128), ([5, 77], 200, 64),
                                        ([40], 384, 64)])
def test_composition_model_meets_the_oracle_within_bf16_tolerance(counts, k, d):
    cw = inputs.make_cross_workload(counts, k, d, seed=500 + k + d + len(counts))
    got, lse = model_forward(cw)
    f = cw.to_f64()
    ref = oracle.stca_forward(f["Q"], f["cand_offsets"], f["S"], f["Wq"], f["WK"], f["WV"])
    off = f["cand_offsets"]
    for u in range(cw.R):
        a, b = int(off[u]), int(off[u + 1])
        if a == b:
            continue
        num = np.linalg.norm(got[a:b] - ref["out"][a:b])
        den = np.linalg.norm(ref["out"][a:b])
        assert num / den <= 1e-2, (u, num / den)
        assert np.abs(got[a:b] - ref["out"][a:b]).max() <= 5e-2
    assert np.abs(lse - ref["lse"]).max() <= 5e-2


def test_composition_model_catches_a_swapped_fold():
    """The check above has teeth: folding W_q W_K^T the other way round fails it."""
    cw = inputs.make_cross_workload([64, 30], 256, 64, seed=7)
    f = cw.to_f64()
    ref = oracle.stca_forward(f["Q"], f["cand_offsets"], f["S"], f["Wq"], f["WK"], f["WV"])
    global fold
    orig = fold
    try:
        fold = lambda P, Wk, scale, to_bf16: orig(Wk, P, scale, to_bf16) if P.shape == Wk.shape \
            else orig(P, Wk, scale, to_bf16)
        got, _ = model_forward(cw)
    finally:
        fold = orig
    err = np.linalg.norm(got - ref["out"]) / np.linalg.norm(ref["out"])
    assert err > 5e-2, err


def model_backward(cw, G, ln2=math.log(2.0)):
    """The backward: the sketch as the key rows of sa_stca_keys.cu's backward (the forward
    recomputed, dO' and dW_V on the GEMM, the tcgen05 kernel's G1 and dKx = dS, then dQ,
    dW_q, dW_K), step by step with its roundings."""
    Q = cw.Q.float().numpy().astype(np.float64)
    S = cw.S.numpy().astype(np.float64)
    Wq, WK, WV = (t.float().numpy().astype(np.float64) for t in (cw.Wq, cw.WK, cw.WV))
    R, k, d = S.shape
    coff = cw.cand_offsets.numpy()
    n = Q.shape[0]
    isd = 1.0 / math.sqrt(d)
    log2e = math.log2(math.e)
    Sb = bf16(S)
    M = fold(Wq, WK, 1.0, False)
    Qp = fold(Q, M.T, log2e * isd, False)
    hq = bf16(Qp)
    lq = bf16(Qp - hq)
    O = np.zeros((n, d))
    lse2 = np.zeros(n)
    for u in range(R):                                         # the forward, recomputed
        a, b = int(coff[u]), int(coff[u + 1])
        if a == b:
            continue
        z = (hq[a:b] + lq[a:b]) @ Sb[u].T
        m = z.max(axis=1, keepdims=True)
        e = np.exp2(z - m)
        l = e.sum(axis=1, keepdims=True)
        O[a:b] = (bf16(e) @ Sb[u] / l).astype(np.float32)
        lse2[a:b] = m[:, 0] + np.log2(l[:, 0])
    Gh, Gl = bf16(G), bf16(G - bf16(G))
    dO = (Gh @ bf16(WV).T + Gl @ bf16(WV).T).astype(np.float32).astype(np.float64)
    dWV = bf16(O).T @ bf16(G)
    dOb = bf16(dO)
    D = (dOb * O).sum(axis=1)                                  # keys_rowdot_kernel
    G1 = np.zeros((n, d))
    dS = np.zeros((R, k, d))
    for u in range(R):                                         # stca_keys_bwd_kernel
        a, b = int(coff[u]), int(coff[u + 1])
        if a == b:
            continue
        A = np.exp2((hq[a:b] + lq[a:b]) @ Sb[u].T - lse2[a:b, None])
        dz = A * (dOb[a:b] @ Sb[u].T - D[a:b, None])
        G1[a:b] = (bf16(dz) @ Sb[u]).astype(np.float32)
        dS[u] = ln2 * (bf16(dz).T @ hq[a:b] + bf16(A * log2e).T @ dOb[a:b])
    Mts = fold(WK, Wq, isd, True)
    G1h, G1l = bf16(G1), bf16(G1 - bf16(G1))
    dQ = G1h @ Mts + G1l @ Mts
    dM = isd * (Q.T @ bf16(G1))
    dWq = dM @ WK
    dWK = dM.T @ Wq
    return {"dQ": dQ, "dS": dS, "dWq": dWq, "dWK": dWK, "dWV": dWV}


@pytest.mark.parametrize("counts,k,d", [([300, 0, 1, 129], 1024, 128), ([5, 77], 200, 64)])
def test_backward_composition_model_meets_the_oracle(counts, k, d):
    cw = inputs.make_cross_workload(counts, k, d, seed=600 + k + d)
    G = np.random.default_rng(601).standard_normal((int(cw.cand_offsets[-1]), d))
    got = model_backward(cw, G)
    f = cw.to_f64()
    ref = oracle.stca_backward(f["Q"], f["cand_offsets"], f["S"], f["Wq"], f["WK"], f["WV"], G)
    for key in ref:
        r = ref[key]
        e = np.linalg.norm(got[key] - r) / max(np.linalg.norm(r), 1e-30)
        assert e <= 1e-2, (key, e)
        assert np.abs(got[key] - r).max() <= 5e-2 * max(np.abs(r).max(), 1e-30), (key, "max-abs")


def test_backward_model_catches_a_missing_ln2():
    """The backward check has teeth: dKx = dS without the ln 2 that turns the log2-unit
    Q' back into natural units fails it."""
    cw = inputs.make_cross_workload([40, 9], 256, 64, seed=602)
    G = np.random.default_rng(603).standard_normal((49, 64))
    got = model_backward(cw, G, ln2=1.0)
    f = cw.to_f64()
    ref = oracle.stca_backward(f["Q"], f["cand_offsets"], f["S"], f["Wq"], f["WK"], f["WV"], G)
    err = np.linalg.norm(got["dS"] - ref["dS"]) / np.linalg.norm(ref["dS"])
    assert err > 5e-2, err
