"""Pins for the fp64 oracle: checks against what the pages and the mathematics fix.

None of these re-types the oracle's C++ and compares it with itself. Each test is
a closed form, an invariant, a special case with a textbook answer, a brute force
at 50 digits, or (for the backward) an independent way of differentiating.
A plausible slip in the oracle (dropped 1/sqrt(d), softmax over tokens instead
of prototypes, transposed W_k or W_v, sum instead of mean, wrong sign in the
backward, a missed dL/dmass term) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(12345)


def rand_case(R=2, lengths=(37, 11), d=8, k=5, seed=0):
    g = np.random.default_rng(seed)
    lengths = np.asarray(lengths[:R], dtype=np.int64)
    off = np.concatenate([[0], np.cumsum(lengths)])
    X = g.standard_normal((int(off[-1]), d))
    P = g.standard_normal((k, d))
    Wk = g.standard_normal((d, d)) / math.sqrt(d)
    Wv = g.standard_normal((d, d)) / math.sqrt(d)
    return X, off, P, Wk, Wv


# --------------------------------------------------------------------------- pages
def test_golden_sketch_size_fixed_in_n():
    """The sketch is k x d whatever n is (blog 'ELI5'; review 'Summary', 1K x 128)."""
    with open(os.path.join(GOLDEN, "pages_numbers.json")) as f:
        gold = json.load(f)
    rr = gold["row_reduction"]
    assert rr["n"] // rr["k"] == rr["ratio_floor"]
    k, d = 16, 8
    X, _, P, Wk, Wv = rand_case(R=1, lengths=(300,), d=d, k=k)
    for n in (1, 7, 300):
        out = oracle.forward(X[:n], [0, n], P, Wk, Wv)
        assert out["sketch"].shape == (1, k, d)
        assert out["mass"].shape == (1, k)
    dep = gold["deployed_sketch"]
    assert (dep["k"], dep["d"]) == (1024, 128)


# --------------------------------------------------------------------------- invariants
def test_unit_mass_per_token():
    """Each token spreads unit mass over prototypes, so total mass = n per user."""
    X, off, P, Wk, Wv = rand_case(R=2, lengths=(37, 11), d=8, k=5)
    out = oracle.forward(X, off, P, Wk, Wv)
    n = np.diff(off)
    np.testing.assert_allclose(out["mass"].sum(axis=1), n, rtol=1e-13)
    assert (out["mass"] > 0).all()
    # lse is log-sum-exp of the scores: exp(s - lse) summed over j must be 1; via
    # the k=1 and P=0 cases below its value is pinned exactly.


def test_thread_count_independent():
    X, off, P, Wk, Wv = rand_case(R=2, lengths=(2500, 1300), d=8, k=5)
    a = oracle.forward(X, off, P, Wk, Wv, nthreads=1)
    b = oracle.forward(X, off, P, Wk, Wv, nthreads=4)
    for key in a:
        assert np.array_equal(a[key], b[key]), key


def test_permutation_invariance():
    X, off, P, Wk, Wv = rand_case(R=1, lengths=(64,), d=8, k=6)
    perm = np.random.default_rng(3).permutation(64)
    a = oracle.forward(X, off, P, Wk, Wv)
    b = oracle.forward(X[perm], off, P, Wk, Wv)
    np.testing.assert_allclose(b["sketch"], a["sketch"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(b["mass"], a["mass"], rtol=1e-12)
    np.testing.assert_allclose(b["lse"], a["lse"][perm], rtol=1e-13)


def test_split_and_merge_equals_whole():
    """Splitting one user's history in two and merging the mass-weighted means
    gives the whole: sketch = (s1 m1 + s2 m2) / (m1 + m2). This is what split-n
    partial sums rely on."""
    X, off, P, Wk, Wv = rand_case(R=1, lengths=(90,), d=8, k=7)
    whole = oracle.forward(X, [0, 90], P, Wk, Wv)
    parts = oracle.forward(X, [0, 33, 90], P, Wk, Wv)
    s, m = parts["sketch"], parts["mass"]
    merged = (s[0] * m[0][:, None] + s[1] * m[1][:, None]) / (m[0] + m[1])[:, None]
    np.testing.assert_allclose(merged, whole["sketch"][0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(m[0] + m[1], whole["mass"][0], rtol=1e-13)
    np.testing.assert_allclose(parts["xsketch"][0] + parts["xsketch"][1], whole["xsketch"][0],
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(parts["lse"], whole["lse"])


def test_batch_equals_single_calls():
    X, off, P, Wk, Wv = rand_case(R=3, lengths=(20, 0, 13), d=8, k=4)
    off = np.array([0, 20, 20, 33])
    batch = oracle.forward(X, off, P, Wk, Wv)
    for u in range(3):
        a, b = off[u], off[u + 1]
        single = oracle.forward(X[a:b], [0, b - a], P, Wk, Wv)
        np.testing.assert_array_equal(batch["sketch"][u], single["sketch"][0])
        np.testing.assert_array_equal(batch["mass"][u], single["mass"][0])
    # the empty user gets zeros
    assert not batch["sketch"][1].any() and not batch["mass"][1].any()


def test_duplicate_prototypes_give_equal_rows():
    X, off, P, Wk, Wv = rand_case(R=1, lengths=(50,), d=8, k=5)
    P[3] = P[1]
    out = oracle.forward(X, off, P, Wk, Wv)
    np.testing.assert_array_equal(out["sketch"][0, 3], out["sketch"][0, 1])
    np.testing.assert_array_equal(out["mass"][0, 3], out["mass"][0, 1])


def test_identical_tokens_rows_equal_value():
    """All tokens equal to x: every row is the mean of identical values, x W_v."""
    d, k, n = 8, 6, 25
    _, _, P, Wk, Wv = rand_case(R=1, lengths=(1,), d=d, k=k)
    x = np.random.default_rng(9).standard_normal(d)
    X = np.tile(x, (n, 1))
    out = oracle.forward(X, [0, n], P, Wk, Wv)
    np.testing.assert_allclose(out["sketch"][0], np.tile(x @ Wv, (k, 1)), rtol=1e-12, atol=1e-14)
    assert np.ptp(out["lse"]) == 0.0


# --------------------------------------------------------------------------- closed forms
def test_k1_is_mean_of_values():
    """k=1: the single prototype takes all mass; the row is mean(X) W_v, lse = score."""
    X, off, P, Wk, Wv = rand_case(R=2, lengths=(31, 9), d=8, k=1)
    Wv = Wv + np.triu(np.ones((8, 8)))  # clearly non-symmetric
    out = oracle.forward(X, off, P, Wk, Wv)
    for u in range(2):
        xs = X[off[u]:off[u + 1]]
        np.testing.assert_allclose(out["sketch"][u, 0], xs.mean(axis=0) @ Wv, rtol=1e-12)
        np.testing.assert_allclose(out["mass"][u, 0], len(xs), rtol=1e-15)
        np.testing.assert_allclose(out["xsketch"][u, 0], xs.sum(axis=0), rtol=1e-12)
    # with one prototype the log-sum-exp equals the score itself
    scores = (X @ Wk) @ P[0] / math.sqrt(8)
    np.testing.assert_allclose(out["lse"], scores, rtol=1e-12, atol=1e-14)


def test_zero_prototypes_uniform():
    """P = 0: all scores are 0, A = 1/k, mass = n/k, rows = mean V, lse = log k."""
    X, off, _, Wk, Wv = rand_case(R=1, lengths=(40,), d=8, k=6)
    P = np.zeros((6, 8))
    out = oracle.forward(X, off, P, Wk, Wv)
    np.testing.assert_allclose(out["mass"][0], np.full(6, 40 / 6), rtol=1e-14)
    np.testing.assert_allclose(out["sketch"][0], np.tile(X.mean(0) @ Wv, (6, 1)), rtol=1e-12)
    np.testing.assert_allclose(out["lse"], np.full(40, math.log(6)), rtol=1e-14)


def _perm_wk(d):
    """W_k = 2 * (permutation matrix of the 3-cycle 0->1->2->0), non-symmetric."""
    pi = list(range(d))
    pi[0], pi[1], pi[2] = 1, 2, 0
    Wk = np.zeros((d, d))
    for c in range(d):
        Wk[c, pi[c]] = 2.0
    return Wk


def test_two_prototype_logistic_exact():
    """Two prototypes, P_1 = 0: A_0t = sigmoid(s_0t). With d=4, W_k = 2*Pi and
    P_0 = a*e_1 we get s_0t = a*2*X_t[0]/sqrt(4) = a*X_t[0]; choosing
    X_t[0] = ln(3)/a gives A_0t = 3/4 exactly, so mass = (0.75 n, 0.25 n) and
    lse_t = ln 4. A dropped 1/sqrt(d) gives 9/10; a transposed W_k makes the score
    depend on X_t[2]; a softmax over tokens gives mass 1 per prototype."""
    d, n, a = 4, 12, 1.7
    g = np.random.default_rng(5)
    X = g.standard_normal((n, d))
    X[:, 0] = math.log(3.0) / a
    P = np.zeros((2, d))
    P[0, 1] = a
    Wk = _perm_wk(d)
    Wv = g.standard_normal((d, d))
    out = oracle.forward(X, [0, n], P, Wk, Wv)
    np.testing.assert_allclose(out["mass"][0], [0.75 * n, 0.25 * n], rtol=1e-14)
    np.testing.assert_allclose(out["lse"], np.full(n, math.log(4.0)), rtol=1e-14)
    meanV = X.mean(0) @ Wv
    np.testing.assert_allclose(out["sketch"][0], np.stack([meanV, meanV]), rtol=1e-12, atol=1e-14)


def test_hard_assignment_is_cluster_means():
    """Large, well-separated prototypes make A one-hot (to within exp(-40)): each
    row is then the mean of V over the tokens whose nearest prototype it is, and
    mass is the cluster size -- the textbook hard-clustering means."""
    d, k, n = 6, 3, 60
    g = np.random.default_rng(11)
    Wk = _perm_wk(d)            # K_t = 2 X_t Pi, and sqrt(d) is undone below
    U = np.eye(d)[:k]           # cluster directions e_0, e_1, e_2
    lab = g.integers(0, k, n)
    X = U[lab] + 0.05 * g.standard_normal((n, d))
    # s_jt = P_j . (2 X_t Pi) / sqrt(d); pick P_j = 40 sqrt(d)/2 * (u_j Pi)
    P = np.stack([(40.0 * math.sqrt(d) / 2.0) * (U[j] @ Wk / 2.0) for j in range(k)])
    Wv = g.standard_normal((d, d))
    out = oracle.forward(X, [0, n], P, Wk, Wv)
    V = X @ Wv
    for j in range(k):
        sel = lab == j
        np.testing.assert_allclose(out["mass"][0, j], sel.sum(), rtol=1e-9)
        np.testing.assert_allclose(out["sketch"][0, j], V[sel].mean(0), rtol=1e-8, atol=1e-10)


# --------------------------------------------------------------------------- brute force
def _mp_forward(X, off, P, Wk, Wv):
    import mpmath as mp
    mp.mp.dps = 50
    n, d = X.shape
    k = P.shape[0]
    R = len(off) - 1
    cv = lambda v: v if isinstance(v, mp.mpf) else mp.mpf(float(v))
    Xm = [[cv(v) for v in row] for row in X]
    Pm = [[cv(v) for v in row] for row in P]
    Wkm = [[cv(v) for v in row] for row in Wk]
    Wvm = [[cv(v) for v in row] for row in Wv]
    sq = mp.sqrt(d)
    sketch = [[[mp.mpf(0)] * d for _ in range(k)] for _ in range(R)]
    mass = [[mp.mpf(0)] * k for _ in range(R)]
    lse = [mp.mpf(0)] * n
    for u in range(R):
        num = [[mp.mpf(0)] * d for _ in range(k)]
        for t in range(int(off[u]), int(off[u + 1])):
            Kt = [mp.fsum(Xm[t][c] * Wkm[c][e] for c in range(d)) for e in range(d)]
            Vt = [mp.fsum(Xm[t][c] * Wvm[c][e] for c in range(d)) for e in range(d)]
            s = [mp.fsum(Pm[j][e] * Kt[e] for e in range(d)) / sq for j in range(k)]
            ex = [mp.exp(v) for v in s]
            Z = mp.fsum(ex)
            lse[t] = mp.log(Z)
            for j in range(k):
                a = ex[j] / Z
                mass[u][j] += a
                for e in range(d):
                    num[j][e] += a * Vt[e]
        for j in range(k):
            for e in range(d):
                sketch[u][j][e] = num[j][e] / mass[u][j] if mass[u][j] else mp.mpf(0)
    return sketch, mass, lse


def test_brute_force_50_digits():
    X, off, P, Wk, Wv = rand_case(R=2, lengths=(4, 2), d=3, k=4, seed=7)
    out = oracle.forward(X, off, P, Wk, Wv)
    sk, ms, ls = _mp_forward(X, off, P, Wk, Wv)
    np.testing.assert_allclose(out["sketch"], np.array(sk, dtype=float), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(out["mass"], np.array(ms, dtype=float), rtol=1e-13)
    np.testing.assert_allclose(out["lse"], np.array(ls, dtype=float), rtol=1e-13)


def test_backward_brute_force_numeric_derivative_50_digits():
    """Every gradient entry against mpmath's numerical derivative of the 50-digit
    brute-force forward, L = sum G . sketch + sum Gm . mass."""
    import mpmath as mp
    X, off, P, Wk, Wv = rand_case(R=2, lengths=(3, 2), d=2, k=3, seed=21)
    g = np.random.default_rng(22)
    G = g.standard_normal((2, 3, 2))
    Gm = g.standard_normal((2, 3))
    got = oracle.backward(X, off, P, Wk, Wv, G, Gm)

    def loss(Xa, Pa, Wka, Wva):
        sk, ms, _ = _mp_forward(Xa, off, Pa, Wka, Wva)
        tot = mp.mpf(0)
        for u in range(2):
            for j in range(3):
                tot += mp.mpf(float(Gm[u, j])) * ms[u][j]
                for e in range(2):
                    tot += mp.mpf(float(G[u, j, e])) * sk[u][j][e]
        return tot

    mp.mp.dps = 50
    h = mp.mpf("1e-20")
    params = {"dX": X, "dP": P, "dWk": Wk, "dWv": Wv}
    for name, arr in params.items():
        for idx in np.ndindex(arr.shape):
            def f(eps, arr=arr, idx=idx, name=name):
                arrs = {"dX": X, "dP": P, "dWk": Wk, "dWv": Wv}
                a2 = [[mp.mpf(float(v)) for v in row] for row in arr]  # exact: arr is fp64
                a2[idx[0]][idx[1]] += eps
                arrs[name] = a2
                return loss(np.array(arrs["dX"], dtype=object), np.array(arrs["dP"], dtype=object),
                            np.array(arrs["dWk"], dtype=object), np.array(arrs["dWv"], dtype=object))
            num = (f(h) - f(-h)) / (2 * h)
            assert abs(float(num) - got[name][idx]) <= 1e-10 * (1 + abs(float(num))), (name, idx)


# --------------------------------------------------------------------------- backward
def _torch_loss_grads(X, off, P, Wk, Wv, G, Gm):
    torch = pytest.importorskip("torch")
    t = lambda a: torch.tensor(a, dtype=torch.float64, requires_grad=True)
    Xt, Pt, Wkt, Wvt = t(X), t(P), t(Wk), t(Wv)
    d = X.shape[1]
    loss = torch.zeros((), dtype=torch.float64)
    for u in range(len(off) - 1):
        xs = Xt[off[u]:off[u + 1]]
        if xs.shape[0] == 0:
            continue
        A = torch.softmax(Pt @ (xs @ Wkt).T / math.sqrt(d), dim=0)      # [k, n]
        mass = A.sum(1)
        sk = (A @ (xs @ Wvt)) / mass[:, None]
        loss = loss + (torch.tensor(G[u]) * sk).sum()
        if Gm is not None:
            loss = loss + (torch.tensor(Gm[u]) * mass).sum()
    loss.backward()
    return {"dX": Xt.grad.numpy(), "dP": Pt.grad.numpy(), "dWk": Wkt.grad.numpy(),
            "dWv": Wvt.grad.numpy()}


@pytest.mark.parametrize("with_gm", [False, True])
def test_backward_matches_torch_autograd(with_gm):
    """Hand-derived backward vs. torch float64 autograd (a library differentiator)."""
    X, off, P, Wk, Wv = rand_case(R=3, lengths=(120, 1, 57), d=8, k=6, seed=31)
    g = np.random.default_rng(32)
    G = g.standard_normal((3, 6, 8))
    Gm = g.standard_normal((3, 6)) if with_gm else None
    got = oracle.backward(X, off, P, Wk, Wv, G, Gm)
    ref = _torch_loss_grads(X, off, P, Wk, Wv, G, Gm)
    for key in ref:
        np.testing.assert_allclose(got[key], ref[key], rtol=1e-10, atol=1e-11, err_msg=key)


def test_backward_matches_finite_differences_of_oracle_forward():
    X, off, P, Wk, Wv = rand_case(R=2, lengths=(9, 5), d=4, k=3, seed=41)
    g = np.random.default_rng(42)
    G = g.standard_normal((2, 3, 4))
    Gm = g.standard_normal((2, 3))
    got = oracle.backward(X, off, P, Wk, Wv, G, Gm)

    def L(X_, P_, Wk_, Wv_):
        o = oracle.forward(X_, off, P_, Wk_, Wv_)
        return float((o["sketch"] * G).sum() + (o["mass"] * Gm).sum())

    h = 1e-6
    base = {"dX": X, "dP": P, "dWk": Wk, "dWv": Wv}
    for name, arr in base.items():
        for idx in np.ndindex(arr.shape):
            plus = {k2: v.copy() for k2, v in base.items()}
            minus = {k2: v.copy() for k2, v in base.items()}
            plus[name][idx] += h
            minus[name][idx] -= h
            num = (L(plus["dX"], plus["dP"], plus["dWk"], plus["dWv"]) -
                   L(minus["dX"], minus["dP"], minus["dWk"], minus["dWv"])) / (2 * h)
            assert abs(num - got[name][idx]) <= 1e-6 * (1 + abs(num)), (name, idx, num)


def test_backward_k1_no_prototype_gradient():
    """With one prototype the softmax is constant 1, so dP = dW_k = 0 exactly."""
    X, off, P, Wk, Wv = rand_case(R=2, lengths=(15, 6), d=5, k=1, seed=51)
    G = np.random.default_rng(52).standard_normal((2, 1, 5))
    got = oracle.backward(X, off, P, Wk, Wv, G, np.ones((2, 1)))
    assert not got["dP"].any() and not got["dWk"].any()


def test_backward_total_mass_loss_has_zero_gradient():
    """L = sum_j mass_j = n does not depend on any input: every gradient is 0."""
    X, off, P, Wk, Wv = rand_case(R=2, lengths=(15, 6), d=5, k=4, seed=61)
    got = oracle.backward(X, off, P, Wk, Wv, np.zeros((2, 4, 5)), np.ones((2, 4)))
    for key, val in got.items():
        assert np.abs(val).max() < 1e-12, key


def test_bad_offsets_rejected():
    X, off, P, Wk, Wv = rand_case(R=2, lengths=(5, 5), d=4, k=3)
    with pytest.raises(ValueError):
        oracle.forward(X, [0, 6, 4], P, Wk, Wv)
    with pytest.raises(ValueError):
        oracle.forward(X, [0, 5, 9], P, Wk, Wv)
