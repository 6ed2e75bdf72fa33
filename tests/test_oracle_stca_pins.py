"""Pins for the candidate-to-sketch cross-attention oracle (oracle/stca_oracle.cpp).

As for the Sketch Attention oracle, nothing here re-types the oracle's C++: each test
is a closed form, an invariant, a special case that reduces to a library routine
(torch's scaled_dot_product_attention), a 50-digit brute force, or an independent
differentiator (torch autograd, mpmath numerical derivatives). A plausible slip (a
dropped 1/sqrt(d), softmax over candidates instead of sketch rows, a transposed
projection, a missing log Z, a dropped term of the softmax backward, a gradient that
skips the value path) fails at least one of them.
"""
import math

import numpy as np
import pytest

import oracle


def rand_case(groups=(5, 0, 9), k=6, d=8, seed=0, s_scale=1.0):
    g = np.random.default_rng(seed)
    off = np.concatenate([[0], np.cumsum(groups)]).astype(np.int64)
    R = len(groups)
    Q = g.standard_normal((int(off[-1]), d))
    S = g.standard_normal((R, k, d)) * s_scale
    Wq, WK, WV = (g.standard_normal((d, d)) / math.sqrt(d) for _ in range(3))
    return Q, off, S, Wq, WK, WV


# --------------------------------------------------------------------------- library routine
def test_matches_torch_scaled_dot_product_attention():
    """Per user, the op is single-head scaled dot-product attention with the candidates
    as queries and the sketch rows as keys and values (torch float64, CPU)."""
    torch = pytest.importorskip("torch")
    F = torch.nn.functional
    Q, off, S, Wq, WK, WV = rand_case(groups=(7, 1, 0, 40), k=9, d=8, seed=3)
    got = oracle.stca_forward(Q, off, S, Wq, WK, WV)
    t = lambda a: torch.tensor(a, dtype=torch.float64)
    for u in range(len(off) - 1):
        a, b = int(off[u]), int(off[u + 1])
        if a == b:
            continue
        q = t(Q[a:b]) @ t(Wq)
        ref = F.scaled_dot_product_attention(q[None], (t(S[u]) @ t(WK))[None],
                                             (t(S[u]) @ t(WV))[None])[0]
        np.testing.assert_allclose(got["out"][a:b], ref.numpy(), rtol=1e-12, atol=1e-13)
        lse = torch.logsumexp(q @ (t(S[u]) @ t(WK)).T / math.sqrt(Q.shape[1]), dim=1)
        np.testing.assert_allclose(got["lse"][a:b], lse.numpy(), rtol=1e-13)


# --------------------------------------------------------------------------- closed forms
def test_single_row_sketch_returns_its_value():
    """k = 1: every candidate reads the one row, out = S_0 W_V, lse = its score."""
    Q, off, S, Wq, WK, WV = rand_case(groups=(4, 3), k=1, d=5, seed=5)
    got = oracle.stca_forward(Q, off, S, Wq, WK, WV)
    for u in range(2):
        a, b = int(off[u]), int(off[u + 1])
        np.testing.assert_allclose(got["out"][a:b], np.tile(S[u, 0] @ WV, (b - a, 1)), rtol=1e-13)
        z = (Q[a:b] @ Wq) @ (S[u, 0] @ WK) / math.sqrt(5)
        np.testing.assert_allclose(got["lse"][a:b], z, rtol=1e-12, atol=1e-14)


def test_zero_query_projection_gives_the_mean_row():
    """W_q = 0: every score is 0, attention is uniform, out = mean_j S_j W_V, lse = ln k."""
    Q, off, S, Wq, WK, WV = rand_case(groups=(6, 2), k=7, d=4, seed=6)
    got = oracle.stca_forward(Q, off, S, np.zeros_like(Wq), WK, WV)
    for u in range(2):
        a, b = int(off[u]), int(off[u + 1])
        np.testing.assert_allclose(got["out"][a:b], np.tile(S[u].mean(0) @ WV, (b - a, 1)),
                                   rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(got["lse"], math.log(7), rtol=1e-14)


def test_two_rows_logistic_exact():
    """Two rows whose keys differ along q: the weights are a logistic function of the
    score gap, checked on values chosen so it is exactly 1/(1 + e^-2)."""
    d = 4
    Wq = WK = WV = np.eye(d)
    S = np.zeros((1, 2, d))
    S[0, 0, 0], S[0, 1, 1] = 2.0, 1.0          # K_0 = 2 e0, V_0 = 2 e0; K_1 = e1, V_1 = e1
    Q = np.array([[2.0, 0.0, 0.0, 0.0]])        # scores z0 = 4 / 2 = 2, z1 = 0
    got = oracle.stca_forward(Q, [0, 1], S, Wq, WK, WV)
    w0 = 1.0 / (1.0 + math.exp(-2.0))
    np.testing.assert_allclose(got["out"][0], [2 * w0, 1 - w0, 0, 0], rtol=1e-14)
    np.testing.assert_allclose(got["lse"][0], math.log(math.exp(2.0) + 1.0), rtol=1e-14)


def test_sharp_query_picks_the_matching_row():
    """A query far along one row's key direction puts (nearly) all weight on it."""
    d, k = 6, 6
    Wq = WK = WV = np.eye(d)
    S = np.eye(k)[None] * 3.0
    Q = 60.0 * np.eye(d)[[4, 1]]
    got = oracle.stca_forward(Q, [0, 2], S, Wq, WK, WV)
    np.testing.assert_allclose(got["out"], S[0, [4, 1]], rtol=0, atol=1e-30)


# --------------------------------------------------------------------------- invariants
def test_row_permutation_invariance():
    Q, off, S, Wq, WK, WV = rand_case(groups=(8, 5), k=7, d=6, seed=7)
    perm = np.random.default_rng(8).permutation(7)
    a = oracle.stca_forward(Q, off, S, Wq, WK, WV)
    b = oracle.stca_forward(Q, off, S[:, perm], Wq, WK, WV)
    np.testing.assert_allclose(a["out"], b["out"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(a["lse"], b["lse"], rtol=1e-13)


def test_batch_equals_single_user_calls_and_candidates_are_independent():
    """Ragged candidate groups: each user's candidates see only that user's sketch, and
    a candidate's output does not depend on the other candidates."""
    Q, off, S, Wq, WK, WV = rand_case(groups=(3, 0, 11, 1), k=5, d=4, seed=9)
    batch = oracle.stca_forward(Q, off, S, Wq, WK, WV)
    for u in range(4):
        a, b = int(off[u]), int(off[u + 1])
        for c in range(a, b):
            one = oracle.stca_forward(Q[c:c + 1], [0, 1], S[u:u + 1], Wq, WK, WV)
            np.testing.assert_allclose(batch["out"][c], one["out"][0], rtol=1e-13)


def test_output_in_convex_hull_of_values():
    """Weights are a probability vector: with W_V = I and sketch rows on the simplex's
    vertices, each output is a probability vector (non-negative, sums to 1)."""
    d = k = 5
    Q, off, _, Wq, WK, _ = rand_case(groups=(9,), k=k, d=d, seed=10)
    S = np.eye(k)[None]
    got = oracle.stca_forward(Q, off, S, Wq, WK, np.eye(d))
    assert (got["out"] >= 0).all()
    np.testing.assert_allclose(got["out"].sum(1), 1.0, rtol=1e-14)


def test_thread_count_independent():
    Q, off, S, Wq, WK, WV = rand_case(groups=(300, 77), k=6, d=4, seed=11)
    g = np.random.default_rng(12).standard_normal(Q.shape)
    a = oracle.stca_backward(Q, off, S, Wq, WK, WV, g, nthreads=1)
    b = oracle.stca_backward(Q, off, S, Wq, WK, WV, g, nthreads=4)
    for key in a:
        assert np.array_equal(a[key], b[key]), key


def test_bad_offsets_rejected():
    Q, off, S, Wq, WK, WV = rand_case(groups=(2, 2), k=3, d=4)
    with pytest.raises(ValueError):
        oracle.stca_forward(Q, [0, 3, 2], S, Wq, WK, WV)
    with pytest.raises(ValueError):
        oracle.stca_forward(Q, [0, 2, 3], S, Wq, WK, WV)


# --------------------------------------------------------------------------- brute force
def _mp_forward(Q, off, S, Wq, WK, WV):
    import mpmath as mp
    mp.mp.dps = 50
    n, d = Q.shape
    k = S.shape[1]
    cv = lambda v: v if isinstance(v, mp.mpf) else mp.mpf(float(v))
    M = lambda a: [[cv(v) for v in row] for row in a]
    Qm, Wqm, WKm, WVm = M(Q), M(Wq), M(WK), M(WV)
    vecmat = lambda x, W: [mp.fsum(x[c] * W[c][e] for c in range(d)) for e in range(d)]
    sq = mp.sqrt(d)
    out, lse = [], []
    for u in range(len(off) - 1):
        Sm = M(S[u])
        K = [vecmat(Sm[j], WKm) for j in range(k)]
        V = [vecmat(Sm[j], WVm) for j in range(k)]
        for c in range(int(off[u]), int(off[u + 1])):
            q = vecmat(Qm[c], Wqm)
            ex = [mp.exp(mp.fsum(q[e] * K[j][e] for e in range(d)) / sq) for j in range(k)]
            Z = mp.fsum(ex)
            out.append([mp.fsum(ex[j] * V[j][e] for j in range(k)) / Z for e in range(d)])
            lse.append(mp.log(Z))
    return out, lse


def test_brute_force_50_digits():
    Q, off, S, Wq, WK, WV = rand_case(groups=(3, 2), k=4, d=3, seed=13)
    got = oracle.stca_forward(Q, off, S, Wq, WK, WV)
    out, lse = _mp_forward(Q, off, S, Wq, WK, WV)
    np.testing.assert_allclose(got["out"], np.array(out, dtype=float), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(got["lse"], np.array(lse, dtype=float), rtol=1e-13)


def test_backward_brute_force_numeric_derivative_50_digits():
    """Every gradient entry against mpmath's numerical derivative of the 50-digit
    brute-force forward, L = sum_c dO_c . out_c."""
    import mpmath as mp
    Q, off, S, Wq, WK, WV = rand_case(groups=(2, 1), k=3, d=2, seed=14)
    G = np.random.default_rng(15).standard_normal(Q.shape)
    got = oracle.stca_backward(Q, off, S, Wq, WK, WV, G)
    mp.mp.dps = 50
    h = mp.mpf("1e-20")
    base = {"dQ": Q, "dS": S, "dWq": Wq, "dWK": WK, "dWV": WV}

    def loss(arrs):
        out, _ = _mp_forward(arrs["dQ"], off, arrs["dS"], arrs["dWq"], arrs["dWK"], arrs["dWV"])
        return mp.fsum(mp.mpf(float(G[c, e])) * out[c][e]
                       for c in range(G.shape[0]) for e in range(G.shape[1]))

    for name, arr in base.items():
        for idx in np.ndindex(arr.shape):
            def f(eps, name=name, idx=idx, arr=arr):
                a2 = np.array([mp.mpf(float(v)) for v in arr.reshape(-1)], dtype=object)
                a2 = a2.reshape(arr.shape)
                a2[idx] += eps
                return loss({**base, name: a2})
            num = (f(h) - f(-h)) / (2 * h)
            assert abs(float(num) - got[name][idx]) <= 1e-10 * (1 + abs(float(num))), (name, idx)


# --------------------------------------------------------------------------- backward
def _torch_grads(Q, off, S, Wq, WK, WV, G):
    torch = pytest.importorskip("torch")
    F = torch.nn.functional
    t = lambda a: torch.tensor(a, dtype=torch.float64, requires_grad=True)
    Qt, St, Wqt, WKt, WVt = t(Q), t(S), t(Wq), t(WK), t(WV)
    loss = torch.zeros((), dtype=torch.float64)
    for u in range(len(off) - 1):
        a, b = int(off[u]), int(off[u + 1])
        if a == b:
            continue
        o = F.scaled_dot_product_attention((Qt[a:b] @ Wqt)[None], (St[u] @ WKt)[None],
                                           (St[u] @ WVt)[None])[0]
        loss = loss + (torch.tensor(G[a:b]) * o).sum()
    loss.backward()
    return {"dQ": Qt.grad.numpy(), "dS": St.grad.numpy(), "dWq": Wqt.grad.numpy(),
            "dWK": WKt.grad.numpy(), "dWV": WVt.grad.numpy()}


def test_backward_matches_torch_autograd():
    """Hand-derived backward vs. torch float64 autograd through scaled_dot_product_attention."""
    Q, off, S, Wq, WK, WV = rand_case(groups=(70, 0, 1, 200), k=9, d=8, seed=16)
    G = np.random.default_rng(17).standard_normal(Q.shape)
    got = oracle.stca_backward(Q, off, S, Wq, WK, WV, G)
    ref = _torch_grads(Q, off, S, Wq, WK, WV, G)
    for key in ref:
        np.testing.assert_allclose(got[key], ref[key], rtol=1e-10, atol=1e-11, err_msg=key)
    assert not got["dS"][1].any()  # a user without candidates gets no sketch gradient


def test_backward_vanishing_cases():
    """W_V = 0 makes the output identically zero, so only dW_V can be non-zero; a sketch
    whose rows are all equal makes every score equal whatever the query, so the query
    side (dQ, dW_q) gets no gradient."""
    Q, off, S, Wq, WK, WV = rand_case(groups=(12, 5), k=6, d=4, seed=18)
    G = np.random.default_rng(20).standard_normal(Q.shape)
    got = oracle.stca_backward(Q, off, S, Wq, WK, np.zeros_like(WV), G)
    for key in ("dQ", "dS", "dWq", "dWK"):
        assert not got[key].any(), key
    assert np.abs(got["dWV"]).max() > 1e-3
    S2 = np.repeat(S[:, :1], 6, axis=1)
    got2 = oracle.stca_backward(Q, off, S2, Wq, WK, WV, G)
    assert np.abs(got2["dQ"]).max() < 1e-13 and np.abs(got2["dWq"]).max() < 1e-12
    assert np.abs(got2["dS"]).max() > 1e-3


def test_composes_with_sketch_attention_backward():
    """The chain history -> sketch -> cross attention: feeding stca_backward's dS into
    the Sketch Attention oracle's backward as dL/dsketch gives the gradient of the
    composed function (torch float64 autograd of both definitions together)."""
    torch = pytest.importorskip("torch")
    F = torch.nn.functional
    g = np.random.default_rng(21)
    d, k = 6, 5
    lengths = (40, 13)
    xoff = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    X = g.standard_normal((int(xoff[-1]), d))
    P = g.standard_normal((k, d))
    Wk_sa, Wv_sa = (g.standard_normal((d, d)) / math.sqrt(d) for _ in range(2))
    coff = np.array([0, 4, 9], dtype=np.int64)
    Qc = g.standard_normal((9, d))
    Wq, WK, WV = (g.standard_normal((d, d)) / math.sqrt(d) for _ in range(3))
    G = g.standard_normal((9, d))

    fwd = oracle.forward(X, xoff, P, Wk_sa, Wv_sa)
    cb = oracle.stca_backward(Qc, coff, fwd["sketch"], Wq, WK, WV, G)
    got = oracle.backward(X, xoff, P, Wk_sa, Wv_sa, cb["dS"])

    t = lambda a: torch.tensor(a, dtype=torch.float64, requires_grad=True)
    Xt, Pt, Wkt, Wvt = t(X), t(P), t(Wk_sa), t(Wv_sa)
    loss = torch.zeros((), dtype=torch.float64)
    for u in range(2):
        xs = Xt[xoff[u]:xoff[u + 1]]
        A = torch.softmax(Pt @ (xs @ Wkt).T / math.sqrt(d), dim=0)
        sk = (A @ (xs @ Wvt)) / A.sum(1)[:, None]
        a, b = int(coff[u]), int(coff[u + 1])
        T = lambda a_: torch.tensor(a_, dtype=torch.float64)
        o = F.scaled_dot_product_attention((T(Qc[a:b]) @ T(Wq))[None], (sk @ T(WK))[None],
                                           (sk @ T(WV))[None])[0]
        loss = loss + (T(G[a:b]) * o).sum()
    loss.backward()
    for key, ref in (("dX", Xt.grad), ("dP", Pt.grad), ("dWk", Wkt.grad), ("dWv", Wvt.grad)):
        np.testing.assert_allclose(got[key], ref.numpy(), rtol=1e-9, atol=1e-11, err_msg=key)


# --------------------------------------------------------------------------- ragged key rows
def _ragged_case(key_counts=(9, 1, 0, 30), groups=(4, 2, 3, 50), d=8, seed=30):
    g = np.random.default_rng(seed)
    coff = np.concatenate([[0], np.cumsum(groups)]).astype(np.int64)
    koff = np.concatenate([[0], np.cumsum(key_counts)]).astype(np.int64)
    Q = g.standard_normal((int(coff[-1]), d))
    Kx = g.standard_normal((int(koff[-1]), d))
    Wq, WK, WV = (g.standard_normal((d, d)) / math.sqrt(d) for _ in range(3))
    return Q, coff, Kx, koff, Wq, WK, WV


def test_ragged_keys_match_torch_sdpa_per_user():
    """Each user attends over its own number of key rows (1, 9, 30, and none: out = 0,
    lse = -inf)."""
    torch = pytest.importorskip("torch")
    F = torch.nn.functional
    Q, coff, Kx, koff, Wq, WK, WV = _ragged_case()
    got = oracle.stca_forward_keys(Q, coff, Kx, koff, Wq, WK, WV)
    t = lambda a: torch.tensor(a, dtype=torch.float64)
    for u in range(4):
        a, b = int(coff[u]), int(coff[u + 1])
        ka, kb = int(koff[u]), int(koff[u + 1])
        if ka == kb:
            assert not got["out"][a:b].any() and np.isneginf(got["lse"][a:b]).all()
            continue
        q, K, V = t(Q[a:b]) @ t(Wq), t(Kx[ka:kb]) @ t(WK), t(Kx[ka:kb]) @ t(WV)
        ref = F.scaled_dot_product_attention(q[None], K[None], V[None])[0]
        np.testing.assert_allclose(got["out"][a:b], ref.numpy(), rtol=1e-12, atol=1e-13)
        lse = torch.logsumexp(q @ K.T / math.sqrt(Q.shape[1]), dim=1)
        np.testing.assert_allclose(got["lse"][a:b], lse.numpy(), rtol=1e-13)


def test_equal_key_counts_reduce_to_the_sketch_case():
    Q, off, S, Wq, WK, WV = rand_case(groups=(5, 0, 9), k=6, d=8, seed=31)
    a = oracle.stca_forward(Q, off, S, Wq, WK, WV)
    b = oracle.stca_forward_keys(Q, off, S.reshape(-1, 8), np.arange(4) * 6, Wq, WK, WV)
    assert np.array_equal(a["out"], b["out"]) and np.array_equal(a["lse"], b["lse"])


def test_recent_suffix_is_the_last_tokens_of_each_history():
    """The recent branch reads the last min(n_u, L) tokens: with L = 4, a user of 10
    tokens contributes rows 6..9, a user of 3 all three, an empty user none."""
    X = np.arange(17 * 2, dtype=float).reshape(17, 2)
    off = np.array([0, 10, 13, 13, 17])
    Kx, koff = oracle.recent_suffix(X, off, 4)
    assert koff.tolist() == [0, 4, 7, 7, 11]
    np.testing.assert_array_equal(Kx, X[[6, 7, 8, 9, 10, 11, 12, 13, 14, 15, 16]])


def test_recent_branch_matches_sdpa_on_the_suffix():
    torch = pytest.importorskip("torch")
    F = torch.nn.functional
    g = np.random.default_rng(32)
    d, L = 8, 25
    off = np.array([0, 100, 110, 110, 160])
    X = g.standard_normal((160, d))
    coff = np.array([0, 3, 5, 6, 9])
    Q = g.standard_normal((9, d))
    Wq, WK, WV = (g.standard_normal((d, d)) / math.sqrt(d) for _ in range(3))
    Kx, koff = oracle.recent_suffix(X, off, L)
    got = oracle.stca_forward_keys(Q, coff, Kx, koff, Wq, WK, WV)
    t = lambda a: torch.tensor(a, dtype=torch.float64)
    for u in (0, 1, 3):
        a, b = int(coff[u]), int(coff[u + 1])
        rows = X[max(off[u], off[u + 1] - L):off[u + 1]]
        ref = F.scaled_dot_product_attention((t(Q[a:b]) @ t(Wq))[None], (t(rows) @ t(WK))[None],
                                             (t(rows) @ t(WV))[None])[0]
        np.testing.assert_allclose(got["out"][a:b], ref.numpy(), rtol=1e-12, atol=1e-13)
    assert not got["out"][5].any()  # user 2 has no history


def test_ragged_backward_matches_torch_autograd():
    torch = pytest.importorskip("torch")
    F = torch.nn.functional
    Q, coff, Kx, koff, Wq, WK, WV = _ragged_case(seed=33)
    G = np.random.default_rng(34).standard_normal(Q.shape)
    got = oracle.stca_backward_keys(Q, coff, Kx, koff, Wq, WK, WV, G)
    tt = lambda a: torch.tensor(a, dtype=torch.float64, requires_grad=True)
    Qt, Kt, Wqt, WKt, WVt = tt(Q), tt(Kx), tt(Wq), tt(WK), tt(WV)
    loss = torch.zeros((), dtype=torch.float64)
    for u in range(4):
        a, b = int(coff[u]), int(coff[u + 1])
        ka, kb = int(koff[u]), int(koff[u + 1])
        if a == b or ka == kb:
            continue
        o = F.scaled_dot_product_attention((Qt[a:b] @ Wqt)[None], (Kt[ka:kb] @ WKt)[None],
                                           (Kt[ka:kb] @ WVt)[None])[0]
        loss = loss + (torch.tensor(G[a:b]) * o).sum()
    loss.backward()
    ref = {"dQ": Qt.grad, "dKx": Kt.grad, "dWq": Wqt.grad, "dWK": WKt.grad, "dWV": WVt.grad}
    for key, r in ref.items():
        np.testing.assert_allclose(got[key], r.numpy(), rtol=1e-10, atol=1e-11, err_msg=key)
