"""GPU forward parity: the CUDA path through the C ABI vs the fp64 oracle.

Small cases compare every output element; they span several 128-token tiles, a ragged
tail, empty users, users shorter than a tile, k not a multiple of 128, and every
cluster size (k = 64 .. 2048). The full-size configurations run in the same launch
configuration that bench.py times and are compared on sampled users (the oracle
recomputes those users exactly), plus the unit-mass property on every user.
"""
import numpy as np
import pytest
import torch

from parity_util import check_forward, gpu_forward, rel_l2
from prototype_sketch_attention_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("lengths,k,d", [
    ([300, 0, 1037], 128, 128),
    ([1, 127, 128, 129], 256, 128),
    ([2000, 55], 1024, 128),
    ([700], 2048, 128),
    ([513, 9], 200, 128),
    ([640, 77], 1024, 64),
    ([130], 64, 64),
    ([4100, 3], 512, 128),
    ([100, 200, 129, 60, 300, 1, 128, 257, 90, 5000, 2, 383, 384, 385], 1024, 128),
    # cluster sizes C = 5, 6 and 8 with more users and tiles per cluster (batches this
    # small leave the helper grid idle: the full-size tests below cover it)
    ([20000, 0, 15000, 129, 7000], 1024, 128),
    ([30000, 700, 20000], 640, 128),
    ([9000, 25000, 1, 12000], 768, 128),
    ([11000, 4000, 0, 9000], 1000, 128),
])
def test_bf16_small_full_compare(lengths, k, d):
    w = inputs.make_workload(lengths, d, k, "bf16", seed=11 + k + d + len(lengths))
    _, out = gpu_forward(w)
    check_forward(w, out)


@pytest.mark.parametrize("lengths,k,d", [
    ([300, 0, 77], 64, 64),
    ([1000], 1000, 128),
    ([129, 5], 2048, 64),
])
def test_fp32_small_full_compare(lengths, k, d):
    w = inputs.make_workload(lengths, d, k, "f32", seed=5 + k)
    _, out = gpu_forward(w)
    check_forward(w, out)


def test_config1_fp32():
    w = inputs.make_config(1)
    _, out = gpu_forward(w)
    check_forward(w, out)


def test_config2_full_user():
    w = inputs.make_config(2)
    _, out = gpu_forward(w)
    check_forward(w, out)


def _unit_mass_all_users(w, out):
    mass = out["mass"].double().sum(dim=1).cpu().numpy()
    n = np.diff(w.offsets.numpy())
    np.testing.assert_allclose(mass, n, rtol=2e-3)


def _range_bounds(T, k, d):
    """Inner bounds between the forward's tile ranges (clusters, then helper CTAs), from
    the launch shape the library reports."""
    from prototype_sketch_attention_b200 import binding
    G, _, H, share = binding.forward_grid(k, d)
    Th = (T * share) >> 10 if H > 0 else 0
    if Th < 32 * H:  # helpers take work only when each gets a full 32-tile chunk
        Th = 0
    T1 = T - Th
    bounds = [g * T1 // G for g in range(1, G)]
    if Th > 0:
        bounds += [T1] + [T1 + b * Th // H for b in range(1, H)]
    return bounds, T1


def _boundary_users(w, k, d):
    """Users whose tiles straddle a bound between two tile ranges of the persistent
    forward grid: two clusters (or helper CTAs) accumulate parts of them, which the
    finalize sums. Longest first."""
    tiles = (np.diff(w.offsets.numpy()) + 127) // 128
    ts = np.concatenate([[0], np.cumsum(tiles)])
    bounds, _ = _range_bounds(int(ts[-1]), k, d)
    users = {int(np.searchsorted(ts, b, side="right") - 1) for b in bounds}
    users = [u for u in users if any(ts[u] < b < ts[u + 1] for b in bounds)]
    return sorted(users, key=lambda u: -int(tiles[u]))


def _helper_users(w, k, d):
    """The user cut at the first helper tile and the users whose tiles are all helper
    tiles (empty when the launch has no helper CTAs)."""
    tiles = (np.diff(w.offsets.numpy()) + 127) // 128
    ts = np.concatenate([[0], np.cumsum(tiles)])
    _, T1 = _range_bounds(int(ts[-1]), k, d)
    return [u for u in range(w.R) if tiles[u] > 0 and ts[u + 1] > T1]


def test_config3_sampled_users():
    """Shortest, median and longest user, and the longest user cut between clusters."""
    w = inputs.make_config(3)
    _, out = gpu_forward(w)
    _unit_mass_all_users(w, out)
    order = np.argsort(w.lengths)
    cut = _boundary_users(w, w.k, w.d)
    assert cut, "the batch spans several clusters"
    helper = _helper_users(w, w.k, w.d)
    assert helper, "the batch reaches the helper grid"
    users = {int(order[0]), int(order[len(order) // 2]), int(order[-1]), cut[0]}
    users |= set(helper[:1] + helper[-1:])
    check_forward(w, out, users=sorted(users))


def test_config5_forward_sampled_users():
    """The benchmark's headline batch, 40 users x 100K tokens, in the benchmark's launch:
    the first, a middle and the last user and two users cut between clusters, against
    the oracle; unit mass for every user."""
    w = inputs.make_config(5, with_grad=False)
    _, out = gpu_forward(w)
    _unit_mass_all_users(w, out)
    cut = _boundary_users(w, w.k, w.d)
    assert len(cut) >= 2, "the batch spans several clusters"
    helper = _helper_users(w, w.k, w.d)
    assert helper, "the batch reaches the helper grid"
    check_forward(w, out, users=sorted({0, 19, 39, cut[0], cut[-1]} | set(helper[:2])))


@pytest.mark.parametrize("k", [256, 512, 640, 768, 1024, 2048])
def test_config4_sampled_users(k):
    """The two shortest users, the median, the longest, the longest user cut between
    clusters, and (where the launch has helper CTAs) the users cut at the first helper
    tile and at the last."""
    w = inputs.make_config(4, k=k)
    _, out = gpu_forward(w)
    _unit_mass_all_users(w, out)
    order = np.argsort(w.lengths)
    cut = _boundary_users(w, k, w.d)
    assert cut, "the batch spans several clusters"
    helper = _helper_users(w, k, w.d)
    users = {int(order[0]), int(order[1]), int(order[150]), int(order[-1]), cut[0]}
    users |= set(helper[:1] + helper[-1:])
    check_forward(w, out, users=sorted(users))


def test_deterministic_bitwise():
    w = inputs.make_workload([5000, 123, 30000, 1], 128, 512, "bf16", seed=77)
    g, a = gpu_forward(w)
    from prototype_sketch_attention_b200 import binding
    b = binding.forward(g["X"], g["offsets"], g["P"], g["Wk"], g["Wv"])
    for key in ("sketch", "mass", "lse", "xsketch"):
        assert torch.equal(a[key], b[key]), key


def test_empty_batches():
    from prototype_sketch_attention_b200 import binding
    w = inputs.make_workload([0, 0], 128, 256, "bf16", seed=3)
    _, out = gpu_forward(w)
    assert not out["sketch"].any() and not out["mass"].any()
    w0 = inputs.make_workload([], 128, 256, "bf16", seed=3)
    g = {k: v.cuda() for k, v in dict(X=w0.X, offsets=w0.offsets, P=w0.P, Wk=w0.Wk, Wv=w0.Wv).items()}
    out0 = binding.forward(g["X"], g["offsets"], g["P"], g["Wk"], g["Wv"])
    assert out0["sketch"].shape == (0, 256, 128)


def test_bad_offsets_latched_on_device():
    from prototype_sketch_attention_b200 import binding
    w = inputs.make_workload([200, 300], 128, 256, "bf16", seed=4)
    g = {k: v.cuda() for k, v in dict(X=w.X, P=w.P, Wk=w.Wk, Wv=w.Wv).items()}
    bad = torch.tensor([0, 400, 300], dtype=torch.int64, device="cuda")  # decreasing
    out = binding.forward(g["X"], bad, g["P"], g["Wk"], g["Wv"])
    assert binding.device_status(out["_ws"]) == binding.SA_ERR_BAD_OFFSETS
    bad2 = torch.tensor([0, 200, 499], dtype=torch.int64, device="cuda")  # != n_total
    out = binding.forward(g["X"], bad2, g["P"], g["Wk"], g["Wv"])
    assert binding.device_status(out["_ws"]) == binding.SA_ERR_BAD_OFFSETS
    # the next good call clears the status and is correct
    _, ok = gpu_forward(w)
    check_forward(w, ok)


def test_bounded_wait_times_out_and_context_survives():
    """The bounded-wait routine gives up on a barrier nothing arrives on, latches
    SA_ERR_TIMEOUT, and the context stays usable."""
    from prototype_sketch_attention_b200 import binding
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert binding.sa_sketch_debug_wait_timeout(ws.data_ptr(), 2_000_000, s) == 0
    assert binding.sa_sketch_get_device_status(ws.data_ptr(), s) == binding.SA_ERR_TIMEOUT
    w = inputs.make_workload([300, 40], 128, 256, "bf16", seed=8)
    _, out = gpu_forward(w)
    check_forward(w, out)


@pytest.mark.parametrize("lengths,k", [
    ([3000, 0, 1500, 77, 9000, 1, 4096], 1024),
    ([700, 0, 300], 200),
    ([500, 600], 2),
])
def test_forward_from_host_matches_device_forward(lengths, k):
    # sa_sketch_forward_host: users cut into parts whose copies overlap the previous
    # part's forward, host buffers in and out; against the device forward and the oracle
    from prototype_sketch_attention_b200 import binding
    w = inputs.make_workload(lengths, 128, k, "bf16", seed=77 + k)
    g = {n: getattr(w, n).cuda() for n in ("X", "offsets", "P", "Wk", "Wv")}
    ref = binding.forward(g["X"], g["offsets"], g["P"], g["Wk"], g["Wv"])
    state = {}
    Xh, offh = w.X.pin_memory(), w.offsets.pin_memory()
    for call in range(2):  # the second call reuses the buffers and streams
        sk, ms = binding.forward_from_host(Xh, offh, g["P"], g["Wk"], g["Wv"], chunks=4,
                                           state=state)
        torch.cuda.current_stream().synchronize()
        assert binding.forward_from_host_status(state) == 0
        exp_s, exp_m = ref["sketch"].cpu().double(), ref["mass"].cpu().double()
        for u in range(w.R):
            assert rel_l2(sk[u].double().numpy(), exp_s[u].numpy()) <= 1e-5
            assert rel_l2(ms[u].double().numpy(), exp_m[u].numpy()) <= 1e-5
        if call == 0:
            check_forward(w, {"sketch": sk.clone(), "mass": ms.clone()})


def test_bf16_extreme_scores_take_the_shifted_path():
    # A few tokens point along one prototype with 10 times its norm (W_k = I): that
    # prototype's score is ~160 in log2 units and the others stay below ~50, so
    # sum_j 2^s overflows fp32 and each warp holding such a token redoes its 32 tokens
    # shifted by the row max. Their softmax is one-hot by a margin that bf16 rounding of
    # P' cannot move, so the bf16 tolerances still apply; the ordinary tokens of those
    # warps check the shifted path's normalisation. (Their own lse is not compared: a
    # score of 160 carries ~0.3 of bf16 rounding from P', beyond lse's 5e-2.)
    import dataclasses
    from parity_util import BF16_ABS
    w = inputs.make_workload([700, 450], 128, 256, "bf16", seed=91)
    X = w.X.float().clone()
    gen = torch.Generator().manual_seed(5)
    idx = torch.arange(3, int(w.offsets[-1]), 97)
    js = torch.randint(0, w.k, (len(idx),), generator=gen)
    X[idx] = 10.0 * w.P.float()[js]
    w2 = dataclasses.replace(w, X=X.to(torch.bfloat16), Wk=torch.eye(w.d).to(torch.bfloat16))
    _, out = gpu_forward(w2)
    ref = check_forward(w2, {k: v for k, v in out.items() if k != "lse"})
    lse = out["lse"].cpu().double().numpy()
    normal = np.ones(len(lse), dtype=bool)
    normal[idx.numpy()] = False
    assert np.abs(lse[normal] - ref["lse"][normal]).max() <= BF16_ABS
    assert np.abs(lse[~normal] - ref["lse"][~normal]).max() <= 1.0  # same dominant score


def test_headline_launch_has_helper_ctas():
    """k = 1024 on a B200: clusters of 8 leave SMs free, and helper CTAs take them (the
    parity cases above with k = 1024 therefore cover the helper kernel)."""
    from prototype_sketch_attention_b200 import binding
    G, C, H, share = binding.forward_grid(1024, 128)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert C == 8 and H == sms - G * C and H > 0 and 0 < share < 1024


@pytest.mark.parametrize("k", [1000, 1024])
def test_helper_ranges_with_empty_and_short_users(k):
    """A batch just large enough for the helper grid (each helper gets a full chunk),
    whose helper ranges hold empty users, users shorter than one tile, a user cut at the
    first helper tile and a long one; at k = 1000 the last prototype slice is partial.
    Every user the helpers touch is compared with the oracle."""
    lengths = [100000] * 10 + [0, 5, 0, 130, 2000, 0, 50000]
    w = inputs.make_workload(lengths, 128, k, "bf16", seed=91 + k)
    _, out = gpu_forward(w)
    _unit_mass_all_users(w, out)
    helper = _helper_users(w, k, w.d)
    assert helper and helper[0] <= 9, "the helper ranges start inside the tenth long user"
    users = set(range(helper[0], w.R))
    check_forward(w, out, users=sorted(users))
