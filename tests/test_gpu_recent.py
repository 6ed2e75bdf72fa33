"""GPU parity of the recent branch of STCA: each user's candidates attend over the user's
last min(n_u, L) history rows, read in place from the history X through per-user key
ranges (sa_stca_recent_ranges + sa_stca_keys_forward / sa_stca_keys_backward), against
the fp64 oracle's ragged-key cross attention on the same seeded inputs. The oracle gets
the selected rows themselves (oracle.recent_suffix). bf16 tolerance as for the other
bf16 paths: per user, relative L2 <= 1e-2 and max |error| <= 5e-2 on the output, max
|error| <= 5e-2 on lse; gradients: relative L2 <= 1e-2 and max |error| <= 5e-2 of the
largest reference entry."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import BF16_ABS, BF16_REL, nthreads, rel_l2
from prototype_sketch_attention_b200 import inputs

pytestmark = pytest.mark.gpu


def _dev():
    return torch.device("cuda")


def _ranges(rw):
    from prototype_sketch_attention_b200 import binding
    kb, ke = binding.recent_ranges(rw.offsets.to(_dev()), rw.L)
    return kb, ke


def _forward(rw, kb=None, ke=None, Kx=None):
    from prototype_sketch_attention_b200 import binding
    dev = _dev()
    if kb is None:
        kb, ke = _ranges(rw)
    Kx = rw.X if Kx is None else Kx
    out = binding.stca_keys_forward(rw.Q.to(dev), rw.cand_offsets.to(dev), Kx.to(dev), kb, ke,
                                    rw.Wq.to(dev), rw.WK.to(dev), rw.WV.to(dev))
    st = binding.device_status(out["_ws"])
    assert st == 0, binding.sa_status_string(st)
    return out["out"].cpu().double().numpy(), out["lse"].cpu().double().numpy()


def _oracle_inputs(rw):
    Kx, koff = oracle.recent_suffix(rw.X.double().numpy(), rw.offsets.numpy(), rw.L)
    return dict(Q=rw.Q.double().numpy(), cand_offsets=rw.cand_offsets.numpy(), Kx=Kx,
                key_offsets=koff, Wq=rw.Wq.double().numpy(), WK=rw.WK.double().numpy(),
                WV=rw.WV.double().numpy())


def _check_forward(coff, got, lse, ref, users=None):
    users = range(len(coff) - 1) if users is None else users
    for u in users:
        a, b = int(coff[u]), int(coff[u + 1])
        if a == b:
            continue
        r = ref["out"][a:b]
        if not np.any(r):  # a user without key rows: out = 0, lse = -inf
            assert not np.any(got[a:b]), (u, "out of a user without keys")
            assert np.all(np.isneginf(lse[a:b])) and np.all(np.isneginf(ref["lse"][a:b])), u
            continue
        e = rel_l2(got[a:b], r)
        assert e <= BF16_REL, (u, "out", e)
        assert np.abs(got[a:b] - r).max() <= BF16_ABS, (u, "out max-abs")
        assert np.abs(lse[a:b] - ref["lse"][a:b]).max() <= BF16_ABS, (u, "lse")


@pytest.mark.parametrize("lengths,counts,d,L", [
    ([300, 5, 0, 1000], [40, 3, 2, 129], 128, 256),       # short, empty and long histories
    ([2000, 130], [1, 300], 64, 1000),
    ([129, 128, 127, 1], [128, 129, 1, 7], 128, 10000),    # ragged key and candidate tiles
    ([5000, 0, 777], [0, 5, 255], 128, 640),               # a user without candidates
])
def test_recent_branch_forward_small_full_compare(lengths, counts, d, L):
    rw = inputs.make_recent_workload(lengths, counts, d, L, seed=900 + d + L + len(lengths))
    got, lse = _forward(rw)
    ref = oracle.stca_forward_keys(**_oracle_inputs(rw), nthreads=nthreads())
    _check_forward(rw.cand_offsets.numpy(), got, lse, ref)


def test_recent_ranges_select_the_last_L_rows():
    rw = inputs.make_recent_workload([0, 3, 10, 25], [1, 1, 1, 1], 64, 10, seed=901)
    kb, ke = _ranges(rw)
    off = rw.offsets.numpy()
    assert kb.cpu().tolist() == [max(off[u], off[u + 1] - 10) for u in range(4)]
    assert ke.cpu().tolist() == off[1:].tolist()


def test_recent_branch_forward_growing_scores():
    """Key rows whose scale grows along each history (0.25 to 2, Q scaled by 2): every
    later key tile holds larger scores, so the running maximum is raised several times
    along the tiles (by more than its margin of 8 in log2 units) and the accumulated
    output rescaled each time. Scores stay within about 15 natural units, where bf16
    inputs meet the tolerance (at 30 units the rounding of Q Wq WK^T alone moves the
    weights by several percent)."""
    rw = inputs.make_recent_workload([6000, 3000, 900], [64, 200, 9], 128, 5000, seed=902,
                                     q_std=2.0)
    off = rw.offsets.numpy()
    ramp = torch.cat([torch.linspace(0.25, 2.0, int(off[u + 1] - off[u])) for u in range(rw.R)])
    rw.X = (rw.X.float() * ramp[:, None]).to(torch.bfloat16)
    got, lse = _forward(rw)
    ref = oracle.stca_forward_keys(**_oracle_inputs(rw), nthreads=nthreads())
    _check_forward(rw.cand_offsets.numpy(), got, lse, ref)


def test_recent_branch_forward_ten_thousand_keys():
    """The pages' recent 10K over histories of 1K-100K rows: eight users, 1..300
    candidates each, every user compared in full."""
    gen = torch.Generator().manual_seed(903)
    lengths = inputs.draw_lengths("loguniform:1000:100000", 8, gen)
    counts = torch.randint(1, 301, (8,), generator=gen).numpy()
    rw = inputs.make_recent_workload(lengths, counts, 128, 10000, seed=904)
    got, lse = _forward(rw)
    ref = oracle.stca_forward_keys(**_oracle_inputs(rw), nthreads=nthreads())
    _check_forward(rw.cand_offsets.numpy(), got, lse, ref)


def test_recent_branch_forward_forty_users_sampled():
    """R = 40 users of 100K rows, 300 candidates each, over the recent 10K (the launch the
    benchmark times); three users' candidates are compared in full with the oracle."""
    rw = inputs.make_recent_workload([100000] * 40, [300] * 40, 128, 10000, seed=905)
    got, lse = _forward(rw)
    coff = rw.cand_offsets.numpy()
    for u in (0, 17, 39):
        sub = inputs.RecentWorkload(
            R=1, d=128, L=10000, lengths=np.array([100000]),
            offsets=torch.tensor([0, 100000]), X=rw.X[int(rw.offsets[u]):int(rw.offsets[u + 1])],
            counts=np.array([300]), cand_offsets=torch.tensor([0, 300]),
            Q=rw.Q[int(coff[u]):int(coff[u + 1])], Wq=rw.Wq, WK=rw.WK, WV=rw.WV)
        ref = oracle.stca_forward_keys(**_oracle_inputs(sub), nthreads=nthreads())
        a = int(coff[u])
        _check_forward(np.array([0, 300]), got[a:a + 300], lse[a:a + 300], ref)


def test_overlapping_key_ranges_forward_and_backward():
    """Explicit ranges over a shared key matrix that overlap: each user reads its own
    range, and dKx sums the users' gradients on the shared rows."""
    from prototype_sketch_attention_b200 import binding
    gen = torch.Generator().manual_seed(906)
    d = 128
    Kx = torch.randn(700, d, generator=gen).to(torch.bfloat16)
    rw = inputs.make_recent_workload([1, 1, 1], [30, 150, 7], d, 1, seed=907)
    ranges = [(0, 300), (100, 500), (450, 700)]
    kb = torch.tensor([r[0] for r in ranges], dtype=torch.int64, device=_dev())
    ke = torch.tensor([r[1] for r in ranges], dtype=torch.int64, device=_dev())
    got, lse = _forward(rw, kb, ke, Kx)
    rows = np.concatenate([np.arange(a, b) for a, b in ranges])
    koff = np.concatenate([[0], np.cumsum([b - a for a, b in ranges])]).astype(np.int64)
    f = dict(Q=rw.Q.double().numpy(), cand_offsets=rw.cand_offsets.numpy(),
             Kx=Kx.double().numpy()[rows], key_offsets=koff, Wq=rw.Wq.double().numpy(),
             WK=rw.WK.double().numpy(), WV=rw.WV.double().numpy())
    ref = oracle.stca_forward_keys(**f, nthreads=nthreads())
    _check_forward(rw.cand_offsets.numpy(), got, lse, ref)
    G = torch.randn(187, d, generator=gen)
    dev = _dev()
    out = binding.stca_keys_backward(rw.Q.to(dev), rw.cand_offsets.to(dev), Kx.to(dev), kb, ke,
                                     rw.Wq.to(dev), rw.WK.to(dev), rw.WV.to(dev), G.to(dev))
    assert binding.device_status(out["_ws"]) == 0
    rb = oracle.stca_backward_keys(**f, dout=G.double().numpy(), nthreads=nthreads())
    dK = np.zeros((700, d))
    np.add.at(dK, rows, rb["dKx"])
    rb["dKx"] = dK
    _check_grads({k: out[k].cpu().double().numpy() for k in rb}, rb)


def test_bad_key_ranges_are_reported():
    from prototype_sketch_attention_b200 import binding
    rw = inputs.make_recent_workload([100, 50], [4, 4], 64, 100, seed=908)
    dev = _dev()
    for lo, hi in (((0, 95), (100, 90)), ((-1, 100), (100, 150)), ((0, 100), (100, 151))):
        kb = torch.tensor(lo, dtype=torch.int64, device=dev)
        ke = torch.tensor(hi, dtype=torch.int64, device=dev)
        out = binding.stca_keys_forward(rw.Q.to(dev), rw.cand_offsets.to(dev), rw.X.to(dev), kb,
                                        ke, rw.Wq.to(dev), rw.WK.to(dev), rw.WV.to(dev))
        assert binding.device_status(out["_ws"]) == binding.SA_ERR_BAD_OFFSETS, (lo, hi)


def test_no_candidates_and_no_keys():
    rw = inputs.make_recent_workload([0, 0], [0, 0], 128, 100, seed=909)
    got, lse = _forward(rw)
    assert got.shape == (0, 128) and lse.shape == (0,)
    rw = inputs.make_recent_workload([0, 0], [3, 1], 128, 100, seed=910)
    got, lse = _forward(rw)
    assert not got.any() and np.all(np.isneginf(lse))


def _check_grads(got, ref):
    for key, r in ref.items():
        g = got[key]
        e = rel_l2(g, r)
        assert e <= BF16_REL, (key, e)
        assert np.abs(g - r).max() <= BF16_ABS * max(np.abs(r).max(), 1e-30), (key, "max-abs")


@pytest.mark.parametrize("lengths,counts,d,L", [
    ([300, 5, 0, 1000], [40, 3, 2, 129], 128, 256),
    ([2000, 130], [1, 300], 64, 1000),
    ([12000, 700, 129], [100, 17, 128], 128, 10000),
])
def test_recent_branch_backward_full_compare(lengths, counts, d, L):
    from prototype_sketch_attention_b200 import binding
    rw = inputs.make_recent_workload(lengths, counts, d, L, seed=920 + d + L)
    n_cand = int(rw.cand_offsets[-1])
    G = torch.randn(n_cand, d, generator=torch.Generator().manual_seed(921))
    dev = _dev()
    kb, ke = _ranges(rw)
    out = binding.stca_keys_backward(rw.Q.to(dev), rw.cand_offsets.to(dev), rw.X.to(dev), kb, ke,
                                     rw.Wq.to(dev), rw.WK.to(dev), rw.WV.to(dev), G.to(dev))
    assert binding.device_status(out["_ws"]) == 0
    f = _oracle_inputs(rw)
    ref = oracle.stca_backward_keys(**f, dout=G.double().numpy(), nthreads=nthreads())
    # the GPU's dKx covers every history row: the suffix rows get the oracle's, others 0
    dX = np.zeros((int(rw.offsets[-1]), d))
    dX[rw.suffix_rows()] = ref["dKx"]
    ref["dKx"] = dX
    got = {k: out[k].cpu().double().numpy() for k in ref}
    _check_grads(got, ref)
    coff = rw.cand_offsets.numpy()
    for u in range(rw.R):  # per user on dQ
        a, b = int(coff[u]), int(coff[u + 1])
        if a < b and np.any(ref["dQ"][a:b]):
            assert rel_l2(got["dQ"][a:b], ref["dQ"][a:b]) <= BF16_REL, u


def test_backward_accumulates_into_a_given_history_gradient():
    """With dKx given, the key rows' gradient is added into it: the result equals the
    buffer's previous contents plus the overwriting call's dKx, bitwise, since with one
    candidate tile per user every row receives exactly one addition in both calls."""
    from prototype_sketch_attention_b200 import binding
    rw = inputs.make_recent_workload([3000, 500, 0], [64, 7, 3], 128, 1000, seed=930)
    G = torch.randn(74, 128, generator=torch.Generator().manual_seed(931))
    dev = _dev()
    kb, ke = _ranges(rw)
    args = (rw.Q.to(dev), rw.cand_offsets.to(dev), rw.X.to(dev), kb, ke, rw.Wq.to(dev),
            rw.WK.to(dev), rw.WV.to(dev), G.to(dev))
    plain = binding.stca_keys_backward(*args)
    base = torch.randn(3500, 128, generator=torch.Generator().manual_seed(932)).to(dev)
    acc = binding.stca_keys_backward(*args, dKx=base.clone())
    assert binding.device_status(acc["_ws"]) == 0
    expect = base + plain["dKx"]
    assert torch.equal(acc["dKx"], expect)
    for key in ("dQ", "dWq", "dWK", "dWV"):
        assert torch.equal(acc[key], plain[key]), key
