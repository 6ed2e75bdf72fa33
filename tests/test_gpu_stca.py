"""GPU parity of the candidate-to-sketch cross attention (sa_stca_forward) against the
fp64 oracle, on the same seeded inputs. bf16 tolerance as for the Sketch Attention
forward: per user, relative L2 <= 1e-2 and max |error| <= 5e-2 on the output; max
|error| <= 5e-2 on lse."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import BF16_ABS, BF16_REL, gpu_forward, nthreads, rel_l2
from prototype_sketch_attention_b200 import inputs

pytestmark = pytest.mark.gpu


def _run(cw):
    from prototype_sketch_attention_b200 import binding
    dev = torch.device("cuda")
    out = binding.stca_forward(cw.Q.to(dev), cw.cand_offsets.to(dev), cw.S.to(dev),
                               cw.Wq.to(dev), cw.WK.to(dev), cw.WV.to(dev))
    st = binding.device_status(out["_ws"])
    assert st == 0, binding.sa_status_string(st)
    return out["out"].cpu().double().numpy(), out["lse"].cpu().double().numpy()


def _check(cw, got, lse):
    f = cw.to_f64()
    ref = oracle.stca_forward(f["Q"], f["cand_offsets"], f["S"], f["Wq"], f["WK"], f["WV"],
                              nthreads=nthreads())
    off = f["cand_offsets"]
    for u in range(cw.R):
        a, b = int(off[u]), int(off[u + 1])
        if a == b:
            continue
        e = rel_l2(got[a:b], ref["out"][a:b])
        assert e <= BF16_REL, (u, "out", e)
        assert np.abs(got[a:b] - ref["out"][a:b]).max() <= BF16_ABS, (u, "out max-abs")
    if len(lse):
        assert np.abs(lse - ref["lse"]).max() <= BF16_ABS, ("lse", np.abs(lse - ref["lse"]).max())


@pytest.mark.parametrize("counts,k,d", [
    ([300, 0, 1, 129], 1024, 128),
    ([5, 77], 200, 64),
    ([130], 64, 128),
    ([1, 2, 3, 255, 256, 257], 2048, 128),
    ([40], 384, 64),
])
def test_cross_attention_small_full_compare(counts, k, d):
    cw = inputs.make_cross_workload(counts, k, d, seed=500 + k + d + len(counts))
    got, lse = _run(cw)
    _check(cw, got, lse)


def test_cross_attention_forty_users_a_few_hundred_candidates():
    """40 users, 1..300 candidates each, over k = 1024 rows of d = 128."""
    gen = torch.Generator().manual_seed(41)
    counts = torch.randint(1, 301, (40,), generator=gen).numpy()
    cw = inputs.make_cross_workload(counts, 1024, 128, seed=42)
    got, lse = _run(cw)
    _check(cw, got, lse)


def test_cross_attention_over_the_forward_sketch():
    """The chain as it runs: Sketch Attention's sketch (GPU) is the cross attention's
    input; the oracle reads that same sketch."""
    w = inputs.make_workload([3000, 700, 0, 1500], 128, 512, "bf16", seed=43)
    _, fwd = gpu_forward(w)
    S = fwd["sketch"].cpu()
    cw = inputs.make_cross_workload([50, 10, 7, 300], 512, 128, seed=44, S=S)
    got, lse = _run(cw)
    _check(cw, got, lse)


def test_cross_attention_without_candidates():
    cw = inputs.make_cross_workload([0, 0], 256, 128, seed=45)
    got, lse = _run(cw)
    assert got.shape == (0, 128) and lse.shape == (0,)


def _check_grads(got, ref):
    for key, r in ref.items():
        g = got[key]
        e = rel_l2(g, r)
        assert e <= BF16_REL, (key, e)
        assert np.abs(g - r).max() <= BF16_ABS * max(np.abs(r).max(), 1e-30), (key, "max-abs")


@pytest.mark.parametrize("counts,k,d", [([300, 0, 1, 129], 1024, 128), ([5, 77], 200, 64),
                                        ([1, 2, 3, 255, 256, 257], 2048, 128)])
def test_cross_attention_backward_small_full_compare(counts, k, d):
    from prototype_sketch_attention_b200 import binding
    cw = inputs.make_cross_workload(counts, k, d, seed=700 + k + d)
    G = torch.randn(int(cw.cand_offsets[-1]), d, generator=torch.Generator().manual_seed(701))
    dev = torch.device("cuda")
    out = binding.stca_backward(cw.Q.to(dev), cw.cand_offsets.to(dev), cw.S.to(dev),
                                cw.Wq.to(dev), cw.WK.to(dev), cw.WV.to(dev), G.to(dev))
    assert binding.device_status(out["_ws"]) == 0
    got = {key: out[key].cpu().double().numpy() for key in ("dQ", "dS", "dWq", "dWK", "dWV")}
    f = cw.to_f64()
    ref = oracle.stca_backward(f["Q"], f["cand_offsets"], f["S"], f["Wq"], f["WK"], f["WV"],
                               G.double().numpy(), nthreads=nthreads())
    _check_grads(got, ref)
    assert not got["dS"][[i for i, c in enumerate(counts) if c == 0]].any()


def test_history_to_candidates_chain_gradient():
    """Sketch Attention, then the cross attention over its sketch, then the cross
    attention's dS fed back to sa_sketch_backward as dL/dsketch: the chain that carries the
    ranking loss's gradient to the history. Each GPU stage is compared with its oracle on
    the inputs that stage actually received (the cross attention on the GPU's sketch, the
    Sketch Attention backward on the GPU's dS), each at the bf16 tolerance; comparing the
    GPU chain with an all-oracle chain would add up three stages' bf16 rounding against
    one stage's bound."""
    from prototype_sketch_attention_b200 import binding
    w = inputs.make_workload([2000, 700, 1500], 128, 256, "bf16", seed=71)
    g, fwd = gpu_forward(w)
    cw = inputs.make_cross_workload([40, 9, 120], 256, 128, seed=72, S=fwd["sketch"].cpu())
    G = torch.randn(169, 128, generator=torch.Generator().manual_seed(73))
    dev = torch.device("cuda")
    cb = binding.stca_backward(cw.Q.to(dev), cw.cand_offsets.to(dev), fwd["sketch"],
                               cw.Wq.to(dev), cw.WK.to(dev), cw.WV.to(dev), G.to(dev))
    sb = binding.backward(g["X"], g["offsets"], g["P"], g["Wk"], g["Wv"], fwd, cb["dS"])
    assert binding.device_status(sb["_ws"]) == 0
    sub = w.to_f64()
    f = cw.to_f64()  # its sketch S is the GPU forward's
    ref_c = oracle.stca_backward(f["Q"], f["cand_offsets"], f["S"], f["Wq"], f["WK"],
                                 f["WV"], G.double().numpy(), nthreads=nthreads())
    _check_grads({key: cb[key].cpu().double().numpy() for key in ref_c}, ref_c)
    ref = oracle.backward(sub["X"], sub["offsets"], sub["P"], sub["Wk"], sub["Wv"],
                          cb["dS"].cpu().double().numpy(), nthreads=nthreads())
    got = {key: sb[key].cpu().double().numpy() for key in ("dX", "dP", "dWk", "dWv")}
    _check_grads(got, ref)
