"""Sharded forward/backward through the CUDA library on one GPU (world_size 1), with
users cut into parts: exercises sa_sketch_combine and the backward with a part's own
xsketch against the fp64 oracle on the whole batch."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import BF16_ABS, BF16_REL, FP32_BWD, FP32_FWD, check_grads, nthreads, rel_l2
from prototype_sketch_attention_b200 import binding, inputs
from prototype_sketch_attention_b200.sharding import plan_shards, sharded_backward, sharded_forward

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("lengths,k,d,dtype,cap", [
    ([3000, 0, 517, 1300], 256, 128, "bf16", 700),
    ([2049, 33], 64, 64, "f32", 500),
])
def test_sharded_cut_users_match_whole_batch(lengths, k, d, dtype, cap):
    w = inputs.make_workload(lengths, d, k, dtype, seed=77, with_grad=True)
    f = w.to_f64()
    plan = plan_shards(lengths, 1, max_part_tokens=cap)
    assert plan.split_users(), "the case must cut some user"
    dev = torch.device("cuda")
    rows = torch.from_numpy(plan.local_rows(0)).to(dev)
    X = w.X.to(dev)[rows].contiguous()
    P, Wk, Wv = w.P.to(dev), w.Wk.to(dev), w.Wv.to(dev)
    fwd = sharded_forward(plan, 0, X, P, Wk, Wv)
    assert fwd["users"] == list(range(len(lengths)))
    ref = oracle.forward(f["X"], f["offsets"], f["P"], f["Wk"], f["Wv"], nthreads=nthreads())
    fp32 = dtype == "f32"
    for u in range(len(lengths)):
        if lengths[u] == 0:
            assert not fwd["sketch"][u].any() and not fwd["mass"][u].any()
            continue
        got = fwd["sketch"][u].double().cpu().numpy()
        e = rel_l2(got, ref["sketch"][u])
        assert e <= (FP32_FWD if fp32 else BF16_REL), (u, e)
        if not fp32:
            assert np.abs(got - ref["sketch"][u]).max() <= BF16_ABS
        assert rel_l2(fwd["mass"][u].double().cpu().numpy(), ref["mass"][u]) <= (FP32_FWD if fp32 else BF16_REL)
    G = w.G.to(dev).float()
    Gm = torch.from_numpy(np.random.default_rng(3).standard_normal((len(lengths), k))).float().to(dev)
    b = sharded_backward(plan, 0, X, P, Wk, Wv, fwd, G, Gm)
    dX = torch.empty_like(b["dX"])
    dX[rows] = b["dX"]
    got = {"dX": dX.double().cpu().numpy(), "dP": b["dP"].double().cpu().numpy(),
           "dWk": b["dWk"].double().cpu().numpy(), "dWv": b["dWv"].double().cpu().numpy()}
    refb = oracle.backward(f["X"], f["offsets"], f["P"], f["Wk"], f["Wv"],
                           w.G.numpy().astype(np.float64), Gm.double().cpu().numpy(), nthreads=nthreads())
    check_grads(got, refb, fp32=fp32)


def test_combine_matches_forward_epilogue():
    # summed halves of a user through sa_sketch_combine == the user's own forward sketch
    w = inputs.make_workload([4000], 128, 512, "bf16", seed=5)
    dev = torch.device("cuda")
    X, P, Wk, Wv = w.X.to(dev), w.P.to(dev), w.Wk.to(dev), w.Wv.to(dev)
    whole = binding.forward(X, torch.tensor([0, 4000], device=dev), P, Wk, Wv)
    halves = binding.forward(X, torch.tensor([0, 1700, 4000], device=dev), P, Wk, Wv)
    U = halves["xsketch"].sum(0, keepdim=True).contiguous()
    M = halves["mass"].sum(0, keepdim=True).contiguous()
    S = binding.combine(U, M, Wv)
    assert rel_l2(S.cpu().numpy(), whole["sketch"].cpu().numpy()) <= 1e-5
    assert rel_l2(M.cpu().numpy(), whole["mass"].cpu().numpy()) <= 1e-5
    with pytest.raises(binding.SketchAttentionError):
        binding.combine(U[:, :, :100].contiguous(), M, Wv)  # d = 100 is not supported
