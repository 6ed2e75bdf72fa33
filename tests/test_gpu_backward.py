"""GPU backward parity: dX, dP, dW_k, dW_v through the C ABI vs the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import check_grads, gpu_forward, nthreads, rel_l2
from prototype_sketch_attention_b200 import binding, inputs

pytestmark = pytest.mark.gpu


def _run(w, g, fwd, G, Gm=None):
    Gd = torch.from_numpy(G).float().cuda()
    Gmd = None if Gm is None else torch.from_numpy(Gm).float().cuda()
    out = binding.backward(g["X"], g["offsets"], g["P"], g["Wk"], g["Wv"], fwd, Gd, Gmd)
    st = binding.device_status(out["_ws"])
    assert st == 0, binding.sa_status_string(st)
    return {k: v.cpu().double().numpy() for k, v in out.items() if not k.startswith("_")}


@pytest.mark.parametrize("lengths,k,d,dtype,with_gm", [
    ([300, 0, 1037], 256, 128, "bf16", True),
    ([129, 5], 200, 64, "bf16", False),
    ([2048], 64, 64, "f32", True),
    ([77, 300], 100, 128, "f32", False),
])
def test_backward_small_full_compare(lengths, k, d, dtype, with_gm):
    w = inputs.make_workload(lengths, d, k, dtype, seed=90 + k, with_grad=True)
    g, fwd = gpu_forward(w)
    rng = np.random.default_rng(5)
    G = w.G.numpy().astype(np.float64)
    Gm = rng.standard_normal((w.R, k)) if with_gm else None
    got = _run(w, g, fwd, G, Gm)
    sub = w.to_f64()
    ref = oracle.backward(sub["X"], sub["offsets"], sub["P"], sub["Wk"], sub["Wv"], G, Gm,
                          nthreads=nthreads())
    check_grads(got, ref, fp32=(dtype == "f32"), offsets=sub["offsets"])


def test_config5_full_size_one_user_gradient():
    """Config 5 at full size (40 users x 100K, k=1024). dL/dsketch is non-zero for one
    user only, so the oracle needs that user alone: every other user's dX is exactly
    zero and dP, dW_k, dW_v are that user's contribution."""
    w = inputs.make_config(5)
    g, fwd = gpu_forward(w)
    u = 17
    G = np.zeros((w.R, w.k, w.d))
    G[u] = w.G[u].double().numpy()
    got = _run(w, g, fwd, G)
    off = w.offsets.numpy()
    sub = w.to_f64([u])
    ref = oracle.backward(sub["X"], sub["offsets"], sub["P"], sub["Wk"], sub["Wv"], G[u:u + 1],
                          nthreads=nthreads())
    dX_u = got["dX"][off[u]:off[u + 1]]
    rest = np.concatenate([got["dX"][:off[u]], got["dX"][off[u + 1]:]])
    assert not rest.any()
    check_grads({"dX": dX_u, "dP": got["dP"], "dWk": got["dWk"], "dWv": got["dWv"]}, ref, fp32=False,
                offsets=sub["offsets"])


@pytest.mark.parametrize("lengths,k,d", [([300, 0, 1037], 256, 128), ([129, 5], 384, 64)])
def test_backward_recomputes_lse_when_not_given(lengths, k, d):
    """The bf16 backward uses the forward's lse when passed and otherwise recomputes it
    (its own log-sum-exp pass). Both must match the oracle, and each other closely."""
    w = inputs.make_workload(lengths, d, k, "bf16", seed=31 + k, with_grad=True)
    g, fwd = gpu_forward(w)
    G = w.G.numpy().astype(np.float64)
    with_lse = _run(w, g, fwd, G)
    no_lse = {key: v for key, v in fwd.items() if key != "lse"}
    without = _run(w, g, no_lse, G)
    sub = w.to_f64()
    ref = oracle.backward(sub["X"], sub["offsets"], sub["P"], sub["Wk"], sub["Wv"], G,
                          nthreads=nthreads())
    check_grads(with_lse, ref, fp32=False, offsets=sub["offsets"])
    check_grads(without, ref, fp32=False, offsets=sub["offsets"])
    for key in ("dX", "dP", "dWk", "dWv"):
        assert rel_l2(without[key], with_lse[key]) <= 2e-3, key


def test_backward_bf16_k_not_multiple_of_128():
    """k = 200: the last 128-prototype tile is partly padding, which every epilogue masks."""
    w = inputs.make_workload([700, 260], 128, 200, "bf16", seed=77, with_grad=True)
    g, fwd = gpu_forward(w)
    G = w.G.numpy().astype(np.float64)
    got = _run(w, g, fwd, G)
    sub = w.to_f64()
    ref = oracle.backward(sub["X"], sub["offsets"], sub["P"], sub["Wk"], sub["Wv"], G,
                          nthreads=nthreads())
    check_grads(got, ref, fp32=False, offsets=sub["offsets"])
