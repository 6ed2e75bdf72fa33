"""The C-ABI calls allocate nothing, never synchronise and enqueue only kernels and
memsets on the caller's stream, so a caller can capture them into a CUDA graph and replay
them (a serving loop with fixed shapes pays the launch sequence once). These tests capture
each call with torch.cuda.CUDAGraph on fresh inputs, replay it on new input values written
into the same buffers, and compare the replay with an eager call on those values, bitwise."""
import pytest
import torch

from prototype_sketch_attention_b200 import binding, inputs

pytestmark = pytest.mark.gpu


def _capture(fn):
    """Warm fn up on a side stream (the first call fills host-side caches), then capture."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        out = fn()
    return g, out


def test_sketch_forward_replays_from_a_graph():
    dev = torch.device("cuda")
    w = inputs.make_workload([3000, 0, 700, 5000], 128, 1024, "bf16", seed=61)
    X, off = w.X.to(dev), w.offsets.to(dev)
    P, Wk, Wv = w.P.to(dev), w.Wk.to(dev), w.Wv.to(dev)
    ws = binding.forward(X, off, P, Wk, Wv)["_ws"]
    g, out = _capture(lambda: binding.forward(X, off, P, Wk, Wv, ws=ws))
    w2 = inputs.make_workload([3000, 0, 700, 5000], 128, 1024, "bf16", seed=62)
    X.copy_(w2.X.to(dev))
    g.replay()
    torch.cuda.synchronize()
    assert binding.device_status(ws) == 0
    ref = binding.forward(X, off, P, Wk, Wv)
    for key in ("sketch", "mass"):
        assert torch.equal(out[key], ref[key]), key


def test_cross_attention_calls_replay_from_a_graph():
    dev = torch.device("cuda")
    rw = inputs.make_recent_workload([20000, 900, 0], [300, 40, 5], 128, 10000, seed=63)
    kb, ke = binding.recent_ranges(rw.offsets.to(dev), 10000)
    args = [rw.Q.to(dev), rw.cand_offsets.to(dev), rw.X.to(dev), kb, ke, rw.Wq.to(dev),
            rw.WK.to(dev), rw.WV.to(dev)]
    G = torch.randn(345, 128, generator=torch.Generator().manual_seed(64)).to(dev)
    fws = binding.stca_keys_forward(*args)["_ws"]
    bws = binding.stca_keys_backward(*args, G)["_ws"]
    gf, fout = _capture(lambda: binding.stca_keys_forward(*args, ws=fws))
    gb, bout = _capture(lambda: binding.stca_keys_backward(*args, G, ws=bws))
    rw2 = inputs.make_recent_workload([20000, 900, 0], [300, 40, 5], 128, 10000, seed=65)
    args[0].copy_(rw2.Q.to(dev))
    args[2].copy_(rw2.X.to(dev))
    G.copy_(torch.randn(345, 128, generator=torch.Generator().manual_seed(66)).to(dev))
    gf.replay()
    gb.replay()
    torch.cuda.synchronize()
    assert binding.device_status(fws) == 0 and binding.device_status(bws) == 0
    ref_f = binding.stca_keys_forward(*args)
    ref_b = binding.stca_keys_backward(*args, G)
    for key in ("out", "lse"):
        assert torch.equal(fout[key], ref_f[key]), key
    for key in ("dQ", "dWq", "dWK", "dWV"):
        assert torch.equal(bout[key], ref_b[key]), key
    # dKx sums reductions in an order that is not fixed: equal to rounding
    assert torch.allclose(bout["dKx"], ref_b["dKx"], rtol=1e-5, atol=1e-6)


def test_sketch_branch_calls_replay_from_a_graph():
    """The sketch branch, with the candidate offsets' host copy passed in (no
    device-to-host copy inside the call)."""
    dev = torch.device("cuda")
    cw = inputs.make_cross_workload([300, 0, 40, 129], 1024, 128, seed=67)
    coff_h = cw.cand_offsets.clone()
    args = [cw.Q.to(dev), cw.cand_offsets.to(dev), cw.S.to(dev), cw.Wq.to(dev), cw.WK.to(dev),
            cw.WV.to(dev)]
    G = torch.randn(469, 128, generator=torch.Generator().manual_seed(68)).to(dev)
    fws = binding.stca_forward(*args)["_ws"]
    bws = binding.stca_backward(*args, G, cand_offsets_host=coff_h)["_ws"]
    gf, fout = _capture(lambda: binding.stca_forward(*args, ws=fws))
    gb, bout = _capture(lambda: binding.stca_backward(*args, G, cand_offsets_host=coff_h, ws=bws))
    cw2 = inputs.make_cross_workload([300, 0, 40, 129], 1024, 128, seed=69)
    args[0].copy_(cw2.Q.to(dev))
    args[2].copy_(cw2.S.to(dev))
    gf.replay()
    gb.replay()
    torch.cuda.synchronize()
    assert binding.device_status(fws) == 0 and binding.device_status(bws) == 0
    ref_f = binding.stca_forward(*args)
    ref_b = binding.stca_backward(*args, G)
    for key in ("out", "lse"):
        assert torch.equal(fout[key], ref_f[key]), key
    for key in ("dQ", "dWq", "dWK", "dWV"):
        assert torch.equal(bout[key], ref_b[key]), key
    assert torch.allclose(bout["dS"], ref_b["dS"], rtol=1e-5, atol=1e-6)


def test_forward_with_the_helper_grid_replays_from_a_graph():
    """A batch large enough for the helper grid: the helper launch (programmatic stream
    serialization behind the clustered grid) is captured with the rest and replayed."""
    dev = torch.device("cuda")
    lengths = [100000] * 10 + [50000]
    from prototype_sketch_attention_b200 import binding as b
    G, C, H, share = b.forward_grid(1024, 128)
    T = sum((n + 127) // 128 for n in lengths)
    assert H > 0 and (T * share) >> 10 >= 32 * H, "the batch reaches the helper grid"
    w = inputs.make_workload(lengths, 128, 1024, "bf16", seed=71)
    X, off = w.X.to(dev), w.offsets.to(dev)
    P, Wk, Wv = w.P.to(dev), w.Wk.to(dev), w.Wv.to(dev)
    ws = binding.forward(X, off, P, Wk, Wv)["_ws"]
    g, out = _capture(lambda: binding.forward(X, off, P, Wk, Wv, ws=ws))
    X.copy_(inputs.make_workload(lengths, 128, 1024, "bf16", seed=72).X.to(dev))
    g.replay()
    torch.cuda.synchronize()
    assert binding.device_status(ws) == 0
    ref = binding.forward(X, off, P, Wk, Wv)
    for key in ("sketch", "mass", "lse"):
        assert torch.equal(out[key], ref[key]), key
