"""The seeded input generator: shapes, determinism and the pages' workload shapes."""
import numpy as np

from prototype_sketch_attention_b200 import inputs


def test_config_shapes_small():
    w = inputs.make_config(1)
    assert (w.R, w.d, w.k, w.dtype) == (1, 64, 64, "f32")
    assert w.n_total == 2048 and w.X.shape == (2048, 64)


def test_deterministic():
    a = inputs.make_workload([5, 7], 8, 4, "bf16", seed=3, with_grad=True)
    b = inputs.make_workload([5, 7], 8, 4, "bf16", seed=3, with_grad=True)
    for key in ("X", "P", "Wk", "Wv", "G"):
        assert (getattr(a, key).float() == getattr(b, key).float()).all()


def test_length_rules():
    import torch
    g = torch.Generator().manual_seed(1)
    u = inputs.draw_lengths("uniform:10000:100000", 400, g)
    assert u.min() >= 10000 and u.max() <= 100000
    lg = inputs.draw_lengths("loguniform:1000:100000", 2000, g)
    assert lg.min() >= 1000 and lg.max() <= 100000
    # log-uniform: the median sits near the geometric mean 10^4
    assert 6000 < np.median(lg) < 16000


def test_to_f64_subset_matches_rows():
    w = inputs.make_workload([3, 0, 4], 8, 4, "bf16", seed=5)
    sub = w.to_f64(users=[2])
    assert list(sub["offsets"]) == [0, 4]
    assert np.array_equal(sub["X"], w.X[3:7].double().numpy())
