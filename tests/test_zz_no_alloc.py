"""The forward entry point that allocates nothing (sa_sketch_forward_noalloc).

It serves callers that cannot allocate device memory: its scratch space is one device
array that the library reserves per GPU. These tests call it through the C ABI and
check it against the regular sa_sketch_forward on the same inputs, twice in a row (the
second call reuses the scratch the first one left behind). The file sorts last so
that a run stopping at the first failure has run every other test before it.
"""
import ctypes

import numpy as np
import pytest
import torch

from parity_util import BF16_ABS, BF16_REL, rel_l2
from prototype_sketch_attention_b200 import binding, inputs

pytestmark = pytest.mark.gpu


def _noalloc(g, R, n_total, d, k, out):
    st = ctypes.c_int(-1)
    rc = binding.sa_sketch_forward_noalloc(
        g["X"].data_ptr(), g["offsets"].data_ptr(), R, n_total, d, g["P"].data_ptr(), k,
        g["Wk"].data_ptr(), g["Wv"].data_ptr(), binding.SA_BF16, out["sketch"].data_ptr(),
        out["mass"].data_ptr(), out["lse"].data_ptr(), out["xsketch"].data_ptr(),
        ctypes.addressof(st), torch.cuda.current_stream().cuda_stream)
    return rc, st.value


def test_noalloc_matches_forward_on_two_calls_in_a_row():
    w = inputs.make_workload([3000, 0, 1500, 77, 9000], 128, 1024, "bf16", seed=4242)
    g = {n: getattr(w, n).cuda() for n in ("X", "offsets", "P", "Wk", "Wv")}
    ref = binding.forward(g["X"], g["offsets"], g["P"], g["Wk"], g["Wv"])
    assert binding.device_status(ref["_ws"]) == 0
    R, n_total, d, k = w.R, w.n_total, w.d, w.k
    for call in range(2):
        out = {"sketch": torch.full((R, k, d), float("nan"), device="cuda"),
               "mass": torch.full((R, k), float("nan"), device="cuda"),
               "lse": torch.full((n_total,), float("nan"), device="cuda"),
               "xsketch": torch.full((R, k, d), float("nan"), device="cuda")}
        rc, st = _noalloc(g, R, n_total, d, k, out)
        assert rc == binding.SA_OK, binding.sa_status_string(rc)
        assert st == binding.SA_OK, binding.sa_status_string(st)
        for key in ("sketch", "mass", "xsketch"):
            got = out[key].cpu().double().numpy()
            exp = ref[key].cpu().double().numpy()
            for u in range(R):
                assert rel_l2(got[u], exp[u]) <= BF16_REL, (call, key, u)
            assert np.abs(got - exp).max() <= BF16_ABS * max(1.0, np.abs(exp).max()), (call, key)
        lse_got = out["lse"].cpu().double().numpy()
        assert np.abs(lse_got - ref["lse"].cpu().double().numpy()).max() <= BF16_ABS, call


def test_noalloc_matches_the_oracle():
    """One case checked against the fp64 oracle directly, so this file stands alone."""
    from parity_util import check_forward
    w = inputs.make_workload([2100, 0, 130, 700], 128, 512, "bf16", seed=4343)
    g = {n: getattr(w, n).cuda() for n in ("X", "offsets", "P", "Wk", "Wv")}
    R, n_total, d, k = w.R, w.n_total, w.d, w.k
    for call in range(2):
        out = {"sketch": torch.full((R, k, d), float("nan"), device="cuda"),
               "mass": torch.full((R, k), float("nan"), device="cuda"),
               "lse": torch.full((n_total,), float("nan"), device="cuda"),
               "xsketch": torch.full((R, k, d), float("nan"), device="cuda")}
        rc, st = _noalloc(g, R, n_total, d, k, out)
        assert rc == binding.SA_OK and st == binding.SA_OK, (call, rc, st)
        check_forward(w, out)


def test_noalloc_argument_errors_match_the_forward():
    w = inputs.make_workload([300], 128, 256, "bf16", seed=5)
    g = {n: getattr(w, n).cuda() for n in ("X", "offsets", "P", "Wk", "Wv")}
    out = {"sketch": torch.empty((1, 256, 128), device="cuda"),
           "mass": torch.empty((1, 256), device="cuda"),
           "lse": torch.empty((300,), device="cuda"),
           "xsketch": torch.empty((1, 256, 128), device="cuda")}
    rc, _ = _noalloc(g, 1, 300, 96, 256, out)
    assert rc == binding.SA_ERR_UNSUPPORTED
    st = ctypes.c_int(-1)
    rc = binding.sa_sketch_forward_noalloc(
        g["X"].data_ptr(), g["offsets"].data_ptr(), 1, 300, 128, g["P"].data_ptr(), 256,
        g["Wk"].data_ptr(), g["Wv"].data_ptr(), 9, out["sketch"].data_ptr(),
        out["mass"].data_ptr(), None, None, ctypes.addressof(st),
        torch.cuda.current_stream().cuda_stream)
    assert rc == binding.SA_ERR_INVALID_ARG and st.value == -1


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # 200 users at k = 2048 need far more than the fixed scratch: rejected before launch
    R, n_total, d, k = 200, 200 * 128, 128, 2048
    x = torch.zeros(n_total, d, dtype=torch.bfloat16, device="cuda")
    off = torch.arange(0, n_total + 1, 128, dtype=torch.int64, device="cuda")
    P = torch.zeros(k, d, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(d, d, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(R * k * d, device="cuda")
    m = torch.empty(R * k, device="cuda")
    rc = binding.sa_sketch_forward_noalloc(
        x.data_ptr(), off.data_ptr(), R, n_total, d, P.data_ptr(), k, W.data_ptr(), W.data_ptr(),
        binding.SA_BF16, out.data_ptr(), m.data_ptr(), None, None, None,
        torch.cuda.current_stream().cuda_stream)
    assert rc == binding.SA_ERR_WORKSPACE


def test_noalloc_runs_without_the_helper_grid_when_the_scratch_is_short():
    """20 users x 60K tokens at k = 1024: with the helper grid's segments the plan needs
    more than the 32 MiB scratch, without them it fits, so the call runs the clustered grid
    alone. The regular forward (with the helper grid) and the oracle agree with it."""
    from parity_util import check_forward
    w = inputs.make_workload([60000] * 20, 128, 1024, "bf16", seed=4444)
    g = {n: getattr(w, n).cuda() for n in ("X", "offsets", "P", "Wk", "Wv")}
    R, n_total, d, k = w.R, w.n_total, w.d, w.k
    _, _, H, _ = binding.forward_grid(k, d)
    assert H > 0
    assert binding.sa_sketch_workspace_size(R, n_total, k, d, binding.SA_BF16, 0) > (32 << 20)
    out = {"sketch": torch.full((R, k, d), float("nan"), device="cuda"),
           "mass": torch.full((R, k), float("nan"), device="cuda"),
           "lse": torch.full((n_total,), float("nan"), device="cuda"),
           "xsketch": torch.full((R, k, d), float("nan"), device="cuda")}
    rc, st = _noalloc(g, R, n_total, d, k, out)
    assert rc == binding.SA_OK and st == binding.SA_OK, (rc, st)
    ref = binding.forward(g["X"], g["offsets"], g["P"], g["Wk"], g["Wv"])
    for key in ("sketch", "mass"):
        got = out[key].cpu().double().numpy()
        exp = ref[key].cpu().double().numpy()
        for u in range(R):
            assert rel_l2(got[u], exp[u]) <= BF16_REL, (key, u)
    check_forward(w, out, users=[0, R - 1])
