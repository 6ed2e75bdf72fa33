"""The torch conveniences of the binding check what the C ABI cannot see (shape, dtype,
memory layout, device) and raise before any CUDA call. CPU only: every case here fails
a check, so nothing reaches the library's compute entry points."""
import pytest
import torch


@pytest.fixture(scope="module")
def binding():
    from prototype_sketch_attention_b200 import build
    build.build()
    from prototype_sketch_attention_b200 import binding as b
    return b


def _inputs(n=10, k=256, d=128, dtype=torch.bfloat16):
    return dict(X=torch.zeros(n, d, dtype=dtype), offsets=torch.tensor([0, 4, n]),
                P=torch.zeros(k, d, dtype=dtype), Wk=torch.zeros(d, d, dtype=dtype),
                Wv=torch.zeros(d, d, dtype=dtype))


def _call_forward(binding, g, **kw):
    return binding.forward(g["X"], g["offsets"], g["P"], g["Wk"], g["Wv"], **kw)


@pytest.mark.parametrize("name,bad,msg", [
    ("P", lambda g: g["P"].float(), "P has dtype"),
    ("Wk", lambda g: g["Wk"].float(), "Wk has dtype"),
    ("Wv", lambda g: g["Wv"][:, :64], "Wv has shape"),
    ("P", lambda g: g["P"][:, :64], "P has shape"),
    ("offsets", lambda g: g["offsets"].int(), "offsets has dtype"),
    ("offsets", lambda g: g["offsets"][None], "offsets must be a 1-D"),
    ("X", lambda g: g["X"].t(), "X must be contiguous"),
    ("X", lambda g: g["X"][:, None], "X must be a 2-D"),
    ("Wk", lambda g: torch.zeros(256, dtype=torch.bfloat16)[::2].reshape(16, 8).t(), "Wk has shape"),
])
def test_forward_rejects_mismatched_inputs(binding, name, bad, msg):
    g = _inputs()
    g[name] = bad(g)
    with pytest.raises(binding.SketchAttentionError, match=msg) as e:
        _call_forward(binding, g)
    assert e.value.status == binding.SA_ERR_INVALID_ARG


def test_forward_rejects_unsupported_dtype(binding):
    g = _inputs(dtype=torch.float16)
    with pytest.raises(TypeError):
        _call_forward(binding, g)


def test_forward_rejects_wrong_outputs(binding):
    g = _inputs()
    R, k, d = 2, 256, 128
    good = {"sketch": torch.zeros(R, k, d), "mass": torch.zeros(R, k)}
    for out, msg in [({"mass": good["mass"]}, "sketch is required"),
                     ({**good, "sketch": torch.zeros(R, k, d, dtype=torch.float64)}, "sketch has dtype"),
                     ({**good, "mass": torch.zeros(R + 1, k)}, "mass has shape"),
                     ({**good, "lse": torch.zeros(9)}, "lse has shape"),
                     ({**good, "xsketch": torch.zeros(R, d, k).transpose(1, 2)}, "xsketch must be contiguous")]:
        with pytest.raises(binding.SketchAttentionError, match=msg):
            _call_forward(binding, g, out=out)


def test_host_tensors_are_refused_before_any_cuda_call(binding):
    g = _inputs()
    with pytest.raises(binding.SketchAttentionError, match="CUDA devices only"):
        _call_forward(binding, g)


def test_backward_rejects_mismatched_gradients(binding):
    g = _inputs()
    R, k, d = 2, 256, 128
    fwd = {"sketch": torch.zeros(R, k, d), "mass": torch.zeros(R, k), "xsketch": torch.zeros(R, k, d)}
    G = torch.zeros(R, k, d)
    cases = [
        (fwd, G[:, :, :64], None, "dsketch has shape"),
        (fwd, G.double(), None, "dsketch has dtype"),
        (fwd, G, torch.zeros(R, k + 1), "dmass has shape"),
        ({**fwd, "xsketch": None}, G, None, "xsketch is required"),
        ({**fwd, "mass": torch.zeros(R, k, dtype=torch.bfloat16)}, G, None, "mass has dtype"),
        (fwd, G, None, "CUDA devices only"),
    ]
    for f, dsk, dm, msg in cases:
        with pytest.raises(binding.SketchAttentionError, match=msg):
            binding.backward(g["X"], g["offsets"], g["P"], g["Wk"], g["Wv"], f, dsk, dm)


def test_combine_rejects_mismatched_inputs(binding):
    R, k, d = 3, 256, 128
    U, M, Wv = torch.zeros(R, k, d), torch.zeros(R, k), torch.zeros(d, d, dtype=torch.bfloat16)
    for args, msg in [((U[:, :, :100].contiguous(), M, Wv), "Wv has shape"),
                      ((U, M[:2], Wv), "mass has shape"),
                      ((U.bfloat16(), M, Wv), "xsketch has dtype"),
                      ((U, M, Wv), "CUDA devices only")]:
        with pytest.raises(binding.SketchAttentionError, match=msg):
            binding.combine(*args)


def test_forward_from_host_rejects_device_or_int32_offsets(binding):
    g = _inputs()
    with pytest.raises(binding.SketchAttentionError, match="offsets_h"):
        binding.forward_from_host(g["X"], g["offsets"].int(), g["P"], g["Wk"], g["Wv"])
    with pytest.raises(binding.SketchAttentionError, match="on the GPU"):
        binding.forward_from_host(g["X"], g["offsets"], g["P"], g["Wk"], g["Wv"])
    with pytest.raises(binding.SketchAttentionError, match="Xh must be"):
        binding.forward_from_host(g["X"].t(), g["offsets"], g["P"], g["Wk"], g["Wv"])
