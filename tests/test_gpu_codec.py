"""GPU sketch cache codec (sa_sketch_pack / sa_sketch_unpack) against the reference in
oracle/codec.py: codes, scales and decoded values bit for bit (integer and byte work:
exact), on random sketches with zero rows, rows spanning the subnormal range after
scaling, and a real Sketch Attention output."""
import numpy as np
import pytest
import torch

from oracle import codec
from parity_util import gpu_forward
from prototype_sketch_attention_b200 import inputs

pytestmark = pytest.mark.gpu


def _sketches(R, k, d, seed):
    g = np.random.default_rng(seed)
    S = g.standard_normal((R, k, d)).astype(np.float32)
    S *= (10.0 ** g.uniform(-6, 3, (R, k, 1))).astype(np.float32)   # row magnitudes
    if k > 4:
        S[0, 3] = 0.0                                               # an all-zero row
        S[0, 4] = 0.0
        S[0, 4, 7] = -1e-30                                         # one tiny value
    S[-1, -1, ::3] *= 1e-4                                          # subnormal codes
    return S


@pytest.mark.parametrize("R,k,d", [(3, 256, 128), (2, 200, 64), (1, 1, 128)])
def test_fp8_pack_unpack_bit_exact(R, k, d):
    from prototype_sketch_attention_b200 import binding
    S = _sketches(R, k, d, seed=R + k + d)
    p = binding.sketch_pack(torch.from_numpy(S).cuda(), binding.SA_CODEC_FP8)
    codes, scales = p["codes"].cpu().numpy(), p["scales"].cpu().numpy()
    ref_c, ref_s = codec.fp8_encode(S)
    assert np.array_equal(scales.view(np.uint32), ref_s.view(np.uint32))
    assert np.array_equal(codes, ref_c)
    D = binding.sketch_unpack(p).cpu().numpy()
    assert np.array_equal(D.view(np.uint32), codec.fp8_decode(ref_c, ref_s).view(np.uint32))


@pytest.mark.parametrize("R,k,d", [(3, 256, 128), (2, 200, 64)])
def test_bf16_pack_unpack_bit_exact(R, k, d):
    from prototype_sketch_attention_b200 import binding
    S = _sketches(R, k, d, seed=10 + R + k + d)
    p = binding.sketch_pack(torch.from_numpy(S).cuda(), binding.SA_CODEC_BF16)
    bits = p["codes"].cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, codec.bf16_bits(S))
    D = binding.sketch_unpack(p).cpu().numpy()
    assert np.array_equal(D, codec.bf16_decode(codec.bf16_bits(S)))


def test_codec_on_a_forward_sketch():
    from prototype_sketch_attention_b200 import binding
    w = inputs.make_workload([3000, 0, 900], 128, 512, "bf16", seed=81)
    _, fwd = gpu_forward(w)
    S = fwd["sketch"]
    p = binding.sketch_pack(S, binding.SA_CODEC_FP8)
    ref_c, ref_s = codec.fp8_encode(S.cpu().numpy())
    assert np.array_equal(p["codes"].cpu().numpy(), ref_c)
    D = binding.sketch_unpack(p)
    # the packed sketch stays within the format's half spacing of the original
    err = (D - S).abs().cpu().numpy()
    Sn = S.abs().cpu().numpy()
    assert (err <= np.maximum(Sn * 2.0 ** -4, 2.0 ** -10 * ref_s[..., None]) * (1 + 1e-6)).all()
