"""Pins for the sketch cache codec reference (oracle/codec.py).

The E4M3 and bfloat16 roundings there are written from the formats' definitions; here
they are checked bit for bit against torch's own conversions (library routines), over
every E4M3 value, the midpoints between neighbours (ties to even), random values across
the whole range and the subnormals, and against closed forms: exact values round-trip,
the error stays within half a spacing, all-zero rows decode to zero.
"""
import numpy as np
import pytest
import torch

from oracle import codec


def _all_e4m3_values():
    b = torch.arange(256, dtype=torch.int64).to(torch.uint8)
    v = b.view(torch.float8_e4m3fn).float().numpy()
    return v[np.isfinite(v)]


def test_e4m3_bits_match_torch_on_every_representable_value():
    v = _all_e4m3_values()
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = codec.e4m3_bits(v)
    keep = v != 0  # +0 and -0: torch keeps the sign of zero, the codec writes +0
    assert np.array_equal(got[keep], ref[keep])
    np.testing.assert_array_equal(codec.e4m3_decode(got), np.where(v == 0, 0.0, v))


def test_e4m3_ties_go_to_even_like_torch():
    v = np.unique(np.abs(_all_e4m3_values()))
    mids = (v[:-1] + v[1:]) / 2  # exactly halfway between neighbours
    for x in (mids, -mids):
        ref = torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8)
        got = codec.e4m3_bits(x.astype(np.float32))
        keep = codec.e4m3_decode(got) != 0  # a tie down to zero: the codec writes +0
        assert np.array_equal(got[keep], ref.numpy()[keep])
        assert (codec.e4m3_decode(ref.numpy()[~keep]) == 0).all()


def test_e4m3_random_values_match_torch():
    g = np.random.default_rng(0)
    x = np.concatenate([g.uniform(-448, 448, 20000), g.uniform(-2.0 ** -6, 2.0 ** -6, 5000),
                        g.standard_normal(5000)]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = codec.e4m3_bits(x)
    keep = codec.e4m3_decode(got) != 0
    assert np.array_equal(got[keep], ref[keep])
    assert (codec.e4m3_decode(ref[~keep]) == 0).all()


def test_bf16_bits_match_torch():
    g = np.random.default_rng(1)
    x = np.concatenate([g.standard_normal(20000) * 10.0 ** g.integers(-20, 20, 20000),
                        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -1.0 - 2.0 ** -8])]
                       ).astype(np.float32)
    ref = torch.from_numpy(x).bfloat16().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(codec.bf16_bits(x), ref)
    np.testing.assert_array_equal(codec.bf16_decode(codec.bf16_bits(x)),
                                  torch.from_numpy(x).bfloat16().float().numpy())


def test_fp8_codec_round_trip_bounds():
    g = np.random.default_rng(2)
    S = g.standard_normal((3, 64, 128)).astype(np.float32)
    S[1, 5] = 0.0  # an all-zero row
    codes, scales = codec.fp8_encode(S)
    assert codes.dtype == np.uint8 and codes.shape == S.shape and scales.shape == (3, 64)
    D = codec.fp8_decode(codes, scales)
    assert not D[1, 5].any() and scales[1, 5] == 1.0
    # every row's largest magnitude maps to 448 exactly, so it round-trips exactly
    j = np.abs(S).argmax(axis=-1)
    np.testing.assert_allclose(np.take_along_axis(D, j[..., None], -1),
                               np.take_along_axis(S, j[..., None], -1), rtol=1e-6)
    # error within half a spacing: 2^-4 relative in the normal range, 2^-10 * scale below
    err = np.abs(D.astype(np.float64) - S)
    bound = np.maximum(np.abs(S) * 2.0 ** -4, 2.0 ** -10 * scales[..., None]) * (1 + 1e-6)
    assert (err <= bound).all()


def test_fp8_codec_is_idempotent_on_decoded_values():
    g = np.random.default_rng(3)
    S = (g.standard_normal((8, 32)) * 5).astype(np.float32)
    c1, s1 = codec.fp8_encode(S)
    D1 = codec.fp8_decode(c1, s1)
    c2, s2 = codec.fp8_encode(D1)
    np.testing.assert_array_equal(s1, s2)
    np.testing.assert_array_equal(c1, c2)


@pytest.mark.parametrize("x,code", [(448.0, 0x7E), (-448.0, 0xFE), (1.0, 0x38), (2.0 ** -9, 0x01),
                                    (2.0 ** -6, 0x08), (0.875 * 2.0 ** -6, 0x07), (3.5, 0x46)])
def test_e4m3_known_codes(x, code):
    """Bit patterns that follow from the format's definition (sign, 4-bit exponent with
    bias 7, 3-bit mantissa; subnormals k 2^-9)."""
    assert int(codec.e4m3_bits(np.array([x]))[0]) == code
