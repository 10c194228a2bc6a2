"""Pins of the KV codec oracle (oracle/codec.py) against facts fixed outside
it: the quantization error bound of uniform b-bit codes, exact extremes and
constant channels, a hand-packed 4-bit byte, and the page placement of the
pool write. A mutation test swaps the nibble order and checks a pin fails."""

import struct

import numpy as np
import pytest
import torch

import oracle.codec as codec
import oracle.prefill as orc


def bf16_values(shape, seed, scale=1.0):
    x = torch.from_numpy(np.random.default_rng(seed).standard_normal(shape) * scale).to(torch.bfloat16)
    return x.to(torch.float64).numpy()


@pytest.mark.parametrize("bits", [8, 4])
def test_round_trip_error_is_within_half_a_step(bits):
    x = bf16_values((300, 4, 128), 1, scale=3.0)
    enc = codec.encode(x, x, bits)
    y = codec.dequantize_f32(codec.unpack(enc.codes_k, bits), enc.scale_k[None], enc.offset_k[None])
    y16 = orc.bits_to_f64(codec.to_bf16_bits(y))
    step = enc.scale_k.astype(np.float64)[None]
    # half a quantization step, plus the fp32 and bf16 roundings of the decoded value
    bound = 0.5 * step * (1 + 1e-6) + 2.0 ** -8 * np.abs(y16) + 1e-30
    assert np.all(np.abs(y16 - x) <= bound)
    # and the codes use the whole range
    c = codec.unpack(enc.codes_k, bits)
    assert c.min() == 0 and c.max() == (1 << bits) - 1


def test_extremes_and_constant_channels():
    x = bf16_values((50, 2, 128), 2)
    x[:, 1, 7] = 0.375                                  # a constant channel
    enc = codec.encode(x, x, 8)
    c = codec.unpack(enc.codes_k, 8)
    assert enc.scale_k[1, 7] == 0 and np.all(c[:, 1, 7] == 0)
    y = codec.dequantize_f32(c, enc.scale_k[None], enc.offset_k[None]).astype(np.float64)
    assert np.all(y[:, 1, 7] == 0.375)
    lo = x.min(axis=0)
    at_min = x == lo[None]
    assert np.all(y[at_min] == lo.astype(np.float32)[np.nonzero(at_min)[1:]])


def test_four_bit_packing_by_hand():
    codes = np.array([[[1, 2, 15, 0]]], dtype=np.uint8)
    packed = codec.pack(codes, 4)
    assert packed.tolist() == [[[0x21, 0x0F]]]          # even channel in the low nibble
    assert np.array_equal(codec.unpack(packed, 4), codes)


def test_decode_places_tokens_like_the_pool_write():
    n, hk, d = 37, 2, 128
    x = bf16_values((n, hk, d), 3)
    enc = codec.encode(x, x * 0.5, 8)
    pages = [5, 1, 3]
    pk = np.full((1, 6, hk, 16, d), 0xFFFF, dtype=np.uint16)
    pv = pk.copy()
    codec.decode_into_pool(pk, pv, 0, pages, enc, n)
    want_k = codec.to_bf16_bits(codec.dequantize_f32(codec.unpack(enc.codes_k, 8), enc.scale_k[None],
                                                     enc.offset_k[None]))
    ref = np.full_like(pk, 0xFFFF)
    orc.pool_write(ref, 0, pages, want_k)
    assert np.array_equal(pk, ref)
    # pages the chunk does not own are untouched
    assert np.all(pk[0, [0, 2, 4]] == 0xFFFF)
    # V: the fp32 value rounded once to binary16 (Python's struct packing)
    v32 = codec.dequantize_f32(codec.unpack(enc.codes_v, 8), enc.scale_v[None], enc.offset_v[None])
    want_v = np.frombuffer(struct.pack(f"<{v32.size}e", *v32.astype(np.float64).ravel().tolist()),
                           dtype=np.uint16).reshape(v32.shape)
    ref_v = np.full_like(pv, 0xFFFF)
    orc.pool_write(ref_v, 0, pages, want_v)
    assert np.array_equal(pv, ref_v)


def test_mutation_nibble_order_is_caught(monkeypatch):
    def swapped(codes, bits):
        return (codes[..., 1::2] | (codes[..., 0::2] << 4)).astype(np.uint8)

    monkeypatch.setattr(codec, "pack", swapped)
    with pytest.raises(AssertionError):
        test_four_bit_packing_by_hand()
