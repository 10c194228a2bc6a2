"""Plain definition of the KV cache codec decoded into the paged pool.

TEST INFRASTRUCTURE: only the tests, the smoke check and the benchmark's
CPU-baseline leg use this module. It shares no code with the CUDA library and
imports nothing from it.

What it computes (CacheGen page, "How the technology works"): a prefilled
chunk's KV cache is turned into a compact stream that is stored or sent, and
on the GPU the stream is decoded back into a KV cache from which generation
starts; the page's glossary names quantization (fewer bits per value, with
different compression levels for different parts of the cache). The pages
give no stream format. This restatement takes the plainest reading of that:

* Per chunk, layer, KV head and channel, the values of the chunk's tokens are
  quantized uniformly between their minimum and maximum: with b bits,
  scale = (max - min) / (2^b - 1), offset = min, code = round((v - offset) /
  scale) clamped to [0, 2^b - 1] (scale 0 when max = min: every code is 0).
  scale and offset are fp32.
* The bit width is chosen per layer (the "different compression levels per
  part"); this library takes b in {4, 8}. Codes of one token and KV head are
  stored channel by channel; with 4 bits two channels share a byte, the even
  channel in the low nibble.
* Decoding: v = fp32(code * scale + offset) (one fused multiply-add, one
  rounding to fp32), rounded once more to the type the pool stores it in (a
  bf16 cache keeps K in bf16 and V in fp16; round to nearest even, V
  saturated beyond 65504), token t of the chunk in page page_ids[t // 16],
  slot t % 16; the slots of the last page past the chunk's end are zeroed (as
  the pool write does).

The entropy coding of the real system is not described by the pages and is
not part of this restatement.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from .prefill import f16_bits_sat

PAGE_SIZE = 16


@dataclass
class EncodedChunk:
    bits: int
    codes_k: np.ndarray        # uint8 [n, H_kv, d] (8 bits) or [n, H_kv, d / 2] (4 bits)
    codes_v: np.ndarray
    scale_k: np.ndarray        # fp32 [H_kv, d]
    offset_k: np.ndarray
    scale_v: np.ndarray
    offset_v: np.ndarray


def quantize(x: np.ndarray, bits: int):
    """x: [n, H_kv, d] fp64 values. Returns codes (uint8, unpacked), scale, offset (fp32)."""
    levels = (1 << bits) - 1
    lo = x.min(axis=0).astype(np.float32)
    hi = x.max(axis=0).astype(np.float32)
    scale = ((hi.astype(np.float64) - lo.astype(np.float64)) / levels).astype(np.float32)
    safe = np.where(scale > 0, scale.astype(np.float64), 1.0)
    q = np.rint((x - lo.astype(np.float64)) / safe)
    q = np.where(scale > 0, q, 0.0)
    codes = np.clip(q, 0, levels).astype(np.uint8)
    return codes, scale, lo


def pack(codes: np.ndarray, bits: int) -> np.ndarray:
    if bits == 8:
        return codes.copy()
    assert bits == 4 and codes.shape[-1] % 2 == 0
    return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)


def unpack(packed: np.ndarray, bits: int) -> np.ndarray:
    if bits == 8:
        return packed.copy()
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = packed & 0x0F
    out[..., 1::2] = packed >> 4
    return out


def encode(k: np.ndarray, v: np.ndarray, bits: int) -> EncodedChunk:
    """Encode one chunk's K, V [n, H_kv, d] (exact values of the bf16 cache)."""
    ck, sk, ok = quantize(k, bits)
    cv, sv, ov = quantize(v, bits)
    return EncodedChunk(bits, pack(ck, bits), pack(cv, bits), sk, ok, sv, ov)


def dequantize_f32(codes: np.ndarray, scale: np.ndarray, offset: np.ndarray) -> np.ndarray:
    """fp32(code * scale + offset): the exact value, rounded once to fp32.

    code < 2^8 and scale has 24 significant bits, so code * scale is exact in
    fp64; the sum with offset is checked exact in fp64 (its rounding error,
    found by the TwoSum error-free transformation, is zero), so the single
    rounding to fp32 is the one a fused multiply-add makes.
    """
    a = codes.astype(np.float64) * scale.astype(np.float64)
    b = np.broadcast_to(offset.astype(np.float64), a.shape)
    s = a + b
    bb = s - a
    err = (a - (s - bb)) + (b - bb)
    assert np.all(err == 0), "sum not exact in fp64"
    return s.astype(np.float32)


def to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def decode_into_pool(pool_k: np.ndarray, pool_v: np.ndarray, layer: int, page_ids, enc: EncodedChunk,
                     n_tokens: int) -> None:
    """Decode one chunk of one layer into its pages (pools [L][pages][H_kv][16][d]
    of a bf16 cache: K bf16 bits, V fp16 bits)."""
    ck = unpack(enc.codes_k, enc.bits)
    cv = unpack(enc.codes_v, enc.bits)
    kb = to_bf16_bits(dequantize_f32(ck, enc.scale_k[None], enc.offset_k[None]))
    vb = f16_bits_sat(dequantize_f32(cv, enc.scale_v[None], enc.offset_v[None]).astype(np.float64))
    page_ids = np.asarray(page_ids, dtype=np.int64)
    assert len(page_ids) == -(-n_tokens // PAGE_SIZE)
    for t in range(n_tokens):
        pool_k[layer, page_ids[t // PAGE_SIZE], :, t % PAGE_SIZE, :] = kb[t]
        pool_v[layer, page_ids[t // PAGE_SIZE], :, t % PAGE_SIZE, :] = vb[t]
    for t in range(n_tokens, len(page_ids) * PAGE_SIZE):
        pool_k[layer, page_ids[t // PAGE_SIZE], :, t % PAGE_SIZE, :] = 0
        pool_v[layer, page_ids[t // PAGE_SIZE], :, t % PAGE_SIZE, :] = 0
