"""Pins of the V storage format of a bf16 cache (oracle/prefill.py, step 1):
each V value is kept as the fp16 value of its bf16 value. Pinned against
torch's bf16 -> fp16 conversion (a library routine) inside the fp16 range,
against closed forms of the IEEE binary16 format at its edges (saturation,
ties to even among subnormals, nan), and against the exactness fact the
format gives (every bf16 value of magnitude in [2^-14, 65280] is an fp16
value). A mutation test plants overflow to infinity and checks a pin fails."""

import numpy as np
import pytest
import torch

import oracle.prefill as orc
from workloads import get_workload, make_layer_inputs, make_layout, scaled


def bf16_bits(values):
    t = torch.tensor(values, dtype=torch.float64).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def all_bf16_bits():
    return np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)


def test_in_range_values_match_torch_conversion():
    b = all_bf16_bits()
    x = orc.bits_to_f64(b)
    keep = np.isfinite(x) & (np.abs(x) <= 65280.0)
    want = torch.from_numpy(b[keep].view(np.int16)).view(torch.bfloat16).to(torch.float16)
    got = orc.v_operand_bits(b[keep])
    assert np.array_equal(got, want.view(torch.int16).numpy().view(np.uint16))


def check_closed_forms():
    cases = [
        (65280.0, 0x7BF8),            # largest bf16 below 2^16: exact (1.11111111b * 2^15)
        (65536.0, 0x7BFF),            # beyond the fp16 range: saturated to 65504
        (-1.0e6, 0xFBFF),
        (float("inf"), 0x7BFF),
        (float("-inf"), 0xFBFF),
        (2.0 ** -14, 0x0400),         # smallest normal fp16
        (2.0 ** -24, 0x0001),         # smallest subnormal
        (2.0 ** -25, 0x0000),         # half of it: tie, to even (zero)
        (3 * 2.0 ** -25, 0x0002),     # 1.5 subnormal steps: tie, to even (two)
        (-(2.0 ** -25), 0x8000),
        (1.0, 0x3C00),
        (-2.5, 0xC100),
    ]
    got = orc.v_operand_bits(bf16_bits([v for v, _ in cases]))
    assert got.tolist() == [h for _, h in cases], [hex(g) for g in got]
    nan = orc.v_operand_bits(bf16_bits([float("nan")]))
    assert np.isnan(orc.f16_bits_to_f64(nan)).all()


def test_closed_forms_at_the_edges():
    check_closed_forms()


def test_exact_on_the_normal_fp16_range():
    b = all_bf16_bits()
    x = orc.bits_to_f64(b)
    keep = np.isfinite(x) & (np.abs(x) >= 2.0 ** -14) & (np.abs(x) <= 65280.0)
    assert np.array_equal(orc.f16_bits_to_f64(orc.v_operand_bits(b[keep])), x[keep])
    # below it the value moves by at most half an fp16 subnormal step
    small = np.isfinite(x) & (np.abs(x) < 2.0 ** -14)
    err = np.abs(orc.f16_bits_to_f64(orc.v_operand_bits(b[small])) - x[small])
    assert err.max() <= 2.0 ** -25


def test_pool_v_pages_hold_the_inputs_values():
    """On a generated layer (values far inside the range) the V pages decode to
    exactly the bf16 inputs, and the K pages keep the bf16 bits."""
    w = scaled(get_workload("llama3_8b_l32"), num_layers=1, num_q_heads=4, num_kv_heads=2,
               chunk_lens=(40, 17), q_len=3)
    lay = make_layout(w)
    inp = make_layer_inputs(w, lay, 0)
    pk, pv = orc.build_layer_pool(lay, inp, np.uint16)
    chunks = [(lay.chunk_pages[c].numpy(), lay.chunk_len[c]) for c in lay.req_chunks[0]]
    want_v = np.concatenate([inp.chunk_v[c].to(torch.float64).numpy() for c in lay.req_chunks[0]])
    want_k = np.concatenate([orc.to_bits(inp.chunk_k[c]) for c in lay.req_chunks[0]])
    assert np.array_equal(orc.f16_bits_to_f64(orc.gather(pv, 0, chunks)), want_v)
    assert np.array_equal(orc.gather(pk, 0, chunks), want_k)


def test_mutation_overflow_to_infinity_is_caught(monkeypatch):
    def no_saturation(b):
        return orc.bits_to_f64(b).astype(np.float16).view(np.uint16)
    monkeypatch.setattr(orc, "v_operand_bits", no_saturation)
    with pytest.raises(AssertionError):
        check_closed_forms()
