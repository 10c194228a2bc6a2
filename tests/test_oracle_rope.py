"""Pins of the oracle's RoPE position re-basing (oracle/prefill.py, step 2b)
against facts fixed outside it: a rotary pair is a complex number turned by
e^{i angle} (numpy's complex exponential), rotations of a pair add their
angles, they keep norms, scores depend only on position differences, and
re-basing a chunk-local rotary key equals rotating the raw key to its global
position. A mutation test plants a wrong pairing and checks a pin fails."""

import numpy as np
import pytest
import torch

import oracle.prefill as orc
from workloads import get_workload, make_layer_inputs, make_layout, scaled

D = 128
BASE = 500000.0


def rng_keys(n, seed=0):
    return np.random.default_rng(seed).standard_normal((n, D))


def as_complex(k):
    return k[..., : D // 2] + 1j * k[..., D // 2:]


def test_rotation_is_complex_multiplication():
    k = rng_keys(40)
    for off in (0, 1, 17, 1000, 65535):
        got = orc.rope_rotate(k, off, BASE)
        theta = BASE ** (-np.arange(D // 2) * 2.0 / D)
        want = as_complex(k) * np.exp(1j * off * theta)
        np.testing.assert_allclose(as_complex(got), want, rtol=0, atol=1e-12)


def test_rotations_add_their_angles_and_keep_norms():
    k = rng_keys(30, 1)
    a, b = 333, 4097
    two = orc.rope_rotate(orc.rope_rotate(k, a, BASE), b, BASE)
    one = orc.rope_rotate(k, a + b, BASE)
    np.testing.assert_allclose(two, one, rtol=0, atol=1e-11)
    np.testing.assert_allclose(np.abs(as_complex(one)), np.abs(as_complex(k)), rtol=1e-13)


def test_scores_depend_only_on_position_differences():
    q, k = rng_keys(5, 2), rng_keys(7, 3)
    s1 = orc.rope_rotate(q, 900, BASE) @ orc.rope_rotate(k, 100, BASE).T
    s2 = orc.rope_rotate(q, 60800, BASE) @ orc.rope_rotate(k, 60000, BASE).T
    np.testing.assert_allclose(s1, s2, rtol=0, atol=1e-10)


def test_rebasing_a_local_rotary_key_gives_the_global_rotary_key():
    raw = rng_keys(25, 4)
    t = np.arange(25)
    local = np.stack([orc.rope_rotate(raw[i], t[i], BASE) for i in range(25)])
    glob = np.stack([orc.rope_rotate(raw[i], 1234 + t[i], BASE) for i in range(25)])
    np.testing.assert_allclose(orc.rope_rotate(local, 1234, BASE), glob, rtol=0, atol=1e-11)


def test_offset_zero_keeps_the_bits_and_rounding_is_once():
    k = torch.from_numpy(rng_keys(64, 5)).to(torch.bfloat16)
    bits = k.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(orc.rope_rebase_bits(bits, 0, BASE), bits)
    got = orc.rope_rebase_bits(bits, 777, BASE)
    want = torch.from_numpy(orc.rope_rotate(orc.bits_to_f64(bits), 777, BASE)).to(torch.bfloat16)
    assert np.array_equal(got, want.view(torch.int16).numpy().view(np.uint16))


def test_first_chunk_of_a_request_is_unchanged_and_later_chunks_move():
    w = scaled(get_workload("llama3_8b_l32"), num_layers=1, num_q_heads=4, num_kv_heads=2,
               chunk_lens=(40, 70, 33), q_len=5)
    lay = make_layout(w)
    inp = make_layer_inputs(w, lay, 0)
    pk, _ = orc.build_layer_pool(lay, inp, np.uint16)
    chunks = [(lay.chunk_pages[c].numpy(), lay.chunk_len[c]) for c in lay.req_chunks[0]]
    plain = orc.gather(pk, 0, chunks)
    reb = orc.gather_rebased(pk, 0, chunks, BASE)
    assert np.array_equal(reb[:40], plain[:40])
    assert not np.array_equal(reb[40:110], plain[40:110])
    # chunk 2 sits at offset 110: each of its keys is turned by 110 positions
    want = orc.rope_rebase_bits(plain[110:143], 110, BASE)
    assert np.array_equal(reb[110:143], want)


def test_attention_with_rebasing_equals_attention_over_global_rotary_keys():
    """Raw keys rotated per chunk to local positions (what a chunk's offline
    prefill stores), re-based, give the scores of keys rotated straight to
    their global positions, up to the one bf16 rounding of the cache."""
    rng = np.random.default_rng(6)
    lens = [20, 45, 31]
    raw = [rng.standard_normal((n, 1, D)) for n in lens]
    local = [torch.from_numpy(np.stack([orc.rope_rotate(r[t], t, BASE) for t in range(len(r))])).to(torch.bfloat16)
             for r in raw]
    offs = np.cumsum([0] + lens)
    glob = np.concatenate([np.stack([orc.rope_rotate(r[t], offs[c] + t, BASE) for t in range(len(r))])
                           for c, r in enumerate(raw)])
    reb = np.concatenate([orc.bits_to_f64(orc.rope_rebase_bits(local[c].view(torch.int16).numpy().view(np.uint16),
                                                                offs[c], BASE)) for c in range(3)])
    q = rng.standard_normal((4, 1, D))
    np.testing.assert_allclose(q[:, 0] @ reb[:, 0].T, q[:, 0] @ glob[:, 0].T, rtol=0, atol=0.2)
    # the two bf16 roundings (of the cached local key, then of the re-based one) are the only
    # difference: bf16 keeps 8 significant bits, so each rounding moves a component by at most
    # 2^-8 of its size and a rotary pair by at most 2^-8 of its length; rotations keep lengths
    err = np.abs(as_complex(reb[:, 0]) - as_complex(glob[:, 0]))
    assert np.all(err <= 2.0 ** -7 * np.abs(as_complex(glob[:, 0])) * (1 + 1e-9))


def test_mutation_interleaved_pairs_is_caught(monkeypatch):
    def interleaved(k, offset, base):
        d = k.shape[-1]
        ang = float(offset) * orc.rope_theta_i(d, base)
        c, s = np.cos(ang), np.sin(ang)
        a, b = k[..., 0::2], k[..., 1::2]
        out = np.empty_like(k)
        out[..., 0::2], out[..., 1::2] = a * c - b * s, b * c + a * s
        return out

    monkeypatch.setattr(orc, "rope_rotate", interleaved)
    with pytest.raises(AssertionError):
        test_rotation_is_complex_multiplication()
