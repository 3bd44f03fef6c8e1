"""Pins of the oracle's paged KV append (the write side of the cache) and of its rounding
routines, against library conversions, closed forms and the defining property of the
rotary embedding (scores depend only on relative position).  CPU only.

Definitions: oracle/mla_oracle.c, "paged KV append" section (paging from llm-atlas
"Inference systems" 07 PagedAttention; the decoupled rope key from 22 DeepSeek V2->V3).
"""
import numpy as np
import pytest
import torch

import oracle

RNG = np.random.default_rng(7)


def _bf16_bits(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _bits_to_f64(bits):
    return torch.from_numpy(np.asarray(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16).double().numpy()


def test_f32_to_bf16_matches_library_rounding():
    xs = np.concatenate([RNG.standard_normal(4000).astype(np.float32) * 10.0 ** RNG.integers(-30, 30, 4000),
                         np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.0e38, -1.5e-39], dtype=np.float32)])
    lib = _bf16_bits(xs)
    ours = np.array([oracle.f32_to_bf16(float(x)) for x in xs], dtype=np.uint16)
    assert np.array_equal(ours, lib)
    assert oracle.f32_to_bf16(float("nan")) & 0x7FC0 == 0x7FC0


def test_f32_to_e4m3_matches_library_inside_the_range_and_saturates_outside():
    xs = np.concatenate([RNG.uniform(-448, 448, 3000), RNG.standard_normal(3000) * 0.01,
                         [0.0, 1.0625, 1.1875, 0.001953125 * 1.5, 240.0, 448.0, -448.0]]).astype(np.float32)
    lib = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([oracle.f32_to_e4m3(float(x)) for x in xs], dtype=np.uint8)
    assert np.array_equal(ours, lib)
    # closed forms: ties go to the even code, magnitudes past the largest finite value saturate
    assert oracle.f32_to_e4m3(1.0625) == 0x38  # halfway between 1.0 (0x38) and 1.125 (0x39)
    assert oracle.f32_to_e4m3(449.0) == 0x7E and oracle.f32_to_e4m3(1.0e6) == 0x7E
    assert oracle.f32_to_e4m3(-500.0) == 0xFE
    assert oracle.f32_to_e4m3(float("nan")) == 0x7F


def test_rope_table_closed_forms():
    t = oracle.rope_table(5000).astype(np.float64)
    assert np.all(t[0, :32] == 1.0) and np.all(t[0, 32:] == 0.0)      # position 0: no rotation
    assert np.allclose(t[:, :32] ** 2 + t[:, 32:] ** 2, 1.0, atol=1e-6)  # unit rotations
    assert np.allclose(t[:, 0], np.cos(np.arange(5000)), atol=1e-6)    # theta_0 = 1
    assert np.allclose(t[:, 32], np.sin(np.arange(5000)), atol=1e-6)
    # theta_16 = 10000^(-1/2) = 0.01
    assert np.allclose(t[:, 16], np.cos(0.01 * np.arange(5000)), atol=1e-6)


def _append_one(s_q, T, kv_dtype=oracle.KV_BF16, kv_scale=1.0, ckv=None, kpe=None, page_ids=None):
    max_pages = (T + 63) // 64
    P = max_pages + 2
    page_ids = np.arange(max_pages, dtype=np.int32)[::-1].copy() if page_ids is None else page_ids
    kv = np.zeros((P, 64, 576), dtype=np.uint16 if kv_dtype == oracle.KV_BF16 else np.uint8)
    ckv = _bf16_bits(RNG.standard_normal((1, s_q, 512))) if ckv is None else ckv
    kpe = _bf16_bits(RNG.standard_normal((1, s_q, 64))) if kpe is None else kpe
    cs = oracle.rope_table(T + 1)
    out = oracle.kv_append(ckv, kpe, cs, kv, kv_dtype, kv_scale, page_ids[None, :], np.array([T], np.int32))
    return out, ckv, kpe, page_ids


def test_append_places_rows_by_block_table_and_copies_the_latent_exactly():
    s_q, T = 5, 130  # positions 125..129 straddle the page boundary at 128
    out, ckv, kpe, pids = _append_one(s_q, T)
    for i in range(s_q):
        pos = T - s_q + i
        row = out[pids[pos // 64], pos % 64]
        assert np.array_equal(row[:512], ckv[0, i])
    written = np.zeros(out.shape[:2], bool)
    for i in range(s_q):
        pos = T - s_q + i
        written[pids[pos // 64], pos % 64] = True
    assert np.all(out[~written] == 0)  # nothing else touched


def test_append_at_position_zero_is_the_unrotated_key():
    out, ckv, kpe, pids = _append_one(1, 1)
    assert np.array_equal(out[pids[0], 0, 512:], kpe[0, 0])


def test_rope_scores_depend_only_on_relative_position():
    """The defining property of the rotary embedding: <R(m) q, R(n) k> = <R(m + d) q, R(n + d) k>."""
    q = RNG.standard_normal(64)
    k = RNG.standard_normal(64)
    qb, kb = _bf16_bits(q), _bf16_bits(k)

    def rot(x_bits, pos):
        out, *_ = _append_one(1, pos + 1, kpe=x_bits[None, None, :], page_ids=np.arange((pos + 64) // 64, dtype=np.int32))
        return _bits_to_f64(out[pos // 64, pos % 64, 512:])

    base = rot(qb, 100) @ rot(kb, 37)
    for d in (1, 500, 3000):
        assert abs(rot(qb, 100 + d) @ rot(kb, 37 + d) - base) < 0.05 * (1 + abs(base))
    # and a rotation keeps each pair's length (up to bf16 rounding)
    r = rot(qb, 777).reshape(32, 2)
    x = _bits_to_f64(qb).reshape(32, 2)
    assert np.allclose(np.hypot(r[:, 0], r[:, 1]), np.hypot(x[:, 0], x[:, 1]), rtol=1e-2)


def test_e4m3_append_stores_exactly_representable_values_exactly():
    scale = 0.25
    codes = RNG.integers(0, 0x7E, (1, 3, 512)).astype(np.uint8)
    vals = np.array([oracle.e4m3_to_double(int(c)) * scale for c in codes.ravel()]).reshape(codes.shape)
    ckv = _bf16_bits(vals)  # every value x * 0.25 of an e4m3 x is exact in bf16
    out, _, _, pids = _append_one(3, 200, kv_dtype=oracle.KV_E4M3, kv_scale=scale, ckv=ckv)
    for i in range(3):
        pos = 197 + i
        assert np.array_equal(out[pids[pos // 64], pos % 64, :512], codes[0, i])


def test_append_rejects_out_of_range_lengths_and_pages():
    with pytest.raises(ValueError):
        _append_one(4, 3)  # T < s_q
    with pytest.raises(ValueError):
        _append_one(2, 70, page_ids=np.array([0, 99], dtype=np.int32))  # page id past the pool
