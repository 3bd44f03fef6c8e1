"""Pins for the float64 oracle (CPU only).

Each test ties the oracle to something other than itself: a library attention routine
on the un-absorbed formulation, closed forms, invariances the definition implies, and
library decoders for the storage types.  Together they are chosen so that a dropped
term (the RoPE columns), a wrong scale, a wrong causal offset, a transposed operand or
a wrong page index fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from scipy.special import logsumexp

import oracle
from mla_attention_decode_paged_b200 import workloads as W

PAGE = 64


def _bf16(x):
    return W._bf16_bits(np.asarray(x, dtype=np.float32))


def _f(bits):
    return W.bf16_bits_to_float32(bits).astype(np.float64)


def _paged(kv_rows_list, rng, spare=1, nan_tail=True):
    """Scatter per-request rows [T_b, 576] (bf16 bits) into a shuffled page pool."""
    npages = [(r.shape[0] + PAGE - 1) // PAGE for r in kv_rows_list]
    P = sum(npages) + spare
    perm = rng.permutation(P)
    pool = np.full((P, PAGE, 576), W.BF16_NAN, dtype=np.uint16)
    bt = np.full((len(kv_rows_list), max(npages)), -1, dtype=np.int32)
    k = 0
    for b, rows in enumerate(kv_rows_list):
        for p in range(npages[b]):
            pg = int(perm[k]); k += 1
            bt[b, p] = pg
            chunk = rows[p * PAGE:(p + 1) * PAGE]
            pool[pg, :chunk.shape[0]] = chunk
    return pool, bt


# ---------------------------------------------------------------- storage decoders

def test_e4m3_decoder_matches_library_float8_on_all_256_bytes():
    lib = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([oracle.e4m3_to_double(b) for b in range(256)])
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(mine), nan)
    assert nan.sum() == 2  # 0x7F and 0xFF, no infinities in e4m3fn
    assert np.array_equal(mine[~nan], lib[~nan])


def test_e4m3_decoder_closed_forms():
    # bit layout s.eeee.mmm, bias 7: largest finite 1.75 * 2^8, smallest subnormal 2^-9
    assert oracle.e4m3_to_double(0x7E) == 448.0
    assert oracle.e4m3_to_double(0xFE) == -448.0
    assert oracle.e4m3_to_double(0x38) == 1.0
    assert oracle.e4m3_to_double(0x01) == 2.0 ** -9
    assert oracle.e4m3_to_double(0x08) == 2.0 ** -6
    assert oracle.e4m3_to_double(0x00) == 0.0
    assert math.isnan(oracle.e4m3_to_double(0x7F))


def test_bf16_decoder_matches_library_on_all_bit_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    lib = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    mine = np.array([oracle.bf16_to_double(int(b)) for b in bits[::97]])
    ref = lib[::97]
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], ref[~nan])


# ---------------------------------------------------------------- pin (i): un-absorbed MHA

def _unabsorbed_case(rng, B, s_q, H, lens, causal, d_nope=128, d_rope=64):
    """Random MLA weights; absorbed q exactly representable in bf16 (small integers / 16)."""
    W_UK = rng.integers(-1, 2, size=(H, 512, d_nope)) * (rng.random((H, 512, d_nope)) < 0.25)
    W_UV = rng.standard_normal((H, 512, d_nope))
    q_nope = rng.integers(-1, 2, size=(B, s_q, H, d_nope))
    q_abs = np.einsum("hcd,bihd->bihc", W_UK, q_nope) / 16.0     # integers / 16, |.| <= 8
    q_rope = _f(_bf16(rng.standard_normal((B, s_q, H, d_rope))))
    q_full = np.concatenate([q_abs, q_rope], axis=-1)
    q_bits = _bf16(q_full)
    assert np.array_equal(_f(q_bits), q_full)  # exact in bf16
    rows = [_bf16(rng.standard_normal((T, 576))) for T in lens]
    pool, bt = _paged(rows, rng)
    return dict(W_UK=W_UK, W_UV=W_UV, q_nope=q_nope / 16.0, q_rope=q_rope, q_bits=q_bits,
                rows=rows, pool=pool, bt=bt)


@pytest.mark.parametrize("causal", [True, False])
def test_pin_unabsorbed_mha_equivalence_via_library_sdpa(causal):
    rng = np.random.default_rng(11)
    B, s_q, H = 2, 3, 4
    lens = [70, 131]
    c = _unabsorbed_case(rng, B, s_q, H, lens, causal)
    scale = 1.0 / math.sqrt(192.0)
    out, lse = oracle.mla_decode(c["q_bits"], c["pool"], oracle.KV_BF16, 1.0, c["bt"],
                                 np.array(lens, np.int32), scale, causal)
    for b, T in enumerate(lens):
        ckv = _f(c["rows"][b])                       # [T, 576]
        latent, krope = ckv[:, :512], ckv[:, 512:]
        for h in range(H):
            # absorbed q . c = (W_UK q_nope / 16) . c = (q_nope / 16) . (c W_UK): per-head key c W_UK
            k_h = np.concatenate([latent @ c["W_UK"][h], krope], axis=1)          # [T, 192]
            v_h = latent @ c["W_UV"][h]                                           # [T, 128]
            q_h = np.concatenate([c["q_nope"][b, :, h], c["q_rope"][b, :, h]], axis=1)  # [s_q, 192]
            mask = np.ones((s_q, T), dtype=bool)
            if causal:
                for i in range(s_q):
                    mask[i, T - s_q + i + 1:] = False
            ref = F.scaled_dot_product_attention(torch.from_numpy(q_h)[None, None], torch.from_numpy(k_h)[None, None],
                                                 torch.from_numpy(v_h)[None, None],
                                                 attn_mask=torch.from_numpy(mask)[None, None], scale=scale)
            ref = ref[0, 0].numpy()
            got = out[b, :, h, :] @ c["W_UV"][h]
            np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-10)
            scores = (q_h @ k_h.T) * scale
            scores[~mask] = -np.inf
            np.testing.assert_allclose(lse[b, :, h], logsumexp(scores, axis=1), rtol=0, atol=1e-11)


def test_pin_textbook_single_query_contiguous_cache():
    """s_q = 1, H = 1, identity block table: plain single-query attention, d_k = 576, d_v = 512."""
    rng = np.random.default_rng(5)
    T = 200
    rows = _bf16(rng.standard_normal((T, 576)))
    P = (T + PAGE - 1) // PAGE
    pool = np.full((P, PAGE, 576), W.BF16_NAN, dtype=np.uint16)
    pool.reshape(-1, 576)[:T] = rows
    bt = np.arange(P, dtype=np.int32)[None]
    q = _bf16(rng.standard_normal((1, 1, 1, 576)))
    scale = 0.05
    out, lse = oracle.mla_decode(q, pool, oracle.KV_BF16, 1.0, bt, np.array([T], np.int32), scale, True)
    k = torch.from_numpy(_f(rows))
    ref = F.scaled_dot_product_attention(torch.from_numpy(_f(q)).reshape(1, 1, 1, 576), k[None, None],
                                         k[None, None, :, :512], scale=scale)
    np.testing.assert_allclose(out[0, 0, 0], ref.numpy().ravel(), rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- closed forms

def test_closed_form_zero_query_gives_mean_and_log_count():
    rng = np.random.default_rng(7)
    B, s_q, H = 2, 4, 2
    lens = [64, 150]
    rows = [_bf16(rng.standard_normal((T, 576))) for T in lens]
    pool, bt = _paged(rows, rng)
    q = np.zeros((B, s_q, H, 576), dtype=np.uint16)
    out, lse = oracle.mla_decode(q, pool, oracle.KV_BF16, 1.0, bt, np.array(lens, np.int32), 0.1, True)
    for b, T in enumerate(lens):
        lat = _f(rows[b])[:, :512]
        for i in range(s_q):
            n = T - s_q + i + 1
            for h in range(H):
                np.testing.assert_allclose(out[b, i, h], lat[:n].mean(axis=0), rtol=1e-12, atol=1e-13)
                assert abs(lse[b, i, h] - math.log(n)) < 1e-13


def test_closed_form_single_visible_row():
    """T_b = s_q under the causal rule: draft 0 sees exactly token 0."""
    rng = np.random.default_rng(8)
    s_q, H = 4, 3
    rows = [_bf16(rng.standard_normal((s_q, 576)))]
    pool, bt = _paged(rows, rng)
    q = _bf16(rng.standard_normal((1, s_q, H, 576)))
    scale = 0.07
    out, lse = oracle.mla_decode(q, pool, oracle.KV_BF16, 1.0, bt, np.array([s_q], np.int32), scale, True)
    k0 = _f(rows[0])[0]
    for h in range(H):
        assert np.array_equal(out[0, 0, h], k0[:512])
        assert abs(lse[0, 0, h] - scale * float(_f(q[0, 0, h]) @ k0)) < 1e-12


def test_closed_form_one_dominant_key():
    rng = np.random.default_rng(9)
    T = 300
    rows = _bf16(rng.standard_normal((T, 576)) * 0.01)
    t0 = 123
    rows[t0] = _bf16(np.full(576, 1.0))
    pool, bt = _paged([rows], rng)
    q = _bf16(np.full((1, 1, 2, 576), 1.0))
    out, _ = oracle.mla_decode(q, pool, oracle.KV_BF16, 1.0, bt, np.array([T], np.int32), 1.0, False)
    np.testing.assert_allclose(out[0, 0, 0], np.ones(512), atol=1e-12)


def test_planted_key_only_reaches_the_last_draft_row():
    """A key with a huge score at position T-1 is visible only to draft s_q-1."""
    rng = np.random.default_rng(10)
    s_q, H, T = 4, 2, 190
    rows = _bf16(rng.standard_normal((T, 576)))
    q = _bf16(rng.standard_normal((1, s_q, H, 576)))
    pool, bt = _paged([rows], rng)
    base_out, base_lse = oracle.mla_decode(q, pool, oracle.KV_BF16, 1.0, bt, np.array([T], np.int32), 0.07, True)
    planted = rows.copy()
    planted[T - 1] = _bf16(np.sign(_f(q[0, s_q - 1, 0])) * 8.0)
    pool2, bt2 = _paged([planted], np.random.default_rng(10))
    out, lse = oracle.mla_decode(q, pool2, oracle.KV_BF16, 1.0, bt2, np.array([T], np.int32), 0.07, True)
    assert np.array_equal(out[0, :s_q - 1], base_out[0, :s_q - 1])
    assert np.array_equal(lse[0, :s_q - 1], base_lse[0, :s_q - 1])
    np.testing.assert_allclose(out[0, s_q - 1, 0], _f(planted[T - 1])[:512], atol=1e-6)


# ---------------------------------------------------------------- invariances (iii), (iv)

def test_pin_page_permutation_invariance_is_bit_exact():
    wl = W.make_workload("agent_spec", seq=("fixed", 300), B=2)
    out, lse = oracle.mla_decode(wl.q, wl.kv, wl.kv_dtype, wl.kv_scale, wl.block_table, wl.seq_lens, wl.scale, True)
    rng = np.random.default_rng(3)
    P = wl.kv.shape[0]
    perm = rng.permutation(P)             # new physical slot of old page p is perm[p]
    kv2 = np.empty_like(wl.kv)
    kv2[perm] = wl.kv
    bt2 = np.where(wl.block_table >= 0, perm[np.maximum(wl.block_table, 0)], -1).astype(np.int32)
    out2, lse2 = oracle.mla_decode(wl.q, kv2, wl.kv_dtype, wl.kv_scale, bt2, wl.seq_lens, wl.scale, True)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


@pytest.mark.parametrize("cuts", [[0, 64, 300], [0, 1, 2, 299, 300], [0, 150, 150, 300], [0, 10, 128, 200, 257, 300]])
def test_pin_split_combine_equals_unsplit(cuts):
    wl = W.make_workload("agent_spec", seq=("fixed", 300), B=2)
    full_out, full_lse = oracle.mla_decode(wl.q, wl.kv, wl.kv_dtype, wl.kv_scale, wl.block_table, wl.seq_lens,
                                           wl.scale, True)
    parts_o, parts_l = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        o, l = oracle.mla_decode(wl.q, wl.kv, wl.kv_dtype, wl.kv_scale, wl.block_table, wl.seq_lens, wl.scale, True,
                                 tok_lo=np.full(2, a, np.int32), tok_hi=np.full(2, b, np.int32))
        parts_o.append(o)
        parts_l.append(l)
    o, l = oracle.combine(np.stack(parts_o), np.stack(parts_l))
    np.testing.assert_allclose(o, full_out, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l, full_lse, rtol=0, atol=1e-12)


def test_empty_split_has_minus_inf_lse_and_zero_output():
    wl = W.make_workload("agent_spec", seq=("fixed", 130), B=1)
    # tokens 128..129 are visible only to drafts whose last visible index reaches them
    o, l = oracle.mla_decode(wl.q, wl.kv, wl.kv_dtype, wl.kv_scale, wl.block_table, wl.seq_lens, wl.scale, True,
                             tok_lo=np.array([129], np.int32), tok_hi=np.array([130], np.int32))
    # draft i sees t <= 130 - 4 + i: t = 129 visible only for i = 3
    assert np.all(np.isneginf(l[0, :3])) and np.all(o[0, :3] == 0)
    assert np.all(np.isfinite(l[0, 3]))


# ---------------------------------------------------------------- fp8 cache

def test_e4m3_pool_equals_bf16_pool_of_decoded_values():
    """With a power-of-two scale every e4m3 value times the scale is exact in bf16, so the
    fp8 cache and the bf16 cache of its decoded values must give identical results."""
    wl = W.make_workload("fp8_batch", B=2, seq=("fixed", 200), spare_pages=1)
    kv_scale = 2.0 ** -5
    decoded = torch.from_numpy(wl.kv).view(torch.float8_e4m3fn).to(torch.float32) * kv_scale
    kv_bf16 = decoded.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert torch.equal(torch.from_numpy(kv_bf16.view(np.int16)).view(torch.bfloat16).float().nan_to_num(7.0),
                       decoded.nan_to_num(7.0))
    o1, l1 = oracle.mla_decode(wl.q, wl.kv, oracle.KV_E4M3, kv_scale, wl.block_table, wl.seq_lens, wl.scale, True)
    o2, l2 = oracle.mla_decode(wl.q, kv_bf16, oracle.KV_BF16, 1.0, wl.block_table, wl.seq_lens, wl.scale, True)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_canaries_are_never_read():
    wl = W.make_workload("ragged_rownorm", B=3, seq=("uniform", 65, 200))
    out, lse = oracle.mla_decode(wl.q, wl.kv, wl.kv_dtype, wl.kv_scale, wl.block_table, wl.seq_lens, wl.scale, True)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))


def test_rejects_lengths_the_definition_does_not_cover():
    wl = W.make_workload("agent_spec", seq=("fixed", 100), B=1)
    with pytest.raises(ValueError):
        oracle.mla_decode(wl.q, wl.kv, wl.kv_dtype, wl.kv_scale, wl.block_table, np.array([3], np.int32),
                          wl.scale, True)  # T < s_q under the causal rule
    bad_bt = wl.block_table.copy()
    bad_bt[0, 0] = wl.kv.shape[0]
    with pytest.raises(ValueError):
        oracle.mla_decode(wl.q, wl.kv, wl.kv_dtype, wl.kv_scale, bad_bt, wl.seq_lens, wl.scale, True)
