"""Pins for the oracle's long-prefix chunked prefill (CPU only), and the identity the
library's prefill rests on.

The prefill reading: the chunk of C query tokens of request b are its last C cache rows,
and chunk token i (position T_b - C + i) sees the cached tokens t <= T_b - C + i.  The
pins tie it to a library causal attention (no prefix, contiguous cache), to C separate
one-token decodes (the mask offset, through a call where no causal offset applies), and
to a planted key (which rows see it).  The last test checks, inside the oracle, the
re-indexing the library uses: sub-chunks of d tokens as decode requests of their own.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from mla_attention_decode_paged_b200 import workloads as W

PAGE = 64


def _wl(B, C, H, lens, seed=0, kv_dtype=W.KV_BF16):
    name = "agent_spec" if kv_dtype == W.KV_BF16 else "fp8_batch"
    return W.make_workload(name, B=B, s_q=C, H=H, seq_lens=lens, seed=seed)


def _prefill(wl):
    return oracle.mla_prefill(wl.q, wl.kv, wl.kv_dtype, wl.kv_scale, wl.block_table, wl.seq_lens, wl.scale)


def _rows(wl, b, T):
    """The first T cache rows of request b as float64 [T, 576] (bf16 cache)."""
    bt = wl.block_table[b]
    pages = wl.kv[bt[:(T + PAGE - 1) // PAGE]].reshape(-1, 576)[:T]
    return W.bf16_bits_to_float32(pages).astype(np.float64)


def test_no_prefix_equals_library_causal_attention():
    """T = C, so the chunk is the whole sequence: textbook causal self-attention, with the
    latent row as key (576 wide) and its first 512 columns as value."""
    C, H = 70, 3
    wl = _wl(1, C, H, [C], seed=5)
    out, lse = _prefill(wl)
    kv = torch.from_numpy(_rows(wl, 0, C))
    q = torch.from_numpy(W.bf16_bits_to_float32(wl.q[0]).astype(np.float64)).permute(1, 0, 2)  # [H, C, 576]
    ref = F.scaled_dot_product_attention(q, kv.expand(H, C, 576), kv[:, :512].expand(H, C, 512), is_causal=True,
                                         scale=wl.scale)
    assert np.abs(out[0].transpose(1, 0, 2) - ref.numpy()).max() < 1e-12
    # the first token sees one key only: its lse is that key's score
    s0 = wl.scale * (q[:, 0] @ kv[0]).numpy()  # [H]
    assert np.abs(lse[0, 0] - s0).max() < 1e-12


def test_every_chunk_row_equals_a_one_token_decode_over_its_prefix():
    """Chunk token i equals a decode with s_q = 1 over the first T - C + i + 1 tokens (one
    draft sees its whole length: no causal offset is involved)."""
    B, C, H = 2, 9, 2
    lens = [9 + 100, 9 + 37]
    wl = _wl(B, C, H, lens, seed=6)
    out, lse = _prefill(wl)
    for b in range(B):
        for i in range(C):
            Ti = lens[b] - C + i + 1
            o1, l1 = oracle.mla_decode(wl.q[b:b + 1, i:i + 1], wl.kv, wl.kv_dtype, wl.kv_scale,
                                       wl.block_table[b:b + 1], np.array([Ti], np.int32), wl.scale, False)
            assert np.abs(out[b, i] - o1[0, 0]).max() < 1e-12
            assert np.abs(lse[b, i] - l1[0, 0]).max() < 1e-12


def test_planted_key_is_seen_from_its_own_token_on():
    """A huge-score key at chunk token k: rows i < k do not see it, rows i >= k snap to it."""
    C, H, prefix, k = 12, 2, 150, 5
    wl = _wl(1, C, H, [prefix + C], seed=7)
    base_out, _ = _prefill(wl)
    t0 = prefix + k
    pg, off = int(wl.block_table[0, t0 // PAGE]), t0 % PAGE
    qf = W.bf16_bits_to_float32(wl.q[0]).astype(np.float64)
    # the planted row is 4 sign(q) over the latent columns of one query row (rope part 0), and
    # head 0 of every chunk row gets q = sign(that row): its score with the planted row is
    # 4 * 512 * scale (about 148), far above every other score
    row = np.zeros(576, np.float32)
    row[:512] = 4.0 * np.sign(qf[0, 0, :512])
    wl.kv[pg, off] = W._bf16_bits(row)
    q = wl.q.copy()
    q[0, :, 0] = W._bf16_bits(np.sign(qf[0, 0]).astype(np.float32))
    wl.q = q
    out, _ = _prefill(wl)
    planted = W.bf16_bits_to_float32(wl.kv[pg, off, :512]).astype(np.float64)
    for i in range(C):
        if i >= k:
            assert np.abs(out[0, i, 0] - planted).max() < 1e-6, i
        else:
            assert np.abs(out[0, i, 0] - planted).max() > 1.0, i
    # head 1 is untouched before the planted token
    assert np.abs(out[0, :k, 1] - base_out[0, :k, 1]).max() == 0.0


@pytest.mark.parametrize("kv_dtype", [W.KV_BF16, W.KV_E4M3])
@pytest.mark.parametrize("C,d", [(24, 12), (24, 8), (7, 1), (16, 16)])
def test_sub_chunks_as_decode_requests_reproduce_the_prefill(C, d, kv_dtype):
    """Sub-chunk j of request b as a decode request of d drafts with length
    T_b - C + (j + 1) d and b's block-table row gives the prefill's rows exactly: q, out
    and lse keep their memory layout ([B, C, H] == [B C/d, d, H])."""
    B, H = 2, 4
    lens = [C + 90, C]
    wl = _wl(B, C, H, lens, seed=8, kv_dtype=kv_dtype)
    out, lse = _prefill(wl)
    n = C // d
    lens_x = np.array([lens[b] - C + (j + 1) * d for b in range(B) for j in range(n)], np.int32)
    bt_x = np.repeat(wl.block_table, n, axis=0)
    q_x = wl.q.reshape(B * n, d, H, 576)
    o2, l2 = oracle.mla_decode(q_x, wl.kv, wl.kv_dtype, wl.kv_scale, bt_x, lens_x, wl.scale, True)
    assert np.array_equal(o2.reshape(out.shape), out)
    assert np.array_equal(l2.reshape(lse.shape), lse)


def test_gpu_prefill_cases_would_reject_a_kernel_without_the_chunk_mask():
    """Negative control for the GPU prefill cases: the same inputs with the chunk's causal
    triangle dropped (every chunk token sees the whole chunk) fail the parity gate."""
    from tests import parity_util as pu
    from tests.test_prefill_gpu import PREFILL_CASES
    for B, C, H, lens, kv_dtype in PREFILL_CASES:
        name = "agent_spec" if kv_dtype == W.KV_BF16 else "fp8_batch"
        wl = W.make_workload(name, B=B, s_q=C, H=H, seq_lens=lens, seed=11)
        ref = _prefill(wl)
        no_mask = oracle.mla_decode(wl.q, wl.kv, wl.kv_dtype, wl.kv_scale, wl.block_table, wl.seq_lens, wl.scale,
                                    False)
        with pytest.raises(AssertionError):
            pu.check_close(*no_mask, *ref, kv_dtype)

