"""Pins of the oracle's query absorption and output projection ("absorb + project",
zhaifeiyue "TokenSpeed" notes, DeepSeek-V3 entry): the defining identity of absorption,
and the whole absorb -> latent decode -> project pipeline of the oracle against
un-absorbed multi-head attention computed by a library SDPA.  CPU only."""
import math

import numpy as np
import torch
import torch.nn.functional as F

import oracle

RNG = np.random.default_rng(21)


def test_absorbed_query_scores_equal_unabsorbed_scores():
    """q_abs . c == q_nope . (c W_UK): the score is unchanged by moving W_UK to the query."""
    H = 3
    w_uk = RNG.standard_normal((H, 512, 128))
    q_nope = RNG.standard_normal((5, H, 128))
    q_rope = RNG.standard_normal((5, H, 64))
    c = RNG.standard_normal((7, 576))
    q = oracle.absorb_q(q_nope, q_rope, w_uk)
    assert q.shape == (5, H, 576) and np.array_equal(q[..., 512:], q_rope)
    for h in range(H):
        k_nope = c[:, :512] @ w_uk[h]                        # [7, 128]
        ref = q_nope[:, h] @ k_nope.T + q_rope[:, h] @ c[:, 512:].T
        np.testing.assert_allclose(q[:, h] @ c.T, ref, rtol=1e-12, atol=1e-10)


def _bf16_exact(x):
    return torch.from_numpy(np.asarray(x, np.float64)).to(torch.bfloat16).double().numpy()


def test_pipeline_equals_unabsorbed_mha_via_library_sdpa():
    B, s_q, H, T = 2, 3, 4, 150
    # integer weights / 16 and small integer q_nope keep the absorbed query exact in bf16
    w_uk = RNG.integers(-2, 3, (H, 512, 128)) / 16.0
    w_uv = RNG.standard_normal((H, 512, 128))
    q_nope = RNG.integers(-1, 2, (B, s_q, H, 128)).astype(np.float64)
    q_rope = _bf16_exact(RNG.standard_normal((B, s_q, H, 64)))
    q = oracle.absorb_q(q_nope, q_rope, w_uk)
    assert np.array_equal(_bf16_exact(q), q)
    q_bits = torch.from_numpy(q).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    rows = _bf16_exact(RNG.standard_normal((B, T, 576)))
    # pages of 64 tokens: each request padded to 192 rows (3 pages), pages in reverse order
    pool = np.zeros((B * 3, 64, 576), np.uint16)
    bt = np.arange(B * 3, dtype=np.int32).reshape(B, 3)[:, ::-1].copy()
    rb = torch.from_numpy(rows).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    for b in range(B):
        for t in range(T):
            pool[bt[b, t // 64], t % 64] = rb[b, t]
    scale = 1.0 / math.sqrt(192.0)
    out, _ = oracle.mla_decode(q_bits, pool, oracle.KV_BF16, 1.0, bt, np.full(B, T, np.int32), scale, True)
    y = oracle.project_out(out, w_uv)                           # [B, s_q, H, 128]
    for b in range(B):
        c = rows[b]
        for h in range(H):
            k_h = np.concatenate([c[:, :512] @ w_uk[h], c[:, 512:]], axis=1)
            v_h = c[:, :512] @ w_uv[h]
            q_h = np.concatenate([q_nope[b, :, h], q_rope[b, :, h]], axis=1)
            mask = np.ones((s_q, T), dtype=bool)
            for i in range(s_q):
                mask[i, T - s_q + i + 1:] = False
            ref = F.scaled_dot_product_attention(torch.from_numpy(q_h)[None, None], torch.from_numpy(k_h)[None, None],
                                                 torch.from_numpy(v_h)[None, None],
                                                 attn_mask=torch.from_numpy(mask)[None, None], scale=scale)[0, 0]
            np.testing.assert_allclose(y[b, :, h], ref.numpy(), rtol=1e-9, atol=1e-9)
