"""Numerics of an fp8 tensor-core scan for the e4m3 cache, emulated in float64 on the CPU.

An e4m3 x e4m3 MMA (tcgen05 kind::f8f6f4) would read the cache bytes as they are, with
no widening to bf16, but both of its operands must be fp8: q for the scores, P for the
output.  The requirement is that lse stays within 1e-3 of the oracle.  These tests
record what the arithmetic allows, on rows of the fp8 workload's shape (H = 128,
s_q = 2, causal, lengths of a few thousand tokens, where the errors are largest):

- q rounded to one e4m3 term (per-row scale amax / 448) moves lse by more than 1e-3:
  that single-term design is ruled out;
- q as two e4m3 terms at one scale (q_hi = e4m3(q), q_lo = e4m3(q - q_hi): two score
  chains accumulating into one accumulator, as many MMA instructions as the bf16 chain)
  with P as one e4m3 term and the row sum taken from the unrounded P meets every bound.

The emulation rounds with torch's float8_e4m3fn (round to nearest even) and keeps
everything else exact; the fp32 accumulation of the MMA is not the limiting error here.
"""
import numpy as np
import pytest
import torch

import oracle
from mla_attention_decode_paged_b200 import workloads as W

LENS = [5563, 4596, 4194, 12231, 6392, 1971]
HEADS = [0, 37, 127]


def _e4m3(x):
    x = np.clip(np.asarray(x, np.float64), -448.0, 448.0).astype(np.float32)
    return torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def _two_terms(x):
    hi = _e4m3(x)
    return hi + _e4m3(x - hi)


@pytest.fixture(scope="module")
def case():
    wl = W.make_workload("fp8_batch", B=len(LENS), seq_lens=LENS)
    codes = torch.from_numpy(wl.kv).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ref_out, ref_lse = oracle.mla_decode(wl.q[:, :, HEADS], wl.kv, wl.kv_dtype, wl.kv_scale, wl.block_table,
                                         wl.seq_lens, wl.scale, True)
    return wl, codes, ref_out, ref_lse


def _emulate(wl, codes, q_terms, p_round, rowsum_from_rounded):
    """out [B, s_q, heads, 512], lse [B, s_q, heads] of the emulated fp8 scan."""
    B, s_q = wl.B, wl.s_q
    out = np.zeros((B, s_q, len(HEADS), 512))
    lse = np.zeros((B, s_q, len(HEADS)))
    log2e = 1.0 / np.log(2.0)
    for b in range(B):
        T = int(wl.seq_lens[b])
        K = codes[wl.block_table[b, :(T + 63) // 64]].reshape(-1, 576)[:T]  # value = code * kv_scale
        q = W.bf16_bits_to_float32(wl.q[b][:, HEADS]).astype(np.float64)
        for i in range(s_q):
            vis = T - s_q + i + 1
            for k in range(len(HEADS)):
                rs = np.abs(q[i, k]).max() / 448.0
                s = (K[:vis] @ q_terms(q[i, k] / rs)) * rs * wl.kv_scale * wl.scale * log2e
                m = s.max()
                p = np.exp2(s - m + 8.0)  # the top of the kernel's P range (lazy max: P <= 256)
                pr = p_round(p)
                l = pr.sum() if rowsum_from_rounded else p.sum()
                out[b, i, k] = (pr @ K[:vis, :512]) * wl.kv_scale / l
                lse[b, i, k] = (m - 8.0 + np.log2(l)) * np.log(2.0)
    return out, lse


def _errors(out, lse, ref_out, ref_lse):
    worst = float((np.abs(out - ref_out) / (5e-2 + 5e-2 * np.abs(ref_out))).max())
    rel_l2 = float(np.linalg.norm(out - ref_out) / np.linalg.norm(ref_out))
    return worst, rel_l2, float(np.abs(lse - ref_lse).max())


def test_exact_operands_reproduce_the_oracle(case):
    """Control: unrounded q and P give the oracle to float64 rounding."""
    wl, codes, ref_out, ref_lse = case
    out, lse = _emulate(wl, codes, lambda x: x, lambda p: p, False)
    worst, rel_l2, lse_err = _errors(out, lse, ref_out, ref_lse)
    assert worst < 1e-9 and lse_err < 1e-10


def test_single_term_e4m3_query_breaks_the_lse_bound(case):
    wl, codes, ref_out, ref_lse = case
    out, lse = _emulate(wl, codes, _e4m3, lambda p: p, False)
    _, _, lse_err = _errors(out, lse, ref_out, ref_lse)
    assert lse_err > 1e-3


def test_two_term_query_and_single_term_p_meet_the_bounds(case):
    wl, codes, ref_out, ref_lse = case
    out, lse = _emulate(wl, codes, _two_terms, _e4m3, False)
    worst, rel_l2, lse_err = _errors(out, lse, ref_out, ref_lse)
    assert lse_err <= 1e-3, lse_err
    assert worst <= 1.0 and rel_l2 <= 3e-2, (worst, rel_l2)
