"""Numerics of the fp8 tensor-core scan for the e4m3 cache, emulated in float64 on the CPU.

The e4m3 scan runs e4m3 x e4m3 MMAs (tcgen05 kind::f8f6f4): the cache bytes are read as
they are, but both operands of each MMA must be fp8, so q (for the scores) and P (for
the output) are cut into e4m3 terms.  lse must stay within 1e-3 of the oracle and the
output within the relative L2 bound.  These tests record why the kernel cuts them the way
it does, on rows of the fp8 workload's shape (H = 128, s_q = 2, causal):

- one e4m3 term of q (per-row scale max|q| / 448) moves lse by more than 1e-3;
- two e4m3 terms at an arbitrary per-row scale still leave a 2^-8 residual; with a
  power-of-two row scale the scaled q is still a bf16 value, whose 8 significant bits two
  4-bit e4m3 terms hold exactly, so the scores are those of the bf16 q;
- P as one e4m3 term costs up to ~4% relative L2 on short rows; two terms, with
  P = 2^(x - m + 4) and the running max raised past a margin of 4 (P <= 256, the bulk
  of a long row far above e4m3's subnormal floor), meet every bound.

The emulation rounds with torch's float8_e4m3fn (round to nearest even) and keeps
everything else exact: on the GPU the kernel's lse matches this emulation to ~5e-6, so
the MMA's accumulation is not the limiting error.
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


def _pow2_two_terms(x):
    """The kernel's q split: scale by the largest power of two 2^k with max|x| 2^k <= 448."""
    k = np.floor(np.log2(448.0 / np.abs(x).max()))
    xs = x * 2.0 ** k
    hi = _e4m3(xs)
    return (hi + _e4m3(xs - hi)) * 2.0 ** -k


def test_power_of_two_scale_makes_the_two_term_query_exact():
    rng = np.random.default_rng(5)
    q = torch.from_numpy(rng.standard_normal((512, 576)).astype(np.float32)).to(torch.bfloat16).double().numpy()
    amax = np.abs(q).max(axis=1, keepdims=True)
    arbitrary = np.stack([_two_terms(r * 448.0 / m) * m / 448.0 for r, m in zip(q, amax[:, 0])])
    pow2 = np.stack([_pow2_two_terms(r) for r in q])
    assert np.abs(arbitrary - q).max() / amax.max() > 1e-4      # the arbitrary scale leaves a residual
    big = np.abs(q) >= amax * 2.0 ** -9                           # above e4m3's subnormal range after scaling
    assert np.array_equal(pow2[big], q[big])                      # exact where it matters
    assert np.abs(pow2 - q).max() <= amax.max() * 2.0 ** -17


def _online(wl, codes, b, heads, q_terms, p_terms, offset, margin):
    """The kernel's page-wise online softmax on request b: running max raised past `margin`,
    P = 2^(x - m + offset) cut into `p_terms`, row sum from the unrounded P."""
    T = int(wl.seq_lens[b])
    K = codes[wl.block_table[b, :(T + 63) // 64]].reshape(-1, 576)[:T]
    q = W.bf16_bits_to_float32(wl.q[b][:, heads]).astype(np.float64)
    out = np.zeros((wl.s_q, len(heads), 512))
    lse = np.zeros((wl.s_q, len(heads)))
    log2e = 1.0 / np.log(2.0)
    for i in range(wl.s_q):
        vis = T - wl.s_q + i + 1
        for k in range(len(heads)):
            s = (K[:vis] @ q_terms(q[i, k])) * wl.kv_scale * wl.scale * log2e
            m, l, O = -np.inf, 0.0, np.zeros(512)
            for p0 in range(0, vis, 64):
                sp = s[p0:p0 + 64]
                mt = sp.max()
                if mt > m + margin:
                    a = np.exp2(m - mt) if m > -np.inf else 0.0
                    l, O, m = l * a, O * a, mt
                P = np.exp2(sp - m + offset)
                assert P.max() <= 448.0
                l += P.sum()
                O += p_terms(P) @ K[p0:p0 + len(sp), :512]
            out[i, k] = O * wl.kv_scale / l
            lse[i, k] = (m - offset + np.log2(l)) * np.log(2.0)
    return out, lse


def test_kernel_scheme_meets_the_bounds_on_short_and_long_rows():
    """Power-of-two two-term q, two-term P with offset 4 and margin 4, on a short and a long
    request (the long one from the fp8 workload's clip length)."""
    wl = W.make_workload("fp8_batch", B=2, seq_lens=[300, 20000])
    codes = torch.from_numpy(wl.kv).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    heads = [0, 64, 127]
    ref_out, ref_lse = oracle.mla_decode(wl.q[:, :, heads], wl.kv, wl.kv_dtype, wl.kv_scale, wl.block_table,
                                         wl.seq_lens, wl.scale, True)
    for b in range(wl.B):
        out, lse = _online(wl, codes, b, heads, _pow2_two_terms, _two_terms, 4.0, 4.0)
        worst, rel_l2, lse_err = _errors(out, lse, ref_out[b], ref_lse[b])
        assert lse_err <= 1e-5, lse_err
        assert worst <= 0.1 and rel_l2 <= 3e-3, (worst, rel_l2)
        # one P term instead: within the element bound but far looser in relative L2
        out1, _ = _online(wl, codes, b, heads, _pow2_two_terms, _e4m3, 4.0, 4.0)
        assert _errors(out1, lse, ref_out[b], ref_lse[b])[1] > 3 * rel_l2
