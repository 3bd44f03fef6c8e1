"""GPU parity of the query absorption and output projection (mla_absorb_q,
mla_project_out) with the float64 oracle, alone and around the decode."""
import numpy as np
import pytest

import oracle
from mla_attention_decode_paged_b200 import workloads as W
from tests import parity_util as pu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    from mla_attention_decode_paged_b200 import build
    build.build(quiet=True)


def _bf16(rng, shape, scale=1.0):
    import torch
    return (torch.from_numpy(rng.standard_normal(shape) * scale).to(torch.bfloat16))


def _close_bf16(got, ref):
    """fp32 accumulation then one bf16 rounding: within 2^-8 relative plus a small floor."""
    got = np.asarray(got, np.float64)
    err = np.abs(got - ref)
    assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 2e-3), float((err - 2.0 ** -8 * np.abs(ref)).max())


# R = B * s_q rows per head: 8, 256 with 16 heads (N tiles halved until the grid fills
# the SMs), 3, 1, 64 x 128 heads (the fp8 workload), 15 (a ragged N tile), 320 with 4
# heads (many small N tiles, the last one ragged), 256 x 64 heads (full 256-row N tiles
# for the absorption, halved for the projection)
@pytest.mark.parametrize("B,s_q,H", [(2, 4, 16), (16, 16, 16), (3, 1, 128), (1, 1, 1), (32, 2, 128), (3, 5, 7),
                                     (20, 16, 4), (16, 16, 64)])
def test_absorb_and_project_match_the_oracle(B, s_q, H):
    import torch
    rng = np.random.default_rng(B * 100 + H)
    q_nope = _bf16(rng, (B, s_q, H, 128))
    q_rope = _bf16(rng, (B, s_q, H, 64))
    w_uk = _bf16(rng, (H, 512, 128), 1.0 / np.sqrt(128))
    w_uv = _bf16(rng, (H, 512, 128), 1.0 / np.sqrt(512))
    out = _bf16(rng, (B, s_q, H, 512))
    import mla_attention_decode_paged_b200 as mla
    dev = [t.cuda() for t in (q_nope, q_rope, w_uk, w_uv, out)]
    q = torch.empty((B, s_q, H, 576), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((B, s_q, H, 128), dtype=torch.bfloat16, device="cuda")
    mla.absorb_q(dev[0], dev[1], dev[2], q)
    mla.project_out(dev[4], dev[3], y)
    torch.cuda.synchronize()
    ref_q = oracle.absorb_q(q_nope.double().numpy(), q_rope.double().numpy(), w_uk.double().numpy())
    ref_y = oracle.project_out(out.double().numpy(), w_uv.double().numpy())
    gq = q.double().cpu().numpy()
    assert np.array_equal(gq[..., 512:], ref_q[..., 512:])  # the rope part is copied
    _close_bf16(gq[..., :512], ref_q[..., :512])
    _close_bf16(y.double().cpu().numpy(), ref_y)


def test_absorb_decode_project_pipeline():
    """q_nope -> absorbed q -> latent decode -> projected output, against the oracle's own
    pipeline (absorbed q rounded to bf16 as the GPU stores it)."""
    import torch
    import mla_attention_decode_paged_b200 as mla
    wl = W.make_workload("agent_spec", B=2, seq=("fixed", 1500))
    rng = np.random.default_rng(3)
    q_nope = _bf16(rng, (wl.B, wl.s_q, wl.H, 128))
    q_rope = _bf16(rng, (wl.B, wl.s_q, wl.H, 64))
    w_uk = _bf16(rng, (wl.H, 512, 128), 1.0 / np.sqrt(128))
    w_uv = _bf16(rng, (wl.H, 512, 128), 1.0 / np.sqrt(512))
    q, kv, bt, sl = pu.to_device(wl)
    mla.absorb_q(q_nope.cuda(), q_rope.cuda(), w_uk.cuda(), q)
    ws = mla.alloc_workspace(wl.B, wl.s_q, wl.H)
    out = torch.empty((wl.B, wl.s_q, wl.H, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((wl.B, wl.s_q, wl.H), dtype=torch.float32, device="cuda")
    mla.plan(sl, wl.s_q, wl.H, ws)
    mla.decode(q, kv, bt, sl, wl.scale, wl.causal, ws, out, lse)
    y = torch.empty((wl.B, wl.s_q, wl.H, 128), dtype=torch.bfloat16, device="cuda")
    mla.project_out(out, w_uv.cuda(), y)
    assert mla.device_status(ws) == 0
    # the oracle pipeline, with the absorbed query the GPU fed to the decode
    wl.q = q.view(torch.int16).cpu().numpy().view(np.uint16)
    ref_out, ref_lse = pu.run_oracle(wl)
    pu.check_close(out.float().cpu().numpy(), lse.cpu().numpy(), ref_out, ref_lse, wl.kv_dtype, what="pipeline decode")
    ref_y = oracle.project_out(ref_out, w_uv.double().numpy())
    got = y.double().cpu().numpy()
    err = np.abs(got - ref_y)
    assert np.all(err <= 3e-2 + 3e-2 * np.abs(ref_y)), float(err.max())
    # and the absorbed query itself against the oracle
    ref_q = oracle.absorb_q(q_nope.double().numpy(), q_rope.double().numpy(), w_uk.double().numpy())
    _close_bf16(q.double().cpu().numpy()[..., :512], ref_q[..., :512])
