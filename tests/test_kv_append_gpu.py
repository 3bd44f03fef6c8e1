"""GPU parity of the paged KV append (mla_kv_append) with the oracle: the whole pool,
byte for byte, for a bf16 and an e4m3 cache; rows that straddle page boundaries; a bad
page id; and decode after append (the draft rows written, then verified)."""
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


def _bf16_bits(rng, shape):
    import torch
    x = torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).to(torch.bfloat16)
    return x.view(torch.int16).numpy().view(np.uint16)


def _setup(kv_dtype, seed=0, B=5, s_q=4, lens=(4, 63, 64, 65, 700)):
    rng = np.random.default_rng(seed)
    lens = np.array(lens[:B], dtype=np.int32)
    max_pages = int((lens.max() + 63) // 64)
    P = B * max_pages + 3
    perm = rng.permutation(P).astype(np.int32)
    bt = np.full((B, max_pages), -1, np.int32)
    k = 0
    for b in range(B):
        for t in range((lens[b] + 63) // 64):
            bt[b, t] = perm[k]
            k += 1
    if kv_dtype == W.KV_BF16:
        pool = rng.integers(0, 1 << 16, (P, 64, 576), dtype=np.uint16)
    else:
        pool = rng.integers(0, 256, (P, 64, 576), dtype=np.uint8)
    ckv = _bf16_bits(rng, (B, s_q, 512))
    kpe = _bf16_bits(rng, (B, s_q, 64))
    cs = oracle.rope_table(int(lens.max()) + 5)
    return pool, bt, lens, ckv, kpe, cs


def _run_gpu(pool, bt, lens, ckv, kpe, cs, kv_dtype, kv_scale):
    import torch
    import mla_attention_decode_paged_b200 as mla
    dev = "cuda"
    kvt = torch.from_numpy(pool.view(np.int16) if kv_dtype == W.KV_BF16 else pool).to(dev)
    if kv_dtype == W.KV_BF16:
        kvt = kvt.view(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    mla.kv_append(torch.from_numpy(ckv.view(np.int16)).to(dev).view(torch.bfloat16),
                  torch.from_numpy(kpe.view(np.int16)).to(dev).view(torch.bfloat16),
                  torch.from_numpy(cs).to(dev), kvt, torch.from_numpy(bt).to(dev), torch.from_numpy(lens).to(dev),
                  kv_scale=kv_scale, status=status)
    torch.cuda.synchronize()
    out = kvt.view(torch.int16).cpu().numpy().view(np.uint16) if kv_dtype == W.KV_BF16 else kvt.cpu().numpy()
    return out, int(status.item())


@pytest.mark.parametrize("kv_dtype,kv_scale", [(W.KV_BF16, 1.0), (W.KV_E4M3, 0.0123)])
def test_append_matches_oracle_byte_for_byte(kv_dtype, kv_scale):
    pool, bt, lens, ckv, kpe, cs = _setup(kv_dtype)
    ref = oracle.kv_append(ckv, kpe, cs, pool, kv_dtype, kv_scale, bt, lens)
    got, status = _run_gpu(pool, bt, lens, ckv, kpe, cs, kv_dtype, kv_scale)
    assert status == 0
    assert np.array_equal(got, ref)


def test_bad_page_id_sets_status_and_leaves_that_request_unwritten():
    pool, bt, lens, ckv, kpe, cs = _setup(W.KV_BF16, seed=1)
    bt_bad = bt.copy()
    bt_bad[4, (lens[4] - 1) // 64] = pool.shape[0] + 7  # the page of request 4's last rows
    got, status = _run_gpu(pool, bt_bad, lens, ckv, kpe, cs, W.KV_BF16, 1.0)
    assert status == 5
    ref = oracle.kv_append(ckv[:4], kpe[:4], cs, pool, W.KV_BF16, 1.0, bt[:4], lens[:4])
    assert np.array_equal(got, ref)  # requests 0-3 as the oracle writes them, request 4 untouched


def test_decode_after_append_verifies_the_new_rows():
    """Write the draft rows, then decode against the updated cache: the oracle decode of
    the oracle-appended pool is the reference."""
    import torch
    import mla_attention_decode_paged_b200 as mla
    wl = W.make_workload("agent_spec", B=3, seq=("fixed", 1000))
    rng = np.random.default_rng(5)
    ckv = _bf16_bits(rng, (wl.B, wl.s_q, 512))
    kpe = _bf16_bits(rng, (wl.B, wl.s_q, 64))
    cs = oracle.rope_table(1100)
    ref_pool = oracle.kv_append(ckv, kpe, cs, wl.kv, wl.kv_dtype, wl.kv_scale, wl.block_table, wl.seq_lens)
    q, kv, bt, sl = pu.to_device(wl)
    mla.kv_append(torch.from_numpy(ckv.view(np.int16)).cuda().view(torch.bfloat16),
                  torch.from_numpy(kpe.view(np.int16)).cuda().view(torch.bfloat16),
                  torch.from_numpy(cs).cuda(), kv, bt, sl)
    ws = mla.alloc_workspace(wl.B, wl.s_q, wl.H)
    out = torch.empty((wl.B, wl.s_q, wl.H, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((wl.B, wl.s_q, wl.H), dtype=torch.float32, device="cuda")
    mla.plan(sl, wl.s_q, wl.H, ws)
    mla.decode(q, kv, bt, sl, wl.scale, wl.causal, ws, out, lse)
    assert mla.device_status(ws) == 0
    wl.kv = ref_pool
    ref_out, ref_lse = pu.run_oracle(wl)
    pu.check_close(out.float().cpu().numpy(), lse.cpu().numpy(), ref_out, ref_lse, wl.kv_dtype, what="decode after append")
