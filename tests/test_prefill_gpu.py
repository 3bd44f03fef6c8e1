"""GPU parity of mla_prefill (long-prefix chunked prefill on the decode path) against the
float64 oracle, element by element, through the C ABI.

Cases cover sub-chunks of several sizes (d = 12, 1, 32, 16, 8 tokens), a chunk with no
prefix (T = C), a ragged partial last page, an e4m3 cache, and a request too short for its
chunk (device status, NaN rows, neighbours intact).
"""
import numpy as np
import pytest

from mla_attention_decode_paged_b200 import workloads as W
from tests import parity_util as pu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    from mla_attention_decode_paged_b200 import build
    build.build(quiet=True)


def _workload(B, C, H, lens, kv_dtype, seed):
    name = "agent_spec" if kv_dtype == W.KV_BF16 else "fp8_batch"
    return W.make_workload(name, B=B, s_q=C, H=H, seq_lens=lens, seed=seed)


def _run_prefill(wl):
    import torch
    import mla_attention_decode_paged_b200 as mla
    q, kv, bt, sl = pu.to_device(wl)
    B, C, H = wl.B, wl.s_q, wl.H
    ws = mla.alloc_prefill_workspace(B, C, H, int(bt.shape[1]))
    out = torch.full((B, C, H, W.DV), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, C, H), float("nan"), dtype=torch.float32, device="cuda")
    mla.prefill(q, kv, bt, sl, wl.scale, ws, out, lse, kv_scale=wl.kv_scale)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy(), mla.device_status(ws)


PREFILL_CASES = [
    (2, 24, 16, [300, 1000], W.KV_BF16),          # d = 12: three 64-row blocks per sub-chunk
    (1, 7, 128, [137], W.KV_BF16),                # d = 1: seven one-token sub-chunks of 128 rows
    (3, 64, 8, [64, 500, 2100], W.KV_BF16),       # d = 32; the first request has no prefix
    (2, 32, 16, [40, 3000], W.KV_E4M3),           # e4m3 cache
    (1, 200, 16, [2000], W.KV_BF16),              # d = 8: 25 sub-chunks
]


@pytest.mark.parametrize("B,C,H,lens,kv_dtype", PREFILL_CASES)
def test_prefill_matches_the_oracle(B, C, H, lens, kv_dtype):
    import oracle
    wl = _workload(B, C, H, lens, kv_dtype, seed=11)
    out, lse, code = _run_prefill(wl)
    assert code == 0
    ref_out, ref_lse = oracle.mla_prefill(wl.q, wl.kv, wl.kv_dtype, wl.kv_scale, wl.block_table, wl.seq_lens,
                                          wl.scale)
    pu.check_close(out, lse, ref_out, ref_lse, kv_dtype, what=f"prefill B={B} C={C} H={H}")


def test_request_shorter_than_its_chunk_is_reported_and_poisons_only_its_rows():
    import oracle
    wl = _workload(2, 16, 16, [10, 800], W.KV_BF16, seed=12)
    out, lse, code = _run_prefill(wl)
    assert code == 5  # MLA_ERR_DEVICE_OOB
    assert np.all(np.isnan(out[0]))
    r = [1]
    ref_out, ref_lse = oracle.mla_prefill(wl.q[r], wl.kv, wl.kv_dtype, wl.kv_scale, wl.block_table[r],
                                          wl.seq_lens[r], wl.scale)
    pu.check_close(out[r], lse[r], ref_out, ref_lse, wl.kv_dtype, what="neighbour of a short request")


def test_prefill_rejects_a_small_workspace():
    import torch
    import mla_attention_decode_paged_b200 as mla
    from mla_attention_decode_paged_b200 import _abi
    wl = _workload(1, 16, 16, [100], W.KV_BF16, seed=13)
    q, kv, bt, sl = pu.to_device(wl)
    need = mla.prefill_workspace_bytes(1, 16, 16, int(bt.shape[1]))
    ws = torch.zeros(need - 256, dtype=torch.uint8, device="cuda")
    out = torch.empty((1, 16, 16, W.DV), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, 16, 16), dtype=torch.float32, device="cuda")
    with pytest.raises(mla.MlaError) as e:
        mla.prefill(q, kv, bt, sl, wl.scale, ws, out, lse)
    assert e.value.code == _abi.MLA_ERR_WORKSPACE_TOO_SMALL


def test_bench_size_prefill_on_sampled_rows():
    """The prefill bench.py times (one request, chunk 1024 x 16 heads ending a 65,536-token
    cache), compared on sampled rows: chunk tokens 0, 511, 1023 (first and last head),
    each against a one-token oracle decode over its visible prefix."""
    import oracle
    C, H, T = 1024, 16, 65536
    wl = _workload(1, C, H, [T], W.KV_BF16, seed=21)
    out, lse, code = _run_prefill(wl)
    assert code == 0
    heads = [0, H - 1]
    for i in (0, 511, C - 1):
        ref_out, ref_lse = oracle.mla_decode(wl.q[:, i:i + 1][:, :, heads], wl.kv, wl.kv_dtype, wl.kv_scale,
                                             wl.block_table, np.array([T - C + i + 1], np.int32), wl.scale, False)
        pu.check_close(out[:, i:i + 1][:, :, heads], lse[:, i:i + 1][:, :, heads], ref_out, ref_lse, wl.kv_dtype,
                       what=f"bench-size prefill token {i}")
