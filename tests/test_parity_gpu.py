"""GPU parity of libmla_decode.so against the float64 oracle, through the C ABI.

Small cases compare every output element; the full-size workloads run in the same
launch configuration as bench.py and compare sampled rows (the first and last request,
the first and last head, every draft token) that the oracle computes one by one.
Every workload carries NaN canaries in page tails and spare pages.
"""
import numpy as np
import pytest

from mla_attention_decode_paged_b200 import workloads as W
from tests import parity_util as pu
from tests import plan_ref

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    from mla_attention_decode_paged_b200 import build
    build.build(quiet=True)


def _case(name, num_sms, **kw):
    wl = W.make_workload(name, **kw)
    out, lse = pu.run_gpu(wl, num_sms=num_sms)
    ref_out, ref_lse = pu.run_oracle(wl)
    return pu.check_close(out.reshape(ref_out.shape), lse, ref_out, ref_lse, wl.kv_dtype, what=f"{name} {kw}")


SMALL = [
    ("tiny", {}),
    ("agent_spec", dict(seq=("fixed", 1000))),
    ("ragged_rownorm", dict(B=3, seq=("uniform", 300, 900))),
    ("long_m256", dict(B=2, seq=("fixed", 777))),
    ("fp8_batch", dict(B=6, seq=("lognormal", 300, 1.0, 65, 2000))),
    ("fp8_batch", dict(B=3, seq=("fixed", 333), causal=False)),
    ("agent_spec", dict(B=2, seq=("fixed", 500), causal=False)),
]


@pytest.mark.parametrize("num_sms", [0, 2, 16])
@pytest.mark.parametrize("name,kw", SMALL)
def test_small_workloads_elementwise(name, kw, num_sms):
    _case(name, num_sms, **kw)


@pytest.mark.parametrize("kw", [
    dict(B=2, s_q=4, H=16, seq_lens=[4, 5]),                    # T = s_q: draft 0 sees one token
    dict(B=1, s_q=1, H=1, seq_lens=[1]),                        # one row, one token
    dict(B=2, s_q=4, H=16, seq_lens=[65, 129]),                 # one-page splits: empty splits for early drafts
    dict(B=3, s_q=3, H=40, seq_lens=[64, 128, 4000]),           # M = 120, pages exactly full
    dict(B=2, s_q=5, H=40, seq_lens=[1500, 63]),                # M = 200: a partial second row block
    dict(B=9, s_q=1, H=16, seq_lens=[1, 2, 63, 64, 65, 127, 128, 129, 3000]),
])
@pytest.mark.parametrize("num_sms", [0, 4])
def test_edge_cases(kw, num_sms):
    _case("agent_spec", num_sms, **kw)


def test_many_short_requests():
    """More requests than the planner has threads: every planner loop makes several passes."""
    _case("agent_spec", 0, B=300, s_q=1, H=16, seq=("uniform", 1, 1500))


def test_zero_length_request_is_reported_and_poisons_only_its_rows():
    import torch
    import mla_attention_decode_paged_b200 as mla
    wl = W.make_workload("agent_spec", B=3, seq=("fixed", 700))
    q, kv, bt, sl = pu.to_device(wl)
    sl0 = torch.tensor([700, 0, 700], dtype=torch.int32, device="cuda")
    ws = mla.alloc_workspace(3, wl.s_q, wl.H)
    out = torch.zeros((3, wl.s_q, wl.H, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((3, wl.s_q, wl.H), dtype=torch.float32, device="cuda")
    mla.plan(sl0, wl.s_q, wl.H, ws)
    mla.decode(q, kv, bt, sl0, wl.scale, True, ws, out, lse)
    assert mla.device_status(ws) == 5
    o = out.float().cpu().numpy()
    assert np.all(np.isnan(o[1]))
    ref_out, ref_lse = pu.run_oracle(wl, requests=[0, 2])
    pu.check_close(o[[0, 2]], lse.cpu().numpy()[[0, 2]], ref_out, ref_lse, wl.kv_dtype, what="zero-length neighbour")


def test_split_count_does_not_change_the_result_beyond_rounding():
    wl = W.make_workload("long_m256", B=2, seq=("fixed", 3000))
    a_out, a_lse = pu.run_gpu(wl, num_sms=4)      # one split per request (4 row blocks, 1 group)
    b_out, b_lse = pu.run_gpu(wl, num_sms=0)      # many splits + combine
    ref_out, ref_lse = pu.run_oracle(wl)
    pu.check_close(a_out, a_lse, ref_out, ref_lse, wl.kv_dtype)
    pu.check_close(b_out, b_lse, ref_out, ref_lse, wl.kv_dtype)
    assert np.abs(a_lse - b_lse).max() < 1e-3


def test_page_permutation_leaves_the_result_within_rounding():
    wl = W.make_workload("agent_spec", B=2, seq=("fixed", 2000))
    out1, lse1 = pu.run_gpu(wl)
    perm = np.random.default_rng(1).permutation(wl.kv.shape[0])
    kv2 = np.empty_like(wl.kv)
    kv2[perm] = wl.kv
    wl.block_table = np.where(wl.block_table >= 0, perm[np.maximum(wl.block_table, 0)], -1).astype(np.int32)
    wl.kv = kv2
    out2, lse2 = pu.run_gpu(wl)
    assert np.abs(lse1 - lse2).max() < 1e-4
    assert np.abs(out1 - out2).max() < 2e-2


def _read_plan(ws):
    import torch
    raw = ws.cpu().numpy()
    h32 = raw[:48].view(np.int32)
    h64 = raw[48:96].view(np.int64)
    G, nseg, B = int(h32[7]), int(h32[8]), int(h32[3])
    gb = raw[h64[0]:h64[0] + 4 * (G + 1)].view(np.int32)
    rs = raw[h64[1]:h64[1] + 4 * (B + 1)].view(np.int32)
    segs = raw[h64[2]:h64[2] + 16 * nseg].view(np.int32).reshape(-1, 4)
    return h32, gb, rs, segs


@pytest.mark.parametrize("lens,s_q,H,num_sms", [([65536] * 4, 4, 16, 148), ([70000, 1, 64, 65, 30000], 2, 128, 148),
                                                ([300] * 3, 8, 32, 8), ([5] * 7, 1, 16, 1),
                                                (list(np.random.default_rng(1).integers(1, 3000, 600)), 1, 16, 148),
                                                ([0, 100, 0, 5000], 1, 16, 148)])
def test_device_plan_matches_host_restatement(lens, s_q, H, num_sms):
    import torch
    import mla_attention_decode_paged_b200 as mla
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = mla.alloc_workspace(len(lens), s_q, H, num_sms=num_sms)
    mla.plan(sl, s_q, H, ws, num_sms=num_sms)
    torch.cuda.synchronize()
    h32, gb, rs, segs = _read_plan(ws)
    G = plan_ref.num_groups_for(num_sms, (s_q * H + 63) // 64)
    egb, ers, esegs = plan_ref.plan(lens, G)
    assert h32[2] == 0x4D4C4131 and h32[7] == G
    assert np.array_equal(gb, egb) and np.array_equal(rs, ers) and np.array_equal(segs, esegs)


def test_bad_page_id_sets_device_status_and_poisons_only_that_request():
    import torch
    import mla_attention_decode_paged_b200 as mla
    wl = W.make_workload("agent_spec", B=3, seq=("fixed", 300))
    wl.block_table[1, 2] = wl.kv.shape[0] + 5
    q, kv, bt, sl = pu.to_device(wl)
    ws = mla.alloc_workspace(wl.B, wl.s_q, wl.H)
    out = torch.zeros((wl.B, wl.s_q, wl.H, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((wl.B, wl.s_q, wl.H), dtype=torch.float32, device="cuda")
    mla.plan(sl, wl.s_q, wl.H, ws)
    mla.decode(q, kv, bt, sl, wl.scale, True, ws, out, lse)
    assert mla.device_status(ws) == 5
    assert mla.device_status(ws) == 0  # cleared by the read
    o = out.float().cpu().numpy()
    assert np.all(np.isnan(o[1])) and np.all(np.isfinite(o[0])) and np.all(np.isfinite(o[2]))


def test_seq_len_beyond_block_table_sets_device_status():
    import torch
    import mla_attention_decode_paged_b200 as mla
    wl = W.make_workload("agent_spec", B=2, seq=("fixed", 128))
    q, kv, bt, sl = pu.to_device(wl)
    sl_bad = torch.tensor([128, 129], dtype=torch.int32, device="cuda")
    ws = mla.alloc_workspace(2, wl.s_q, wl.H)
    out = torch.zeros((2, wl.s_q, wl.H, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((2, wl.s_q, wl.H), dtype=torch.float32, device="cuda")
    mla.plan(sl_bad, wl.s_q, wl.H, ws)
    mla.decode(q, kv, bt, sl_bad, wl.scale, True, ws, out, lse)
    assert mla.device_status(ws) == 5
    assert np.all(np.isnan(out[1].float().cpu().numpy()))


@pytest.mark.parametrize("name", ["agent_spec", "ragged_rownorm", "long_m256", "fp8_batch"])
def test_full_size_workload_sampled_rows(name):
    """The full workload in the bench's launch configuration; oracle on sampled rows."""
    wl = W.make_workload(name)
    out, lse = pu.run_gpu(wl)
    reqs = [0, wl.B - 1]
    heads = [0, wl.H - 1]
    ref_out, ref_lse = pu.run_oracle(wl, heads=heads, requests=reqs)
    got_out = out[reqs][:, :, heads]
    got_lse = lse[reqs][:, :, heads]
    pu.check_close(got_out, got_lse, ref_out, ref_lse, wl.kv_dtype, what=name)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))


def test_bounded_wait_gives_up_with_a_status_and_the_context_stays_usable():
    """The scan kernel's mbarrier wait, run on a barrier that nothing arrives at, ends after
    its limit with the timeout status instead of hanging; decoding works afterwards."""
    import torch
    import mla_attention_decode_paged_b200 as mla
    from mla_attention_decode_paged_b200 import _abi
    wl = W.make_workload("agent_spec", B=2, seq=("fixed", 900))
    ws = mla.alloc_workspace(wl.B, wl.s_q, wl.H)
    stream = torch.cuda.current_stream().cuda_stream
    assert mla.device_status(ws) == 0  # a fresh workspace starts with a clear status word
    assert _abi.mla_debug_wait_timeout(ws.data_ptr(), ws.numel(), stream) == 0
    assert mla.device_status(ws) == 6  # MLA_ERR_DEVICE_TIMEOUT
    assert mla.device_status(ws) == 0
    out, lse = pu.run_gpu(wl)
    ref_out, ref_lse = pu.run_oracle(wl)
    pu.check_close(out.reshape(ref_out.shape), lse, ref_out, ref_lse, wl.kv_dtype, what="after a timeout")
