"""GPU parity of libmla_decode.so against the float64 oracle, through the C ABI.

Small cases compare every output element; the full-size workloads run in the same
launch configuration as bench.py and compare sampled rows that the oracle computes one
by one (a request the plan split and one it held whole where the workload has both,
seeded heads, every draft token); a planted key checks the draft mask at full length.
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


@pytest.mark.parametrize("kw", [
    dict(B=2, s_q=2, H=128, seq_lens=[2, 3]),                   # T = s_q: draft 0 sees one token
    dict(B=9, s_q=1, H=64, seq_lens=[1, 2, 63, 64, 65, 127, 128, 129, 3000]),
    dict(B=3, s_q=2, H=128, seq_lens=[64 * 3, 64 * 5 + 7, 64 * 2]),  # odd and even page counts
    dict(B=2, s_q=4, H=48, seq_lens=[1500, 63]),                # M = 192: a partial third row block
])
@pytest.mark.parametrize("num_sms", [0, 4, 16])
def test_edge_cases_e4m3(kw, num_sms):
    """The e4m3 scan takes a split's pages in pairs: single-page units (odd counts, one-page
    splits), pages exactly full and partial last pages, on plans of several shapes."""
    _case("fp8_batch", num_sms, **kw)


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


@pytest.mark.parametrize("lens,s_q,H,num_sms", [([65536] * 4, 4, 16, 148), ([70000, 1, 64, 65, 30000], 2, 128, 148),
                                                ([300] * 3, 8, 32, 8), ([5] * 7, 1, 16, 1),
                                                (list(np.random.default_rng(1).integers(1, 3000, 600)), 1, 16, 148),
                                                ([0, 100, 0, 5000], 1, 16, 148),
                                                # more groups than pages: runs of equal cuts
                                                ([1, 1, 1], 1, 16, 1023), ([64] * 3 + [0] * 5 + [65], 4, 16, 1000),
                                                # several thousand requests (several per planner thread), some empty
                                                (list(np.where(np.random.default_rng(2).random(5000) < 0.1, 0,
                                                               np.random.default_rng(3).integers(1, 4000, 5000))),
                                                 1, 16, 148),
                                                ([-5, 10, 0], 2, 16, 148), ([131072] * 16, 16, 16, 148),
                                                # the largest batch the planner's shared memory holds
                                                (list(np.random.default_rng(4).integers(1, 200, 12000)), 1, 16, 148)])
def test_device_plan_matches_host_restatement(lens, s_q, H, num_sms):
    import torch
    import mla_attention_decode_paged_b200 as mla
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = mla.alloc_workspace(len(lens), s_q, H, num_sms=num_sms)
    mla.plan(sl, s_q, H, ws, num_sms=num_sms)
    torch.cuda.synchronize()
    h32, gb, rs, segs = pu.read_plan(ws)
    G = plan_ref.num_groups_for(num_sms, (s_q * H + 63) // 64)
    egb, ers, esegs = plan_ref.plan(lens, G)
    assert h32[2] == 0x4D4C4131 and h32[7] == G
    assert np.array_equal(gb, egb) and np.array_equal(rs, ers) and np.array_equal(segs, esegs)
    bad = [b for b, t in enumerate(lens) if t <= 0]  # a request without tokens is reported, the first one
    assert (h32[0], h32[1]) == ((5, bad[0]) if bad else (0, 0))
    # each group's head record (read by the scan beside the header): its segment range and
    # a copy of its first segment
    heads = ws.cpu().numpy()[256:256 + 32 * G].view(np.int32).reshape(G, 8)
    assert np.array_equal(heads[:, 0], egb[:-1]) and np.array_equal(heads[:, 1], egb[1:])
    for g in range(G):
        want = esegs[egb[g]] if egb[g] < egb[g + 1] else np.zeros(4, np.int32)
        assert np.array_equal(heads[g, 4:], want), g


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
    l = lse.cpu().numpy()
    assert np.all(np.isnan(l[1])) and np.all(np.isfinite(l[[0, 2]]))


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
    assert np.all(np.isnan(lse[1].cpu().numpy())), "a poisoned split request reports NaN lse too"
    assert np.all(np.isfinite(lse[0].cpu().numpy()))


@pytest.mark.parametrize("name", ["agent_spec", "fp8_batch"])
def test_causal_length_shorter_than_the_drafts_is_reported(name):
    """Under the draft mask a request needs at least s_q tokens (its drafts' own rows): a
    shorter one is reported (device status) and its rows are NaN; its neighbours are exact."""
    import torch
    import mla_attention_decode_paged_b200 as mla
    wl = W.make_workload(name, B=3, seq=("fixed", 700))
    q, kv, bt, sl = pu.to_device(wl)
    short = wl.s_q - 1  # >= 1: the request has tokens, but fewer than its drafts
    sl_bad = torch.tensor([700, short, 700], dtype=torch.int32, device="cuda")
    ws = mla.alloc_workspace(3, wl.s_q, wl.H)
    out = torch.zeros((3, wl.s_q, wl.H, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((3, wl.s_q, wl.H), dtype=torch.float32, device="cuda")
    mla.plan(sl_bad, wl.s_q, wl.H, ws)
    mla.decode(q, kv, bt, sl_bad, wl.scale, True, ws, out, lse, kv_scale=wl.kv_scale)
    assert mla.device_status(ws) == 5
    o, l = out.float().cpu().numpy(), lse.cpu().numpy()
    assert np.all(np.isnan(o[1])) and np.all(np.isnan(l[1]))
    ref_out, ref_lse = pu.run_oracle(wl, requests=[0, 2])
    pu.check_close(o[[0, 2]], l[[0, 2]], ref_out, ref_lse, wl.kv_dtype, what="short-request neighbours")


def _sample_requests_and_heads(wl, segs, seed):
    """Requests the plan split and requests it held whole (the first of each, where the
    workload has them), one more seeded request, and heads {0, H-1} plus three seeded
    heads."""
    rng = np.random.default_rng(seed)
    split = sorted({int(b) for b, _, _, sp in segs if sp})
    whole = sorted({int(b) for b, _, _, sp in segs if not sp})
    reqs = {split[0]} if split else set()
    if whole:
        reqs.add(whole[0])
    reqs.add(int(rng.integers(0, wl.B)))
    heads = {0, wl.H - 1} | {int(h) for h in rng.choice(wl.H, size=min(3, wl.H), replace=False)}
    return sorted(reqs), sorted(heads), split, whole


@pytest.mark.parametrize("name", ["agent_spec", "ragged_rownorm", "long_m256", "fp8_batch"])
def test_full_size_workload_sampled_rows(name):
    """The full workload in the bench's launch configuration; the oracle on sampled rows of a
    request the plan split (partials + combine) and of one it held whole (direct bf16 out),
    where the workload has both, on seeded heads and every draft token."""
    wl = W.make_workload(name)
    out, lse, ws = pu.run_gpu(wl, return_ws=True)
    _, _, _, segs = pu.read_plan(ws)
    reqs, heads, split, whole = _sample_requests_and_heads(wl, segs, seed=W.WORKLOAD_ORDER.index(name))
    assert split, "the bench configuration splits at least one request"
    if name == "fp8_batch":
        assert whole, "the ragged fp8 batch has requests that one share holds whole"
        assert any(b in whole for b in reqs) and any(b in split for b in reqs)
    ref_out, ref_lse = pu.run_oracle(wl, heads=heads, requests=reqs)
    got_out = out[reqs][:, :, heads]
    got_lse = lse[reqs][:, :, heads]
    pu.check_close(got_out, got_lse, ref_out, ref_lse, wl.kv_dtype, what=f"{name} requests {reqs} heads {heads}")
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))


def _plant(wl, b, h0):
    """A cache row at position T_b - 1 of request b whose score with draft s_q - 1, head h0
    is huge: every value is +-the largest magnitude, with the sign of that query."""
    T = int(wl.seq_lens[b])
    page, slot = int(wl.block_table[b, (T - 1) // 64]), (T - 1) % 64
    sign = np.sign(W.bf16_bits_to_float32(wl.q[b, wl.s_q - 1, h0]))
    if wl.kv_dtype == W.KV_BF16:
        row = W._bf16_bits(np.where(sign >= 0, 8.0, -8.0).astype(np.float32))
    else:
        row = np.where(sign >= 0, 0x7E, 0xFE).astype(np.uint8)  # e4m3 +-448
    return page, slot, row


@pytest.mark.parametrize("name", ["agent_spec", "fp8_batch"])
def test_planted_key_at_full_length_reaches_only_the_last_draft(name):
    """At full length a mask error moves an output far less than the tolerance, so the mask
    is checked with a planted key: a huge-score row at position T_b - 1 (visible to draft
    s_q - 1 only).  Every other row of the batch must come out bit-identical to the run
    without it, and the last draft's row must snap to the planted row, as in the oracle."""
    import torch
    import mla_attention_decode_paged_b200 as mla
    wl = W.make_workload(name)
    b = int(np.argmax(wl.seq_lens)) if name == "fp8_batch" else 1
    h0 = 3
    tensors = pu.to_device(wl)
    base_out, base_lse, ws = pu.run_gpu(wl, tensors=tensors, return_ws=True)
    _, _, rs, _ = pu.read_plan(ws)
    assert rs[b + 1] - rs[b] > 1, "the planted request is split over several CTAs"
    page, slot, row = _plant(wl, b, h0)
    kv = tensors[1]
    row_t = torch.from_numpy(row.view(np.int16) if wl.kv_dtype == W.KV_BF16 else row)
    if wl.kv_dtype == W.KV_BF16:
        row_t = row_t.view(torch.bfloat16)
    kv[page, slot] = row_t.to(kv.device)
    out, lse = pu.run_gpu(wl, tensors=tensors)
    last = wl.s_q - 1
    keep = np.ones(out.shape[:3], dtype=bool)
    keep[b, last] = False
    assert np.array_equal(out[keep], base_out[keep]), "a row that cannot see the planted key changed"
    assert np.array_equal(lse[keep], base_lse[keep]), "an lse that cannot see the planted key changed"
    # the last draft of request b against the oracle on the planted cache
    wl.kv[page, slot] = row
    heads = [0, h0, wl.H - 1]
    ref_out, ref_lse = pu.run_oracle(wl, heads=heads, requests=[b])
    pu.check_close(out[[b]][:, :, heads], lse[[b]][:, :, heads], ref_out, ref_lse, wl.kv_dtype, what="planted")
    planted = (W.bf16_bits_to_float32(row) if wl.kv_dtype == W.KV_BF16 else
               np.where(row == 0x7E, 448.0, -448.0) * wl.kv_scale)[:512]
    np.testing.assert_allclose(out[b, last, h0], planted, rtol=2e-2, atol=2e-2)
    # and the earlier drafts of request b stay far from it
    assert np.abs(out[b, :last, h0] - planted).min() > 1.0


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
