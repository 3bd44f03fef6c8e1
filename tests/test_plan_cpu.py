"""CPU checks of the split-plan logic and of the parity gate itself."""
import numpy as np
import pytest

import oracle
from mla_attention_decode_paged_b200 import workloads as W
from tests import parity_util as pu
from tests import plan_ref


@pytest.mark.parametrize("lens,G", [([65536] * 4, 74), ([256], 74), ([65, 129], 74), ([100, 5000, 64, 1], 3),
                                    (list(np.random.default_rng(0).integers(1, 70000, 32)), 37), ([64] * 10, 1),
                                    (list(np.random.default_rng(1).integers(1, 3000, 600)), 148),
                                    (list(np.random.default_rng(2).integers(1, 200, 1000)), 1023)])
def test_plan_covers_every_page_once_in_order_and_balances(lens, G):
    gb, rs, segs = plan_ref.plan(lens, G)
    tiles = [(t + 63) // 64 for t in lens]
    # every request's segments tile [0, tiles_b) contiguously, in order
    for b, n in enumerate(tiles):
        s = segs[rs[b]:rs[b + 1]]
        assert np.all(s[:, 0] == b)
        assert s[0, 1] == 0 and s[-1, 2] == n
        assert np.all(s[1:, 1] == s[:-1, 2]) and np.all(s[:, 2] > s[:, 1])
        assert np.all(s[:, 3] == (len(s) > 1))
    # shares differ by at most one page
    work = [int((segs[gb[g]:gb[g + 1], 2] - segs[gb[g]:gb[g + 1], 1]).sum()) for g in range(G)]
    assert sum(work) == sum(tiles)
    assert max(work) - min(work) <= 1
    assert len(segs) <= len(lens) + G
    assert np.all(np.diff(gb) >= 0) and gb[-1] == len(segs)


def test_rel_l2_gate_rejects_an_all_zero_output():
    """Negative controls: an all-zero output and a run with the causal mask switched off
    must both fail the gate that the parity tests apply."""
    wl = W.make_workload("agent_spec", B=1, seq=("fixed", 4096))
    out, lse = oracle.mla_decode(wl.q, wl.kv, wl.kv_dtype, wl.kv_scale, wl.block_table, wl.seq_lens, wl.scale, True)
    zeros = np.zeros_like(out)
    with pytest.raises(AssertionError):
        pu.check_close(zeros, lse, out, lse, W.KV_BF16)
    # a causal mask turned off also fails
    out_nc, lse_nc = oracle.mla_decode(wl.q, wl.kv, wl.kv_dtype, wl.kv_scale, wl.block_table, wl.seq_lens,
                                       wl.scale, False)
    with pytest.raises(AssertionError):
        pu.check_close(out_nc, lse_nc, out, lse, W.KV_BF16)
    pu.check_close(out.astype(np.float32), lse.astype(np.float32), out, lse, W.KV_BF16)
