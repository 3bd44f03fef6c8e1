"""The seeded workload generator: deterministic, the documented shapes and length
distributions, NaN canaries where no request may read, and values exact in their
storage type.  CPU only (small overrides of each workload)."""
import numpy as np
import pytest

from mla_attention_decode_paged_b200 import workloads as W


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_same_seed_same_bytes_and_documented_shapes(name):
    a = W.make_workload(name, B=2, seq=("fixed", 130))
    b = W.make_workload(name, B=2, seq=("fixed", 130))
    assert np.array_equal(a.q, b.q) and np.array_equal(a.kv, b.kv)  # bit patterns
    assert np.array_equal(a.block_table, b.block_table) and a.kv_scale == b.kv_scale
    spec = W.WORKLOADS[name]
    assert a.q.shape == (2, spec.s_q, spec.H, W.DQK)
    assert a.kv.shape[1:] == (W.PAGE, W.DQK)
    assert a.kv.dtype == (np.uint16 if spec.kv_dtype == W.KV_BF16 else np.uint8)
    c = W.make_workload(name, B=2, seq=("fixed", 130), seed=spec.seed + 100)
    assert not np.array_equal(a.q, c.q)


def test_full_size_length_distributions():
    assert np.all(W.make_workload("agent_spec", chunk_pages=4096, seq=("fixed", 64)).seq_lens == 64)
    lens = W.draw_seq_lens(W.WORKLOADS["ragged_rownorm"], np.random.default_rng(0))
    assert lens.min() >= 32768 and lens.max() <= 65536
    lens = W.draw_seq_lens(W.dataclasses.replace(W.WORKLOADS["fp8_batch"], B=4000), np.random.default_rng(0))
    assert lens.min() >= 512 and lens.max() <= 65536
    assert 6000 < np.median(lens) < 11000   # median 8192 before clipping


def test_canaries_sit_exactly_where_no_request_reads():
    wl = W.make_workload("agent_spec", B=3, seq_lens=[100, 64, 1])
    nan = W.BF16_NAN
    used = set()
    for b, T in enumerate(wl.seq_lens):
        for t in range(int(T)):
            pg = wl.block_table[b, t // W.PAGE]
            used.add((int(pg), t % W.PAGE))
            assert not np.any(wl.kv[pg, t % W.PAGE] == nan)
    for pg in range(wl.kv.shape[0]):
        for r in range(W.PAGE):
            if (pg, r) not in used:
                assert np.all(wl.kv[pg, r] == nan)
    # block-table slots past a request's pages hold -1
    assert wl.block_table[1, 1] == -1 and wl.block_table[2, 1] == -1


def test_e4m3_pool_scale_and_range():
    wl = W.make_workload("fp8_batch", B=2, seq=("fixed", 300))
    vals = wl.kv[wl.kv != W.E4M3_NAN]
    assert wl.kv_scale > 0
    # the largest magnitude in the pool maps to (about) the largest finite e4m3 value
    mags = vals & 0x7F
    assert mags.max() in (0x7E, 0x7D)
