"""Plan + decode recorded once in a CUDA graph and replayed on new inputs.

The C ABI allocates, frees and synchronises nothing inside mla_decode_plan / mla_decode,
so both can be captured; what a replay reads is whatever the buffers hold at replay
time. Two batches of the same shapes (different lengths, block tables, q and cache
values) are written in place into one set of buffers; each replay of the same graph must
match the float64 oracle on the batch it found there.
"""
import numpy as np
import pytest

from mla_attention_decode_paged_b200 import workloads as W
from tests import parity_util as pu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,kw", [
    ("agent_spec", dict(B=3, seq=("uniform", 300, 2500))),
    ("fp8_batch", dict(B=4, seq=("lognormal", 300, 1.0, 65, 2000))),
])
def test_plan_and_decode_replayed_from_a_graph_on_new_inputs(name, kw):
    import torch
    import mla_attention_decode_paged_b200 as mla
    from mla_attention_decode_paged_b200 import build
    build.build(quiet=True)
    batches = [W.make_workload(name, seed=11, **kw), W.make_workload(name, seed=12, **kw)]
    # one kv scale for both (it is a launch argument, fixed in the graph): the second
    # batch's bytes are read at the first's scale, by the oracle too
    batches[1].kv_scale = batches[0].kv_scale
    wl0 = batches[0]
    P = max(w.kv.shape[0] for w in batches)
    MP = max(w.block_table.shape[1] for w in batches)
    dev = "cuda"
    q = torch.empty(wl0.q.shape, dtype=torch.bfloat16, device=dev)
    kv = torch.empty((P,) + wl0.kv.shape[1:], dtype=torch.bfloat16 if wl0.kv_dtype == W.KV_BF16 else torch.uint8,
                     device=dev)
    bt = torch.empty((wl0.B, MP), dtype=torch.int32, device=dev)
    sl = torch.empty((wl0.B,), dtype=torch.int32, device=dev)
    ws = mla.alloc_workspace(wl0.B, wl0.s_q, wl0.H, device=dev)
    out = torch.empty((wl0.B, wl0.s_q, wl0.H, W.DV), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((wl0.B, wl0.s_q, wl0.H), dtype=torch.float32, device=dev)

    def load(wl):
        # in place: the graph holds these buffers' addresses
        qd, kvd, btd, sld = pu.to_device(wl, dev)
        q.copy_(qd)
        kv.zero_()
        kv[:kvd.shape[0]].copy_(kvd)
        bt.fill_(-1)
        bt[:, :btd.shape[1]].copy_(btd)
        sl.copy_(sld)
        out.fill_(float("nan"))
        lse.fill_(float("nan"))

    def step(stream):
        mla.plan(sl, wl0.s_q, wl0.H, ws, stream=stream)
        mla.decode(q, kv, bt, sl, wl0.scale, wl0.causal, ws, out, lse, kv_scale=wl0.kv_scale, stream=stream)

    load(wl0)
    step(torch.cuda.current_stream())  # eager once: per-device attributes and the tensor map are set
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=cap):
        step(cap)
    torch.cuda.synchronize()
    for wl in batches + batches[:1]:
        load(wl)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        assert mla.device_status(ws) == 0
        ref_out, ref_lse = pu.run_oracle(wl)
        pu.check_close(out.float().cpu().numpy().reshape(ref_out.shape), lse.cpu().numpy(), ref_out, ref_lse,
                       wl.kv_dtype, what=f"graph replay {name} seed {wl.spec.seed}")
