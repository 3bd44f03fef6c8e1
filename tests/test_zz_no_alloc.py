"""mla_decode_noalloc: the entry point for callers that cannot allocate device memory
(a plugin inside a runtime that owns all device memory, or a path that cannot afford
cudaMalloc's implicit synchronisation).  It runs on the library's static scratch array
instead of a caller workspace.

Checked through the C ABI, on two calls in a row (the second call finds the first
call's leftovers in the shared scratch), against the float64 oracle and against
mla_decode with a caller workspace, within the parity tolerances.  This file is
collected last on purpose.
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


def _noalloc(wl, tensors, out, lse):
    import torch
    from mla_attention_decode_paged_b200 import _abi
    q, kv, bt, sl = tensors
    rc = _abi.mla_decode_noalloc(q.data_ptr(), kv.data_ptr(), wl.kv_dtype, float(wl.kv_scale), bt.data_ptr(),
                                 int(bt.shape[1]), sl.data_ptr(), wl.B, wl.s_q, wl.H, int(kv.shape[0]),
                                 float(wl.scale), int(wl.causal), out.data_ptr(), lse.data_ptr(),
                                 int(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, f"mla_decode_noalloc returned {rc}"
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("name,kw", [("agent_spec", dict(B=3, seq=("fixed", 2000))),
                                     ("fp8_batch", dict(B=4, seq=("lognormal", 500, 1.0, 65, 3000)))])
def test_noalloc_matches_the_oracle_and_the_workspace_entry_point_on_two_calls_in_a_row(name, kw):
    import torch
    wl = W.make_workload(name, **kw)
    tensors = pu.to_device(wl)
    ws_out, ws_lse = pu.run_gpu(wl, tensors=tensors)
    ref_out, ref_lse = pu.run_oracle(wl)
    for call in range(2):
        out = torch.full((wl.B, wl.s_q, wl.H, W.DV), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((wl.B, wl.s_q, wl.H), float("nan"), dtype=torch.float32, device="cuda")
        got_out, got_lse = _noalloc(wl, tensors, out, lse)
        pu.check_close(got_out, got_lse, ref_out, ref_lse, wl.kv_dtype, what=f"noalloc call {call} vs the oracle")
        pu.check_close(got_out, got_lse, ws_out.astype(np.float64), ws_lse.astype(np.float64), wl.kv_dtype,
                       what=f"noalloc call {call} vs mla_decode")


def test_noalloc_rejects_a_shape_beyond_its_scratch():
    import torch
    from mla_attention_decode_paged_b200 import _abi
    B, s_q, H = 4096, 16, 16  # partials alone would need far more than the 48 MiB scratch
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    p = dummy.data_ptr()
    rc = _abi.mla_decode_noalloc(p, p, 0, 1.0, p, 1, p, B, s_q, H, 1, 0.07, 1, p, p,
                                 int(torch.cuda.current_stream().cuda_stream))
    assert rc == _abi.MLA_ERR_WORKSPACE_TOO_SMALL
