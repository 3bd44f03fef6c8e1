"""Shared helpers of the parity tests: run the CUDA library on a workload and compare
with the float64 oracle.

Tolerances (from the target spec of this path): max |out - ref| <= 2e-2 + 2e-2 |ref|
for a bf16 cache (5e-2 + 5e-2 |ref| for e4m3) and |lse - ref| <= 1e-3.  Because
near-uniform attention over tens of thousands of tokens gives outputs of magnitude
~1e-2, the absolute bound alone would accept an all-zero output, so the tests also
gate the relative L2 error ||out - ref|| / ||ref|| <= 1e-2 (bf16) / 3e-2 (e4m3), and a
negative control shows that gate rejects zeros.
"""
from __future__ import annotations

import numpy as np

import oracle
from mla_attention_decode_paged_b200 import workloads as W

TOL = {W.KV_BF16: dict(atol=2e-2, rtol=2e-2, rel_l2=1e-2), W.KV_E4M3: dict(atol=5e-2, rtol=5e-2, rel_l2=3e-2)}
LSE_ATOL = 1e-3


def check_close(out_gpu, lse_gpu, out_ref, lse_ref, kv_dtype, what=""):
    """Element-wise bound, rel-L2 gate and lse bound; returns the error summary."""
    t = TOL[kv_dtype]
    out_gpu = np.asarray(out_gpu, dtype=np.float64)
    lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
    assert out_gpu.shape == out_ref.shape, (out_gpu.shape, out_ref.shape)
    assert np.all(np.isfinite(out_gpu)), f"{what}: non-finite output"
    assert np.all(np.isfinite(lse_gpu)), f"{what}: non-finite lse"
    err = np.abs(out_gpu - out_ref)
    bound = t["atol"] + t["rtol"] * np.abs(out_ref)
    worst = float((err / bound).max())
    rel_l2 = float(np.linalg.norm(out_gpu - out_ref) / max(np.linalg.norm(out_ref), 1e-300))
    lse_err = float(np.abs(lse_gpu - lse_ref).max())
    summary = dict(max_abs=float(err.max()), worst_ratio=worst, rel_l2=rel_l2, lse_err=lse_err)
    assert worst <= 1.0, f"{what}: element bound exceeded {summary}"
    assert rel_l2 <= t["rel_l2"], f"{what}: relative L2 {summary}"
    assert lse_err <= LSE_ATOL, f"{what}: lse {summary}"
    return summary


def to_device(wl, device="cuda"):
    import torch
    q = torch.from_numpy(wl.q.view(np.int16)).view(torch.bfloat16).to(device)
    if wl.kv_dtype == W.KV_BF16:
        kv = torch.from_numpy(wl.kv.view(np.int16)).view(torch.bfloat16).to(device)
    else:
        kv = torch.from_numpy(wl.kv).to(device)
    bt = torch.from_numpy(wl.block_table).to(device)
    sl = torch.from_numpy(wl.seq_lens).to(device)
    return q, kv, bt, sl


def run_gpu(wl, num_sms: int = 0, device="cuda", tensors=None, check_status=True, return_ws=False):
    """Plan + decode on the GPU; returns (out float32 numpy, lse numpy), and the workspace
    tensor (which holds the plan) when ``return_ws``."""
    import torch
    import mla_attention_decode_paged_b200 as mla
    q, kv, bt, sl = tensors if tensors is not None else to_device(wl, device)
    ws = mla.alloc_workspace(wl.B, wl.s_q, wl.H, num_sms=num_sms, device=device)
    out = torch.full((wl.B, wl.s_q, wl.H, W.DV), float("nan"), dtype=torch.bfloat16, device=device)
    lse = torch.full((wl.B, wl.s_q, wl.H), float("nan"), dtype=torch.float32, device=device)
    mla.plan(sl, wl.s_q, wl.H, ws, num_sms=num_sms)
    mla.decode(q, kv, bt, sl, wl.scale, wl.causal, ws, out, lse, kv_scale=wl.kv_scale)
    torch.cuda.synchronize()
    if check_status:
        code = mla.device_status(ws)
        assert code == 0, f"device status {code}"
    if return_ws:
        return out.float().cpu().numpy(), lse.cpu().numpy(), ws
    return out.float().cpu().numpy(), lse.cpu().numpy()


def read_plan(ws):
    """The plan in a workspace, read back to the host: (header int32 words, group -> first
    segment, request -> first segment, segments [n, 4] = (b, first page, end page, split))."""
    raw = ws.cpu().numpy()
    h32 = raw[:48].view(np.int32)
    h64 = raw[48:96].view(np.int64)
    G, nseg, B = int(h32[7]), int(h32[8]), int(h32[3])
    gb = raw[h64[0]:h64[0] + 4 * (G + 1)].view(np.int32)
    rs = raw[h64[1]:h64[1] + 4 * (B + 1)].view(np.int32)
    segs = raw[h64[2]:h64[2] + 16 * nseg].view(np.int32).reshape(-1, 4)
    return h32, gb, rs, segs


def run_oracle(wl, heads=None, requests=None):
    """Oracle on the whole workload, or on a subset of requests and heads."""
    q = wl.q
    bt, sl = wl.block_table, wl.seq_lens
    if requests is not None:
        q, bt, sl = q[requests], bt[requests], sl[requests]
    if heads is not None:
        q = q[:, :, heads]
    return oracle.mla_decode(q, wl.kv, wl.kv_dtype, wl.kv_scale, bt, sl, wl.scale, wl.causal)
