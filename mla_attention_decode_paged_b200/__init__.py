"""Paged, weight-absorbed MLA decode for B200 (sm_100a).

The work happens in ``libmla_decode.so`` (C ABI declared in ``include/mla_decode.h``);
``_abi`` binds its entry points under the same names, and the helpers below only turn
torch CUDA tensors into pointers and sizes.  torch is used for device memory and
streams, nothing else.
"""
from __future__ import annotations

from . import _abi
from ._abi import (MLA_KV_BF16, MLA_KV_E4M3, MlaError, mla_decode_plan, mla_decode_version,
                   mla_decode_workspace_size, mla_get_device_status, mla_kv_append, mla_split_kv_combine,
                   mla_absorb_q, mla_project_out, mla_prefill, mla_prefill_sub_chunk,
                   mla_prefill_workspace_size)

PAGE = 64
DQK = 576
DV = 512


def _stream_ptr(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _check(rc, what):
    if rc != 0:
        raise MlaError(rc, what)


def _kv_dtype(kv_pages):
    import torch
    if kv_pages.dtype == torch.bfloat16:
        return MLA_KV_BF16
    if kv_pages.dtype in (torch.uint8, torch.float8_e4m3fn):
        return MLA_KV_E4M3
    raise TypeError(f"unsupported cache dtype {kv_pages.dtype}")


def workspace_bytes(B: int, s_q: int, H: int, num_sms: int = 0) -> int:
    n = mla_decode_workspace_size(B, s_q, H, num_sms)
    if n == 0:
        raise MlaError(_abi.MLA_ERR_UNSUPPORTED, "mla_decode_workspace_size")
    return n


def alloc_workspace(B: int, s_q: int, H: int, num_sms: int = 0, device=None):
    """A zero-filled uint8 CUDA tensor large enough (and 256-byte aligned) for plan + decode;
    zero-filled so that its status word starts clear."""
    import torch
    n = workspace_bytes(B, s_q, H, num_sms)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def plan(seq_lens, s_q: int, H: int, workspace, num_sms: int = 0, stream=None):
    """Enqueue the split planner for int32 CUDA ``seq_lens`` [B] into ``workspace``."""
    B = int(seq_lens.shape[0])
    _check(mla_decode_plan(seq_lens.data_ptr(), B, s_q, H, num_sms, workspace.data_ptr(), workspace.numel(),
                           _stream_ptr(stream)), "mla_decode_plan")


def decode(q, kv_pages, block_table, seq_lens, scale: float, causal: bool, workspace, out, lse,
           kv_scale: float = 1.0, stream=None, scan_only: bool = False):
    """Enqueue mla_decode (decode + split combine) on torch CUDA tensors.

    q bf16 [B, s_q, H, 576]; kv_pages bf16 or uint8 (e4m3 bytes) / float8_e4m3fn
    [P, 64, 576]; block_table int32 [B, max_pages]; seq_lens int32 [B]; out bf16
    [B, s_q, H, 512]; lse float32 [B, s_q, H].  The plan in ``workspace`` must have
    been made from the same seq_lens.  ``scan_only`` runs the split scan without the
    combine (mla_decode_scan); follow it with ``combine``.
    """
    import torch
    B, s_q, H, d = q.shape
    assert d == DQK and q.dtype == torch.bfloat16 and q.is_contiguous()
    kv_dtype = _kv_dtype(kv_pages)
    assert kv_pages.is_contiguous() and kv_pages.shape[1:] == (PAGE, DQK)
    assert block_table.dtype == torch.int32 and block_table.is_contiguous()
    assert seq_lens.dtype == torch.int32 and out.dtype == torch.bfloat16 and lse.dtype == torch.float32
    fn = _abi.mla_decode_scan if scan_only else _abi.mla_decode
    _check(fn(q.data_ptr(), kv_pages.data_ptr(), kv_dtype, float(kv_scale), block_table.data_ptr(),
              int(block_table.shape[1]), seq_lens.data_ptr(), B, s_q, H, int(kv_pages.shape[0]),
              float(scale), int(bool(causal)), workspace.data_ptr(), workspace.numel(),
              out.data_ptr(), lse.data_ptr(), _stream_ptr(stream)), "mla_decode_scan" if scan_only else "mla_decode")


def combine(workspace, B: int, s_q: int, H: int, out, lse, stream=None):
    _check(mla_split_kv_combine(workspace.data_ptr(), workspace.numel(), B, s_q, H, out.data_ptr(),
                                lse.data_ptr(), _stream_ptr(stream)), "mla_split_kv_combine")


def device_status(workspace, stream=None) -> int:
    """Read and clear the device status word (synchronises the stream)."""
    rc, code = mla_get_device_status(workspace.data_ptr(), _stream_ptr(stream))
    _check(rc, "mla_get_device_status")
    return code


def kv_append(ckv_new, kpe_new, rope_cos_sin, kv_pages, block_table, seq_lens, kv_scale: float = 1.0,
              status=None, stream=None):
    """Write the s_q new latent rows of each request into the paged cache (the draft
    tokens, positions T_b - s_q + i), rotating their rope key (see mla_kv_append in
    include/mla_decode.h).  ckv_new bf16 [B, s_q, 512], kpe_new bf16 [B, s_q, 64],
    rope_cos_sin float32 [max_pos, 64]; kv_pages bf16 or float8_e4m3fn / uint8
    [P, 64, 576]; status: optional int32 CUDA tensor of one element."""
    import torch
    B, s_q, _ = ckv_new.shape
    kv_dtype = MLA_KV_BF16 if kv_pages.dtype == torch.bfloat16 else MLA_KV_E4M3
    _check(mla_kv_append(ckv_new.data_ptr(), kpe_new.data_ptr(), rope_cos_sin.data_ptr(), rope_cos_sin.shape[0],
                         kv_pages.data_ptr(), kv_dtype, float(kv_scale), block_table.data_ptr(), block_table.shape[1],
                         seq_lens.data_ptr(), B, s_q, kv_pages.shape[0],
                         None if status is None else status.data_ptr(), _stream_ptr(stream)), "mla_kv_append")


def absorb_q(q_nope, q_rope, w_uk, q, stream=None):
    """q[..., 0:512] = W_UK[h] q_nope, q[..., 512:576] = q_rope per head (mla_absorb_q).
    q_nope bf16 [B, s_q, H, 128], q_rope bf16 [B, s_q, H, 64], w_uk bf16 [H, 512, 128],
    q bf16 [B, s_q, H, 576]."""
    H = q_nope.shape[-2]
    R = q_nope.numel() // (H * 128)
    _check(mla_absorb_q(q_nope.data_ptr(), q_rope.data_ptr(), w_uk.data_ptr(), R, H, q.data_ptr(),
                        _stream_ptr(stream)), "mla_absorb_q")


def project_out(out, w_uv, y, stream=None):
    """y = out W_UV[h] per head (mla_project_out): out bf16 [B, s_q, H, 512], w_uv bf16
    [H, 512, 128], y bf16 [B, s_q, H, 128]."""
    H = out.shape[-2]
    R = out.numel() // (H * 512)
    _check(mla_project_out(out.data_ptr(), w_uv.data_ptr(), R, H, y.data_ptr(), _stream_ptr(stream)),
           "mla_project_out")


def prefill_workspace_bytes(B: int, chunk: int, H: int, max_pages: int, num_sms: int = 0) -> int:
    n = mla_prefill_workspace_size(B, chunk, H, max_pages, num_sms)
    if n == 0:
        raise MlaError(_abi.MLA_ERR_UNSUPPORTED, "mla_prefill_workspace_size")
    return n


def alloc_prefill_workspace(B: int, chunk: int, H: int, max_pages: int, device=None):
    """A zero-filled uint8 CUDA tensor large enough for mla_prefill."""
    import torch
    return torch.zeros(prefill_workspace_bytes(B, chunk, H, max_pages), dtype=torch.uint8, device=device or "cuda")


def prefill(q, kv_pages, block_table, seq_lens, scale: float, workspace, out, lse, kv_scale: float = 1.0,
            stream=None):
    """Enqueue mla_prefill: the chunk of q.shape[1] query tokens of each request, whose rows
    are the request's last cache rows, attends causally to its paged cache.  q bf16
    [B, chunk, H, 576]; out bf16 [B, chunk, H, 512]; lse float32 [B, chunk, H]; the other
    arguments as for ``decode``; ``workspace`` from ``alloc_prefill_workspace``."""
    import torch
    B, chunk, H, d = q.shape
    assert d == DQK and q.dtype == torch.bfloat16 and q.is_contiguous()
    kv_dtype = _kv_dtype(kv_pages)
    assert kv_pages.is_contiguous() and kv_pages.shape[1:] == (PAGE, DQK)
    assert block_table.dtype == torch.int32 and block_table.is_contiguous()
    assert seq_lens.dtype == torch.int32 and out.dtype == torch.bfloat16 and lse.dtype == torch.float32
    assert out.is_contiguous() and lse.is_contiguous()
    _check(mla_prefill(q.data_ptr(), kv_pages.data_ptr(), kv_dtype, float(kv_scale), block_table.data_ptr(),
                       int(block_table.shape[1]), seq_lens.data_ptr(), B, chunk, H, int(kv_pages.shape[0]),
                       float(scale), workspace.data_ptr(), workspace.numel(), out.data_ptr(), lse.data_ptr(),
                       _stream_ptr(stream)), "mla_prefill")
