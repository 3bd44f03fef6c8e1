"""ctypes binding of libmla_decode.so: the C entry points under the same names.

Argument marshalling only.  Every step of the decode runs in the library's kernels;
there is no fallback: if the shared library is missing or fails to load, every call
raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmla_decode.so")

MLA_OK = 0
MLA_ERR_INVALID_ARG = 1
MLA_ERR_UNSUPPORTED = 2
MLA_ERR_WORKSPACE_TOO_SMALL = 3
MLA_ERR_CUDA = 4
MLA_ERR_DEVICE_OOB = 5
MLA_ERR_DEVICE_TIMEOUT = 6
MLA_ERR_PLAN_MISMATCH = 7
STATUS_NAMES = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED", 3: "MLA_ERR_WORKSPACE_TOO_SMALL",
                4: "MLA_ERR_CUDA", 5: "MLA_ERR_DEVICE_OOB", 6: "MLA_ERR_DEVICE_TIMEOUT",
                7: "MLA_ERR_PLAN_MISMATCH"}
MLA_KV_BF16 = 0
MLA_KV_E4M3 = 1

_lib = None


class MlaError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what} failed: {STATUS_NAMES.get(code, code)}")
        self.code = code


def lib() -> ctypes.CDLL:
    """Load the library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m mla_attention_decode_paged_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, I64, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        L.mla_decode_workspace_size.argtypes = [I, I, I, I]
        L.mla_decode_workspace_size.restype = SZ
        L.mla_decode_plan.argtypes = [P, I, I, I, I, P, SZ, P]
        L.mla_decode_plan.restype = I
        L.mla_decode.argtypes = [P, P, I, F, P, I, P, I, I, I, I64, F, I, P, SZ, P, P, P]
        L.mla_decode.restype = I
        L.mla_decode_scan.argtypes = [P, P, I, F, P, I, P, I, I, I, I64, F, I, P, SZ, P, P, P]
        L.mla_decode_scan.restype = I
        L.mla_decode_noalloc.argtypes = [P, P, I, F, P, I, P, I, I, I, I64, F, I, P, P, P]
        L.mla_decode_noalloc.restype = I
        L.mla_split_kv_combine.argtypes = [P, SZ, I, I, I, P, P, P]
        L.mla_split_kv_combine.restype = I
        L.mla_get_device_status.argtypes = [P, ctypes.POINTER(ctypes.c_int), P]
        L.mla_get_device_status.restype = I
        L.mla_absorb_q.argtypes = [P, P, P, I, I, P, P]
        L.mla_absorb_q.restype = I
        L.mla_project_out.argtypes = [P, P, I, I, P, P]
        L.mla_project_out.restype = I
        L.mla_kv_append.argtypes = [P, P, P, I, P, I, F, P, I, P, I, I, I64, P, P]
        L.mla_kv_append.restype = I
        L.mla_debug_wait_timeout.argtypes = [P, SZ, P]
        L.mla_debug_wait_timeout.restype = I
        L.mla_prefill_sub_chunk.argtypes = [I, I]
        L.mla_prefill_sub_chunk.restype = I
        L.mla_prefill_workspace_size.argtypes = [I, I, I, I, I]
        L.mla_prefill_workspace_size.restype = SZ
        L.mla_prefill.argtypes = [P, P, I, F, P, I, P, I, I, I, I64, F, P, SZ, P, P, P]
        L.mla_prefill.restype = I
        L.mla_decode_version.argtypes = []
        L.mla_decode_version.restype = ctypes.c_char_p
        _lib = L
    return _lib


def mla_decode_workspace_size(B: int, s_q: int, H: int, num_sms: int = 0) -> int:
    return int(lib().mla_decode_workspace_size(B, s_q, H, num_sms))


def mla_decode_plan(seq_lens_ptr: int, B: int, s_q: int, H: int, num_sms: int, workspace_ptr: int,
                    ws_bytes: int, stream: int) -> int:
    return lib().mla_decode_plan(seq_lens_ptr, B, s_q, H, num_sms, workspace_ptr, ws_bytes, stream)


def mla_decode(q_ptr, kv_ptr, kv_dtype, kv_scale, block_table_ptr, max_pages_per_req, seq_lens_ptr, B, s_q, H,
               num_pages, scale, causal, workspace_ptr, ws_bytes, out_ptr, lse_ptr, stream) -> int:
    return lib().mla_decode(q_ptr, kv_ptr, kv_dtype, kv_scale, block_table_ptr, max_pages_per_req, seq_lens_ptr,
                            B, s_q, H, num_pages, scale, int(causal), workspace_ptr, ws_bytes, out_ptr, lse_ptr,
                            stream)


def mla_decode_scan(q_ptr, kv_ptr, kv_dtype, kv_scale, block_table_ptr, max_pages_per_req, seq_lens_ptr, B, s_q,
                    H, num_pages, scale, causal, workspace_ptr, ws_bytes, out_ptr, lse_ptr, stream) -> int:
    return lib().mla_decode_scan(q_ptr, kv_ptr, kv_dtype, kv_scale, block_table_ptr, max_pages_per_req, seq_lens_ptr,
                                 B, s_q, H, num_pages, scale, int(causal), workspace_ptr, ws_bytes, out_ptr, lse_ptr,
                                 stream)


def mla_decode_noalloc(q_ptr, kv_ptr, kv_dtype, kv_scale, block_table_ptr, max_pages_per_req, seq_lens_ptr, B,
                       s_q, H, num_pages, scale, causal, out_ptr, lse_ptr, stream) -> int:
    """mla_decode on the library's static scratch (no workspace argument, no allocation)."""
    return lib().mla_decode_noalloc(q_ptr, kv_ptr, kv_dtype, kv_scale, block_table_ptr, max_pages_per_req,
                                    seq_lens_ptr, B, s_q, H, num_pages, scale, int(causal), out_ptr, lse_ptr, stream)


def mla_split_kv_combine(workspace_ptr, ws_bytes, B, s_q, H, out_ptr, lse_ptr, stream) -> int:
    return lib().mla_split_kv_combine(workspace_ptr, ws_bytes, B, s_q, H, out_ptr, lse_ptr, stream)


def mla_get_device_status(workspace_ptr, stream) -> tuple:
    code = ctypes.c_int(-1)
    rc = lib().mla_get_device_status(workspace_ptr, ctypes.byref(code), stream)
    return rc, code.value


def mla_absorb_q(q_nope_ptr, q_rope_ptr, w_uk_ptr, R, H, q_ptr, stream) -> int:
    return lib().mla_absorb_q(q_nope_ptr, q_rope_ptr, w_uk_ptr, R, H, q_ptr, stream)


def mla_project_out(out_ptr, w_uv_ptr, R, H, y_ptr, stream) -> int:
    return lib().mla_project_out(out_ptr, w_uv_ptr, R, H, y_ptr, stream)


def mla_kv_append(ckv_ptr, kpe_ptr, cos_sin_ptr, max_pos, kv_ptr, kv_dtype, kv_scale, block_table_ptr,
                  max_pages_per_req, seq_lens_ptr, B, s_q, num_pages, status_ptr, stream) -> int:
    return lib().mla_kv_append(ckv_ptr, kpe_ptr, cos_sin_ptr, max_pos, kv_ptr, kv_dtype, kv_scale, block_table_ptr,
                               max_pages_per_req, seq_lens_ptr, B, s_q, num_pages, status_ptr, stream)


def mla_prefill_sub_chunk(chunk: int, H: int) -> int:
    return int(lib().mla_prefill_sub_chunk(chunk, H))


def mla_prefill_workspace_size(B: int, chunk: int, H: int, max_pages_per_req: int, num_sms: int = 0) -> int:
    return int(lib().mla_prefill_workspace_size(B, chunk, H, max_pages_per_req, num_sms))


def mla_prefill(q_ptr, kv_ptr, kv_dtype, kv_scale, block_table_ptr, max_pages_per_req, seq_lens_ptr, B, chunk, H,
                num_pages, scale, workspace_ptr, ws_bytes, out_ptr, lse_ptr, stream) -> int:
    return lib().mla_prefill(q_ptr, kv_ptr, kv_dtype, kv_scale, block_table_ptr, max_pages_per_req, seq_lens_ptr,
                             B, chunk, H, num_pages, scale, workspace_ptr, ws_bytes, out_ptr, lse_ptr, stream)


def mla_debug_wait_timeout(workspace_ptr, ws_bytes, stream) -> int:
    """The scan kernel's bounded wait on a barrier nothing arrives at (20 ms limit)."""
    return lib().mla_debug_wait_timeout(workspace_ptr, ws_bytes, stream)


def mla_decode_version() -> str:
    return lib().mla_decode_version().decode()
