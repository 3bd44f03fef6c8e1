"""Float64 CPU oracle for paged, weight-absorbed MLA decode.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package; the product library never
does.  It shares no code with the CUDA path.  ``build()`` compiles ``mla_oracle.c``
with the system C compiler (plain C + OpenMP).

Every function here follows the definitions written at the top of
``mla_oracle.c`` (paging from llm-atlas "Inference systems" 07 PagedAttention,
absorbed attention over a 512 + 64 latent row from the zhaifeiyue TokenSpeed notes'
DeepSeek-V3 entry, draft-token visibility from llm-atlas 16 Speculative decoding,
split partials and their LSE combination from "Faster kernels, slower engine" 7.1).

Pins (tests/test_oracle_pins.py) tie each function to something other than itself:
un-absorbed multi-head attention through a library SDPA, closed forms, page
permutation and split invariance, and the e4m3 table of a library float8 type.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mla_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libmla_oracle.so")
_lock = threading.Lock()
_lib = None

KV_BF16 = 0
KV_E4M3 = 1
PAGE = 64
DQK = 576
DV = 512


def build(force: bool = False) -> str:
    """Compile the oracle shared library (gcc, -O2, OpenMP, IEEE arithmetic)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off", "-o", tmp, _SRC,
               "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
            lib.oracle_mla_decode_range.argtypes = [P, P, i32, f64, P, i32, P, i32, i32, i32,
                                                    i64, i32, f64, i32, P, P, P, P]
            lib.oracle_mla_decode_range.restype = ctypes.c_int
            lib.oracle_combine.argtypes = [P, P, i32, i64, P, P]
            lib.oracle_combine.restype = None
            lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
            lib.oracle_e4m3_to_double.restype = f64
            lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_bf16_to_double.restype = f64
            lib.oracle_rope_table.argtypes = [i32, f64, P]
            lib.oracle_rope_table.restype = None
            lib.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
            lib.oracle_f32_to_bf16.restype = ctypes.c_uint16
            lib.oracle_f32_to_e4m3.argtypes = [ctypes.c_float]
            lib.oracle_f32_to_e4m3.restype = ctypes.c_uint8
            lib.oracle_kv_append.argtypes = [P, P, P, i32, P, i32, ctypes.c_float, P, i32, P, i32, i32, i64, i32]
            lib.oracle_kv_append.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def mla_decode(q_bits, kv, kv_dtype, kv_scale, block_table, seq_lens, scale, causal,
               tok_lo=None, tok_hi=None, page=PAGE):
    """Float64 reference of the paged absorbed-MLA decode.

    q_bits: uint16 [B, s_q, H, 576] (bf16 bit patterns); kv: uint16 (bf16 bits) or
    uint8 (e4m3 bytes) [P, page, 576]; block_table int32 [B, max_pages]; seq_lens int32
    [B].  Optional tok_lo / tok_hi int32 [B] restrict each request to the token window
    [tok_lo, tok_hi) (a split).  Returns (out float64 [B, s_q, H, 512], lse float64
    [B, s_q, H]).
    """
    lib = _load()
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    B, s_q, H, d = q_bits.shape
    assert d == DQK
    kv = np.ascontiguousarray(kv)
    assert kv.dtype == (np.uint16 if kv_dtype == KV_BF16 else np.uint8)
    assert kv.shape[1] == page and kv.shape[2] == DQK
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    lo = None if tok_lo is None else np.ascontiguousarray(tok_lo, dtype=np.int32)
    hi = None if tok_hi is None else np.ascontiguousarray(tok_hi, dtype=np.int32)
    out = np.zeros((B, s_q, H, DV), dtype=np.float64)
    lse = np.zeros((B, s_q, H), dtype=np.float64)
    rc = lib.oracle_mla_decode_range(_ptr(q_bits), _ptr(kv), int(kv_dtype), float(kv_scale),
                                     _ptr(bt), int(bt.shape[1]), _ptr(sl), B, s_q, H,
                                     int(kv.shape[0]), int(page), float(scale), int(bool(causal)),
                                     _ptr(lo), _ptr(hi), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (code {rc})")
    return out, lse


def mla_prefill(q_bits, kv, kv_dtype, kv_scale, block_table, seq_lens, scale, page=PAGE):
    """Float64 reference of long-prefix chunked prefill over the paged cache (the prefill
    workloads with a long-prefix KV cache of the "TokenSpeed" launch digest, MLA kernel
    paragraphs).  The chunk of C = q_bits.shape[1] query tokens of request b are its last C
    cache rows (seq_lens counts them); chunk token i, at position T_b - C + i, sees the
    cached tokens t <= T_b - C + i.  That is the visibility rule of the decode definition
    with s_q = C under the causal flag, so the result is that definition evaluated with
    s_q = C.  Returns (out float64 [B, C, H, 512], lse float64 [B, C, H])."""
    return mla_decode(q_bits, kv, kv_dtype, kv_scale, block_table, seq_lens, scale, True, page=page)


def combine(outs, lses):
    """LSE-weighted combination of partial results: outs [n, ..., 512], lses [n, ...]."""
    lib = _load()
    outs = np.ascontiguousarray(outs, dtype=np.float64)
    lses = np.ascontiguousarray(lses, dtype=np.float64)
    n = outs.shape[0]
    rows = int(np.prod(lses.shape[1:])) if lses.ndim > 1 else 1
    out = np.zeros(outs.shape[1:], dtype=np.float64)
    lse = np.zeros(lses.shape[1:], dtype=np.float64)
    lib.oracle_combine(_ptr(outs), _ptr(lses), n, rows, _ptr(out), _ptr(lse))
    return out, lse


def e4m3_to_double(byte: int) -> float:
    return _load().oracle_e4m3_to_double(int(byte) & 0xFF)


def bf16_to_double(bits: int) -> float:
    return _load().oracle_bf16_to_double(int(bits) & 0xFFFF)


def rope_table(max_pos: int, base: float = 10000.0):
    """float32 [max_pos, 64]: cos(pos * base^(-2j/64)) for j < 32, then the sines."""
    t = np.zeros((max_pos, 64), dtype=np.float32)
    _load().oracle_rope_table(int(max_pos), float(base), _ptr(t))
    return t


def f32_to_bf16(x: float) -> int:
    return int(_load().oracle_f32_to_bf16(float(x)))


def f32_to_e4m3(x: float) -> int:
    return int(_load().oracle_f32_to_e4m3(float(x)))


def kv_append(ckv_bits, kpe_bits, cos_sin, kv, kv_dtype, kv_scale, block_table, seq_lens, page=PAGE):
    """Reference of the paged KV append, in place on a copy of ``kv`` (returned).

    ckv_bits uint16 [B, s_q, 512] and kpe_bits uint16 [B, s_q, 64] (bf16 bit patterns);
    cos_sin float32 [max_pos, 64]; kv uint16 / uint8 [P, page, 576].  Raises on a length
    or page id out of range.
    """
    lib = _load()
    ckv_bits = np.ascontiguousarray(ckv_bits, dtype=np.uint16)
    kpe_bits = np.ascontiguousarray(kpe_bits, dtype=np.uint16)
    B, s_q, d = ckv_bits.shape
    assert d == DV and kpe_bits.shape == (B, s_q, 64)
    cs = np.ascontiguousarray(cos_sin, dtype=np.float32)
    out = np.array(kv, copy=True, order="C")
    assert out.dtype == (np.uint16 if kv_dtype == KV_BF16 else np.uint8)
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    rc = lib.oracle_kv_append(_ptr(ckv_bits), _ptr(kpe_bits), _ptr(cs), int(cs.shape[0]), _ptr(out), int(kv_dtype),
                              float(kv_scale), _ptr(bt), int(bt.shape[1]), _ptr(sl), B, s_q, int(out.shape[0]),
                              int(page))
    if rc != 0:
        raise ValueError("oracle rejected a length or page id")
    return out


def absorb_q(q_nope, q_rope, w_uk):
    """Float64 reference of the query absorption: q[..., :512] = W_UK[h] q_nope (per head),
    q[..., 512:] = q_rope.  q_nope [..., H, 128], q_rope [..., H, 64], w_uk [H, 512, 128]
    (any real dtype; computed in float64 with a library matmul)."""
    qn = np.asarray(q_nope, dtype=np.float64)
    w = np.asarray(w_uk, dtype=np.float64)
    qa = np.einsum("hcd,...hd->...hc", w, qn)
    return np.concatenate([qa, np.asarray(q_rope, dtype=np.float64)], axis=-1)


def project_out(out, w_uv):
    """Float64 reference of the output projection: y = out W_UV[h] per head.
    out [..., H, 512], w_uv [H, 512, 128]."""
    return np.einsum("...hc,hcd->...hd", np.asarray(out, dtype=np.float64), np.asarray(w_uv, dtype=np.float64))
