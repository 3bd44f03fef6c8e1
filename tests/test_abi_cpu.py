"""CPU checks of the C ABI: the library loads, exports every declared entry point, sizes
workspaces, and rejects bad arguments on the host before touching a device."""
import ctypes
import os
import re

import numpy as np
import pytest

import mla_attention_decode_paged_b200 as mla
from mla_attention_decode_paged_b200 import _abi
from mla_attention_decode_paged_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    build_mod.build(quiet=True)


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(mla_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_entry_point():
    names = declared_functions()
    assert {"mla_decode", "mla_decode_plan", "mla_split_kv_combine", "mla_decode_workspace_size",
            "mla_get_device_status"} <= set(names)
    L = ctypes.CDLL(_abi.LIB_PATH)
    for n in names:
        assert hasattr(L, n), f"{n} declared but not exported"


def test_version_string():
    assert "sm_100a" in mla.mla_decode_version()


def test_workspace_size_is_pure_host_and_grows_with_shape():
    a = mla.mla_decode_workspace_size(4, 4, 16, 148)
    b = mla.mla_decode_workspace_size(16, 16, 16, 148)
    assert a > 0 and b > a
    assert a % 256 == 0
    # partials: (B + groups) x row blocks x 128 rows x 512 fp32 at least
    assert b >= (16 + 37) * 2 * 128 * 512 * 4
    assert mla.mla_decode_workspace_size(0, 4, 16, 148) == 0
    assert mla.mla_decode_workspace_size(4, -1, 16, 148) == 0
    # the planner keeps two int64 per request in shared memory (at most 200 KB): beyond about
    # 12,700 requests the shape is unsupported, and the size says so
    assert mla.mla_decode_workspace_size(12000, 1, 16, 148) > 0
    assert mla.mla_decode_workspace_size(13000, 1, 16, 148) == 0


def _decode_args(**kw):
    a = dict(q_ptr=16, kv_ptr=16, kv_dtype=0, kv_scale=1.0, block_table_ptr=16, max_pages_per_req=4,
             seq_lens_ptr=16, B=2, s_q=4, H=16, num_pages=8, scale=0.07, causal=1, workspace_ptr=256,
             ws_bytes=1 << 30, out_ptr=16, lse_ptr=16, stream=None)
    a.update(kw)
    return a


@pytest.mark.parametrize("kw,code", [
    (dict(q_ptr=None), _abi.MLA_ERR_INVALID_ARG),
    (dict(out_ptr=None), _abi.MLA_ERR_INVALID_ARG),
    (dict(B=0), _abi.MLA_ERR_INVALID_ARG),
    (dict(num_pages=0), _abi.MLA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), _abi.MLA_ERR_INVALID_ARG),
    (dict(kv_dtype=3), _abi.MLA_ERR_UNSUPPORTED),
    (dict(kv_dtype=1, kv_scale=0.0), _abi.MLA_ERR_INVALID_ARG),
    (dict(kv_dtype=1, kv_scale=float("inf")), _abi.MLA_ERR_INVALID_ARG),
    (dict(s_q=17, H=16), _abi.MLA_ERR_UNSUPPORTED),
    (dict(q_ptr=18), _abi.MLA_ERR_INVALID_ARG),
    (dict(workspace_ptr=272), _abi.MLA_ERR_INVALID_ARG),
    (dict(ws_bytes=1024), _abi.MLA_ERR_WORKSPACE_TOO_SMALL),
])
def test_decode_rejects_bad_arguments_before_any_launch(kw, code):
    a = _decode_args(**kw)
    assert _abi.mla_decode(*a.values()) == code


def test_plan_rejects_bad_arguments():
    assert _abi.mla_decode_plan(None, 2, 4, 16, 148, 256, 1 << 30, None) == _abi.MLA_ERR_INVALID_ARG
    assert _abi.mla_decode_plan(16, 2, 4, 16, 148, 256, 1024, None) == _abi.MLA_ERR_WORKSPACE_TOO_SMALL
    assert _abi.mla_decode_plan(16, 2, 4, 16, -1, 256, 1 << 30, None) == _abi.MLA_ERR_INVALID_ARG
    assert _abi.mla_decode_plan(16, 2, 4, 16, 148, 300, 1 << 30, None) == _abi.MLA_ERR_INVALID_ARG


def test_combine_rejects_bad_arguments():
    assert _abi.mla_split_kv_combine(None, 1 << 30, 2, 4, 16, 16, 16, None) == _abi.MLA_ERR_INVALID_ARG
    assert _abi.mla_split_kv_combine(256, 1 << 30, 2, 32, 16, 16, 16, None) == _abi.MLA_ERR_UNSUPPORTED
    assert _abi.mla_split_kv_combine(256, 16, 2, 4, 16, 16, 16, None) == _abi.MLA_ERR_WORKSPACE_TOO_SMALL


def test_status_query_rejects_null():
    rc, _ = _abi.mla_get_device_status(None, None)
    assert rc == _abi.MLA_ERR_INVALID_ARG


def test_timeout_probe_rejects_bad_workspace_before_any_launch():
    assert _abi.mla_debug_wait_timeout(None, 1 << 20, None) == _abi.MLA_ERR_INVALID_ARG
    assert _abi.mla_debug_wait_timeout(256 + 16, 1 << 20, None) == _abi.MLA_ERR_INVALID_ARG  # not 256-aligned
    assert _abi.mla_debug_wait_timeout(256, 64, None) == _abi.MLA_ERR_WORKSPACE_TOO_SMALL


def test_kv_append_rejects_bad_arguments_before_any_launch():
    ok = dict(ckv=256, kpe=256, cs=256, max_pos=100, kv=256, dt=0, scale=1.0, bt=256, mp=4, sl=256, B=2, s_q=4,
              P=10, status=None)

    def call(**kw):
        a = dict(ok, **kw)
        return _abi.mla_kv_append(a["ckv"], a["kpe"], a["cs"], a["max_pos"], a["kv"], a["dt"], a["scale"], a["bt"],
                                  a["mp"], a["sl"], a["B"], a["s_q"], a["P"], a["status"], None)
    assert call(ckv=None) == _abi.MLA_ERR_INVALID_ARG
    assert call(B=0) == _abi.MLA_ERR_INVALID_ARG
    assert call(max_pos=0) == _abi.MLA_ERR_INVALID_ARG
    assert call(dt=7) == _abi.MLA_ERR_INVALID_ARG
    assert call(dt=1, scale=0.0) == _abi.MLA_ERR_INVALID_ARG
    assert call(ckv=256 + 8) == _abi.MLA_ERR_INVALID_ARG  # latent rows need 16-byte alignment
    assert call(status=256 + 2) == _abi.MLA_ERR_INVALID_ARG


def test_absorb_and_project_reject_bad_arguments_before_any_launch():
    assert _abi.mla_absorb_q(None, 256, 256, 4, 16, 256, None) == _abi.MLA_ERR_INVALID_ARG
    assert _abi.mla_absorb_q(256, 256, 256, 0, 16, 256, None) == _abi.MLA_ERR_INVALID_ARG
    assert _abi.mla_absorb_q(256, 256, 256, 4, 16, 256 + 8, None) == _abi.MLA_ERR_INVALID_ARG  # q needs 16 B
    assert _abi.mla_project_out(256, None, 4, 16, 256, None) == _abi.MLA_ERR_INVALID_ARG
    assert _abi.mla_project_out(256, 256, 4, 0, 256, None) == _abi.MLA_ERR_INVALID_ARG
    assert _abi.mla_project_out(256, 256, 4, 16, 256 + 2, None) == _abi.MLA_ERR_INVALID_ARG


@pytest.mark.parametrize("chunk,H,d", [(24, 16, 12), (1000, 16, 8), (7, 128, 1), (64, 8, 32), (4096, 128, 2),
                                       (16, 16, 16), (1, 1, 1), (256, 1, 256), (5, 300, 0), (0, 16, 0)])
def test_prefill_sub_chunk_examples(chunk, H, d):
    assert mla.mla_prefill_sub_chunk(chunk, H) == d


def test_prefill_sub_chunk_is_the_cheapest_divisor():
    rng = np.random.default_rng(0)
    for _ in range(300):
        chunk, H = int(rng.integers(1, 3000)), int(rng.integers(1, 257))
        d = mla.mla_prefill_sub_chunk(chunk, H)
        divs = [e for e in range(1, chunk + 1) if chunk % e == 0 and e * H <= 256]
        cost = {e: (chunk // e) * -(-(e * H) // 64) for e in divs}
        assert d == max(e for e in divs if cost[e] == min(cost.values())), (chunk, H, d)


def test_prefill_workspace_holds_the_decode_workspace_and_the_copied_tables():
    B, chunk, H, mp = 3, 24, 16, 40
    d = mla.mla_prefill_sub_chunk(chunk, H)
    n = chunk // d
    ws = mla.mla_prefill_workspace_size(B, chunk, H, mp, 148)
    assert ws % 256 == 0
    assert ws >= mla.mla_decode_workspace_size(B * n, d, H, 148) + 4 * B * n * (mp + 1)
    assert mla.mla_prefill_workspace_size(B, chunk, 300, mp, 148) == 0
    assert mla.mla_prefill_workspace_size(0, chunk, H, mp, 148) == 0
    assert mla.mla_prefill_workspace_size(B, chunk, H, 0, 148) == 0
    # more sub-chunk requests than the planner takes
    assert mla.mla_prefill_workspace_size(20000, 7, 64, mp, 148) == 0


def test_prefill_rejects_bad_arguments_before_any_launch():
    ok = dict(q=256, kv=256, dt=0, ks=1.0, bt=256, mp=4, sl=256, B=2, chunk=8, H=16, P=8, scale=0.07, ws=256,
              wsb=1 << 30, out=256, lse=256)

    def call(**kw):
        a = dict(ok, **kw)
        return _abi.mla_prefill(*a.values(), None)
    assert call(q=None) == _abi.MLA_ERR_INVALID_ARG
    assert call(sl=None) == _abi.MLA_ERR_INVALID_ARG
    assert call(chunk=0) == _abi.MLA_ERR_INVALID_ARG
    assert call(P=0) == _abi.MLA_ERR_INVALID_ARG
    assert call(scale=float("inf")) == _abi.MLA_ERR_INVALID_ARG
    assert call(dt=3) == _abi.MLA_ERR_UNSUPPORTED
    assert call(dt=1, ks=-1.0) == _abi.MLA_ERR_INVALID_ARG
    assert call(H=300) == _abi.MLA_ERR_UNSUPPORTED
    assert call(q=256 + 8) == _abi.MLA_ERR_INVALID_ARG
    assert call(sl=256 + 2) == _abi.MLA_ERR_INVALID_ARG
    assert call(ws=256 + 16) == _abi.MLA_ERR_INVALID_ARG
