"""The C-ABI library on the host: it loads, exports every declared entry
point, and rejects bad arguments before launching anything (CPU only)."""
import ctypes
import os
import re

import numpy as np
import pytest

import head_latent_attention_get_b200 as M
from head_latent_attention_get_b200 import _capi as C
from tests import sched_checks as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for f in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if f.endswith(".h"):
            text = open(os.path.join(ROOT, "include", f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_library_exports_every_declared_function():
    names = declared_functions()
    assert "mla_decode_paged" in names and "mla_get_metadata" in names and len(names) >= 10
    L = C.lib()
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing


def test_status_strings():
    for code in range(7):
        assert M.mla_status_string(code).startswith("MLA_")
    assert M.mla_status_string(99) == "MLA_ERR_UNKNOWN"


def test_workspace_size_layout():
    # header 256 + lse [(U+P) x R] f32 (256-aligned) + o [(U+P) x R x 512] f32
    U, R, P = 64, 128, 74
    lse = (U + P) * R * 4
    o_off = -(-(256 + lse) // 256) * 256
    total = -(-(o_off + (U + P) * R * 512 * 4) // 256) * 256
    assert M.mla_workspace_size(64, 1, 128, 1, 0, 74) == total
    assert M.mla_workspace_size(32, 1, 128, 1, 2048, 74) == M.mla_workspace_size(32, 1, 128, 1, 0, 74)
    assert M.mla_workspace_size(0, 1, 16, 1, 0, 10) == 0


def _fake_args(**over):
    # non-null, 16-byte aligned fake device pointers: only host checks run
    base = dict(q=None, kcache=None, block_table=None, cache_seqlens=None, tile_md=None, num_splits=None,
                out=None, lse=None, workspace=None)
    a = C.MlaDecodeArgs()
    for i, k in enumerate(base):
        setattr(a, k, 0x100000 * (i + 1))
    a.workspace_bytes = 1 << 40
    a.batch, a.s_q, a.h_q, a.h_kv = 2, 1, 16, 1
    a.d_qk, a.d_v, a.page_size = 576, 512, 64
    a.num_pages, a.block_table_stride, a.num_sm_parts = 8, 4, 148
    a.softmax_scale, a.causal, a.kv_format = 1 / 24, 0, C.MLA_KV_BF16
    for k, v in over.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("over,code", [
    (dict(q=None), C.MLA_ERR_INVALID_ARG),
    (dict(out=0x100008), C.MLA_ERR_INVALID_ARG),              # misaligned
    (dict(d_qk=512), C.MLA_ERR_INVALID_ARG),
    (dict(d_v=576), C.MLA_ERR_INVALID_ARG),
    (dict(page_size=128), C.MLA_ERR_INVALID_ARG),
    (dict(batch=0), C.MLA_ERR_INVALID_ARG),
    (dict(kv_format=7), C.MLA_ERR_INVALID_ARG),
    (dict(softmax_scale=float("nan")), C.MLA_ERR_INVALID_ARG),
    (dict(h_kv=2, h_q=32), C.MLA_ERR_UNSUPPORTED),
    (dict(s_q=1 << 11, h_q=1 << 10), C.MLA_ERR_UNSUPPORTED),  # more than 2^20 rows per request
    (dict(workspace_bytes=1024), C.MLA_ERR_WORKSPACE_TOO_SMALL),
    (dict(sink=0x300002), C.MLA_ERR_INVALID_ARG),             # misaligned sink
])
def test_decode_rejects_bad_arguments(over, code):
    a = _fake_args(**over)
    assert C.lib().mla_decode_paged(ctypes.byref(a), None) == code


def test_sparse_rejects_bad_topk_and_rows():
    a = _fake_args()
    L = C.lib()
    assert L.mla_decode_sparse(ctypes.byref(a), 0x200000, 100, None) == C.MLA_ERR_INVALID_ARG
    assert L.mla_decode_sparse(ctypes.byref(a), None, 128, None) == C.MLA_ERR_INVALID_ARG
    assert L.mla_decode_paged(None, None) == C.MLA_ERR_INVALID_ARG
    a256 = _fake_args(h_q=256)                        # sparse units are one query token: <= 128 rows
    assert L.mla_decode_sparse(ctypes.byref(a256), 0x200000, 128, None) == C.MLA_ERR_UNSUPPORTED


def test_metadata_rejects_bad_arguments():
    L = C.lib()
    assert L.mla_get_metadata(0x1000, 2, 1, 16, 1, 0, 0, 0x2000, 0x3000, None) == C.MLA_ERR_INVALID_ARG
    assert L.mla_get_metadata(0x1000, 2, 1, 16, 1, 100, 8, 0x2000, 0x3000, None) == C.MLA_ERR_INVALID_ARG
    assert L.mla_get_metadata(None, 2, 1, 16, 1, 0, 8, 0x2000, 0x3000, None) == C.MLA_ERR_INVALID_ARG
    assert L.mla_get_metadata(0x1000, 2, 1, 16, 2, 0, 8, 0x2000, 0x3000, None) == C.MLA_ERR_UNSUPPORTED
    assert L.mla_combine(None, 0, None, 1, 1, 1, None, None, None) == C.MLA_ERR_INVALID_ARG
    ws, ns, out, lse, sink = 0x100000, 0x200000, 0x300000, 0x400000, 0x500000
    big = 1 << 40
    for h_q, sk in ((0, sink), (16, sink + 2)):   # h_q <= 0, misaligned
        assert L.mla_combine_sink(ws, big, ns, 4, 32, 8, h_q, sk, out, lse, None) == C.MLA_ERR_INVALID_ARG
    assert L.mla_combine_sink(ws, 1024, ns, 4, 32, 8, 16, sink, out, lse, None) == C.MLA_ERR_WORKSPACE_TOO_SMALL
    assert L.mla_query_device_status(None, None, None) == C.MLA_ERR_INVALID_ARG


@pytest.mark.parametrize("s_q,h_q,topk,expect", [
    (1, 128, 0, (1, 128)), (2, 16, 0, (1, 32)), (6, 16, 0, (1, 96)), (6, 64, 0, (3, 128)),
    (3, 64, 0, (2, 96)), (1, 256, 0, (2, 128)), (3, 43, 0, (3, 43)), (5, 32, 0, (2, 80)),
    (4, 128, 0, (4, 128)), (2, 128, 2048, (2, 128)), (3, 64, 128, (3, 64)),
])
def test_decode_geometry(s_q, h_q, topk, expect):
    assert M.mla_decode_geometry(s_q, h_q, 1, topk) == expect
    assert S.units_per_request(s_q, h_q, topk) == expect[0]
    U, R = expect[0], expect[1]
    lse = (U + 8) * R * 4
    o_off = -(-(256 + lse) // 256) * 256
    assert M.mla_workspace_size(1, s_q, h_q, 1, topk, 8) == -(-(o_off + (U + 8) * R * 512 * 4) // 256) * 256


def test_decode_geometry_rejects():
    L = C.lib()
    a, b = ctypes.c_int(0), ctypes.c_int(0)
    assert L.mla_decode_geometry(1, 256, 1, 128, ctypes.byref(a), ctypes.byref(b)) == C.MLA_ERR_UNSUPPORTED
    assert L.mla_decode_geometry(1 << 11, 1 << 10, 1, 0, ctypes.byref(a), ctypes.byref(b)) == C.MLA_ERR_UNSUPPORTED
    assert L.mla_decode_geometry(1, 16, 2, 0, ctypes.byref(a), ctypes.byref(b)) == C.MLA_ERR_UNSUPPORTED
    assert L.mla_decode_geometry(0, 16, 1, 0, ctypes.byref(a), ctypes.byref(b)) == C.MLA_ERR_INVALID_ARG
    assert L.mla_decode_geometry(1, 16, 1, 0, None, ctypes.byref(b)) == C.MLA_ERR_INVALID_ARG


def host_schedule(seqlens, batch, s_q, h_q, topk, parts):
    U = batch * M.mla_decode_geometry(s_q, h_q, 1, topk)[0]
    md = np.zeros(parts * 8, dtype=np.int32)
    ns = np.zeros(U + 1, dtype=np.int32)
    sl = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
    assert M.mla_get_metadata_host(sl, batch, s_q, h_q, 1, topk, parts, md, ns) == 0
    return md, ns


@pytest.mark.parametrize("case", [
    ("tiny", [70, 129], 1, 16, 0, 148),
    ("dsv3", [4096] * 64, 1, 128, 0, 74),
    ("single", [65536], 2, 16, 0, 148),
    ("zeros", [0, 5, 0, 0, 300, 0], 1, 16, 0, 7),
    ("all_zero", [0, 0, 0], 1, 16, 0, 5),
    ("more_parts_than_tiles", [1, 2, 3], 1, 64, 0, 148),
    ("sparse", [32768] * 32, 1, 128, 2048, 74),
    ("sparse_sq2", [4096] * 3, 2, 64, 192, 11),
    ("mtp6_64heads", [4096, 300, 0, 9000], 6, 64, 0, 74),
    ("rows96_blocks", [70, 129, 5000], 3, 64, 0, 74),
    ("256heads", [4096] * 8, 1, 256, 0, 74),
    ("equal_units_two_pieces", [32768] * 32, 1, 128, 2048, 74),
    ("equal_units_odd_steps", [300] * 7, 1, 100, 0, 40),
    ("equal_units_more_parts_than_steps", [200] * 3, 1, 128, 0, 148),
    ("equal_units_64_rows_cost_axis", [32768] * 32, 1, 64, 2048, 148),
])
def test_host_scheduler_invariants(case):
    _, lens, s_q, h_q, topk, parts = case
    md, ns = host_schedule(lens, len(lens), s_q, h_q, topk, parts)
    S.check_schedule(md, ns, lens, len(lens), s_q, topk, parts, h_q=h_q)


def test_host_scheduler_random_and_mtp():
    rng = np.random.default_rng(3)
    for _ in range(40):
        B = int(rng.integers(1, 300))
        lens = rng.integers(0, 20000, size=B)
        lens[rng.random(B) < 0.1] = 0
        parts = int(rng.integers(1, 160))
        md, ns = host_schedule(lens, B, 1, 16, 0, parts)
        S.check_schedule(md, ns, lens, B, 1, 0, parts)
    from workloads import mla_workloads as W
    w = W.get_workload("mtp")
    md, ns = host_schedule(w.seqlens, w.batch, 2, 16, 0, 148)
    info = S.check_schedule(md, ns, w.seqlens, w.batch, 2, 0, 148)
    assert info["splits"] <= w.batch + 148


def test_args_struct_layout_matches_header(tmp_path):
    """The ctypes mirror of mla_decode_args has the C compiler's size and
    field offsets (gcc on the header itself)."""
    fields = [f for f, _ in C.MlaDecodeArgs._fields_]
    src = tmp_path / "layout.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "mla.h"\nint main(void) {\n'
                   '  printf("%zu\\n", sizeof(mla_decode_args));\n'
                   + "".join(f'  printf("%zu\\n", offsetof(mla_decode_args, {f}));\n' for f in fields)
                   + "  return 0;\n}\n")
    exe = tmp_path / "layout"
    import subprocess
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = [int(x) for x in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()]
    assert got[0] == ctypes.sizeof(C.MlaDecodeArgs)
    assert got[1:] == [getattr(C.MlaDecodeArgs, f).offset for f in fields]


def test_decode_geometry_is_the_fewest_equal_blocks():
    """For every s_q <= 8 and h_q <= 300: blocks tile the request's rows
    exactly, hold at most 128 rows, and no smaller block count would do."""
    for s_q in range(1, 9):
        for h_q in range(1, 301, 7):
            upr, rows = M.mla_decode_geometry(s_q, h_q, 1, 0)
            R = s_q * h_q
            assert upr * rows == R and rows <= 128
            assert all(R % n or R // n > 128 for n in range(1, upr))


def test_host_scheduler_random_shapes_with_row_blocks():
    """Random batches, query tokens, heads (1..300, so up to 18 row-block
    units per request), sparse or paged, and part counts: every schedule is
    an exact cover with consistent split counts and balanced parts."""
    rng = np.random.default_rng(11)
    for _ in range(60):
        B = int(rng.integers(1, 40))
        s_q = int(rng.integers(1, 9))
        h_q = int(rng.integers(1, 301))
        sparse = bool(rng.random() < 0.3) and h_q <= 128
        topk = 64 * int(rng.integers(1, 6)) if sparse else 0
        lens = rng.integers(0, 9000, size=B)
        parts = int(rng.integers(1, 160))
        md, ns = host_schedule(lens, B, s_q, h_q, topk, parts)
        S.check_schedule(md, ns, lens, B, s_q, topk, parts, h_q=h_q)


def test_pre_post_steps_validate_arguments_on_the_host():
    """mla_q_norm_rope / mla_out_rope_fp8 reject bad arguments before any
    launch (fake, aligned device pointers: nothing is dereferenced)."""
    L = C.lib()
    q, qo, g, cs, sn = 0x100000, 0x200000, 0x300000, 0x400000, 0x500000
    assert L.mla_q_norm_rope(q, qo, 2, 1, 16, 600, g, 1e-6, cs, sn, None) == C.MLA_ERR_INVALID_ARG
    assert L.mla_q_norm_rope(q + 8, qo, 2, 1, 16, 576, g, 1e-6, cs, sn, None) == C.MLA_ERR_INVALID_ARG
    assert L.mla_q_norm_rope(q, qo, 2, 1, 16, 576, g + 4, 1e-6, cs, sn, None) == C.MLA_ERR_INVALID_ARG
    assert L.mla_q_norm_rope(q, qo, 2, 1, 16, 576, None, 1e-6, cs, sn, None) == C.MLA_ERR_INVALID_ARG
    assert L.mla_q_norm_rope(q, qo, 2, 1, 16, 576, g, -1.0, cs, sn, None) == C.MLA_ERR_INVALID_ARG
    assert L.mla_q_norm_rope(q, qo, 0, 1, 16, 576, g, 1e-6, cs, sn, None) == C.MLA_ERR_INVALID_ARG
    o, o8, sc = 0x100000, 0x200000, 0x300000
    assert L.mla_out_rope_fp8(o, 2, 1, 16, 512, None, None, o8, sc, None) == C.MLA_ERR_INVALID_ARG
    assert L.mla_out_rope_fp8(o, 2, 1, 16, 500, cs, sn, o8, sc, None) == C.MLA_ERR_INVALID_ARG
    assert L.mla_out_rope_fp8(o, 2, 1, 16, 576, None, None, o8 + 4, sc, None) == C.MLA_ERR_INVALID_ARG
    assert L.mla_out_rope_fp8(o, 2, 1, 16, 576, None, None, o8, sc + 2, None) == C.MLA_ERR_INVALID_ARG
    assert L.mla_out_rope_fp8(None, 2, 1, 16, 576, None, None, o8, sc, None) == C.MLA_ERR_INVALID_ARG
