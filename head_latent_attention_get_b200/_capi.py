"""ctypes binding of libmla_b200.so (include/mla.h).

Argument marshalling only: every entry point forwards to the C ABI of the
same name; all computation happens in the library's CUDA kernels. Tensors are
passed by data pointer, streams as the raw cudaStream_t of a torch stream.
Loading fails with an exception if the library is missing: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmla_b200.so")

MLA_OK = 0
MLA_ERR_INVALID_ARG = 1
MLA_ERR_UNSUPPORTED = 2
MLA_ERR_WORKSPACE_TOO_SMALL = 3
MLA_ERR_CUDA = 4
MLA_ERR_DEVICE_TIMEOUT = 5
MLA_ERR_DEVICE_BOUNDS = 6
MLA_KV_BF16 = 0
MLA_KV_FP8_E4M3 = 1
MLA_KV_NVFP4 = 2
MLA_DEVICE_STATUS_TIMEOUT = 1
MLA_DEVICE_STATUS_BOUNDS = 2
MLA_DEBUG_WITHHOLD_SCORES = 1
MLA_DEBUG_SKIP_COMBINE = 2
MLA_TILE_MD_INTS = 8
MLA_MAX_ROWS = 128
MLA_NOALLOC_WORKSPACE_BYTES = 48 << 20


class MLAError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {mla_status_string(code)} ({code})")
        self.code = code


class MlaDecodeArgs(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("kcache", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
        ("cache_seqlens", ctypes.c_void_p), ("tile_md", ctypes.c_void_p), ("num_splits", ctypes.c_void_p),
        ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("batch", ctypes.c_int), ("s_q", ctypes.c_int), ("h_q", ctypes.c_int), ("h_kv", ctypes.c_int),
        ("d_qk", ctypes.c_int), ("d_v", ctypes.c_int), ("page_size", ctypes.c_int),
        ("num_pages", ctypes.c_int), ("block_table_stride", ctypes.c_int), ("num_sm_parts", ctypes.c_int),
        ("softmax_scale", ctypes.c_float), ("causal", ctypes.c_int), ("kv_format", ctypes.c_int),
        ("timeout_ns", ctypes.c_uint64), ("debug_flags", ctypes.c_uint32),
        ("sink", ctypes.c_void_p), ("q_scale", ctypes.c_void_p), ("kv_scale", ctypes.c_void_p),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m head_latent_attention_get_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        i, vp, sz = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
        L.mla_status_string.restype = ctypes.c_char_p
        L.mla_status_string.argtypes = [i]
        L.mla_decode_geometry.restype = i
        L.mla_decode_geometry.argtypes = [i, i, i, i, ctypes.POINTER(i), ctypes.POINTER(i)]
        L.mla_get_num_sm_parts.restype = i
        L.mla_get_num_sm_parts.argtypes = [i, i, i, i, i, ctypes.POINTER(i)]
        L.mla_get_metadata.restype = i
        L.mla_get_metadata.argtypes = [vp, i, i, i, i, i, i, vp, vp, vp]
        L.mla_get_metadata_host.restype = i
        L.mla_get_metadata_host.argtypes = [vp, i, i, i, i, i, i, vp, vp]
        L.mla_workspace_size.restype = sz
        L.mla_workspace_size.argtypes = [i, i, i, i, i, i]
        L.mla_decode_paged.restype = i
        L.mla_decode_paged.argtypes = [ctypes.POINTER(MlaDecodeArgs), vp]
        L.mla_decode_paged_noalloc.restype = i
        L.mla_decode_paged_noalloc.argtypes = [ctypes.POINTER(MlaDecodeArgs), vp]
        L.mla_decode_sparse.restype = i
        L.mla_decode_sparse.argtypes = [ctypes.POINTER(MlaDecodeArgs), vp, i, vp]
        L.mla_combine.restype = i
        L.mla_combine.argtypes = [vp, sz, vp, i, i, i, vp, vp, vp]
        L.mla_combine_sink.restype = i
        L.mla_combine_sink.argtypes = [vp, sz, vp, i, i, i, i, vp, vp, vp, vp]
        L.mla_query_device_status.restype = i
        L.mla_query_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32), vp]
        L.mla_clear_device_status.restype = i
        L.mla_clear_device_status.argtypes = [vp, vp]
        f = ctypes.c_float
        L.mla_q_norm_rope.restype = i
        L.mla_q_norm_rope.argtypes = [vp, vp, i, i, i, i, vp, f, vp, vp, vp]
        L.mla_out_rope_fp8.restype = i
        L.mla_out_rope_fp8.argtypes = [vp, i, i, i, i, vp, vp, vp, vp, vp]
        _lib = L
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(code: int, where: str):
    if code != MLA_OK:
        raise MLAError(code, where)


def mla_status_string(code: int) -> str:
    return lib().mla_status_string(code).decode()


def mla_decode_geometry(s_q: int, h_q: int, h_kv: int = 1, topk: int = 0):
    """(units per request, rows per unit) of a decode problem."""
    upr, rows = ctypes.c_int(0), ctypes.c_int(0)
    _check(lib().mla_decode_geometry(s_q, h_q, h_kv, topk, ctypes.byref(upr), ctypes.byref(rows)),
           "mla_decode_geometry")
    return upr.value, rows.value


def mla_get_num_sm_parts(device: int, s_q: int, h_q: int, h_kv: int = 1, topk: int = 0) -> int:
    out = ctypes.c_int(0)
    _check(lib().mla_get_num_sm_parts(device, s_q, h_q, h_kv, topk, ctypes.byref(out)), "mla_get_num_sm_parts")
    return out.value


def mla_get_metadata(cache_seqlens, batch, s_q, h_q, h_kv, topk, num_sm_parts, tile_md, num_splits,
                     stream=None):
    _check(lib().mla_get_metadata(_ptr(cache_seqlens), batch, s_q, h_q, h_kv, topk, num_sm_parts,
                                  _ptr(tile_md), _ptr(num_splits), _stream(stream)), "mla_get_metadata")


def mla_get_metadata_host(cache_seqlens, batch, s_q, h_q, h_kv, topk, num_sm_parts, tile_md, num_splits):
    """Host pointers (numpy int32 arrays, or CPU tensors)."""
    return lib().mla_get_metadata_host(_ptr(cache_seqlens), batch, s_q, h_q, h_kv, topk, num_sm_parts,
                                       _ptr(tile_md), _ptr(num_splits))


def mla_workspace_size(batch, s_q, h_q, h_kv, topk, num_sm_parts) -> int:
    return lib().mla_workspace_size(batch, s_q, h_q, h_kv, topk, num_sm_parts)


def make_args(*, q, kcache, block_table, cache_seqlens, tile_md, num_splits, out, lse, workspace,
              batch, s_q, h_q, h_kv, num_pages, num_sm_parts, softmax_scale, causal, kv_format,
              block_table_stride=None, d_qk=576, d_v=512, page_size=64, timeout_ns=0, debug_flags=0,
              workspace_bytes=None, sink=None, q_scale=None, kv_scale=None) -> MlaDecodeArgs:
    a = MlaDecodeArgs()
    a.q, a.kcache, a.block_table = _ptr(q), _ptr(kcache), _ptr(block_table)
    a.cache_seqlens, a.tile_md, a.num_splits = _ptr(cache_seqlens), _ptr(tile_md), _ptr(num_splits)
    a.out, a.lse, a.workspace = _ptr(out), _ptr(lse), _ptr(workspace)
    a.workspace_bytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    a.batch, a.s_q, a.h_q, a.h_kv = batch, s_q, h_q, h_kv
    a.d_qk, a.d_v, a.page_size = d_qk, d_v, page_size
    a.num_pages = num_pages
    a.block_table_stride = block_table.shape[-1] if block_table_stride is None else block_table_stride
    a.num_sm_parts = num_sm_parts
    a.softmax_scale = softmax_scale
    a.causal = int(bool(causal))
    a.kv_format = kv_format
    a.timeout_ns = timeout_ns
    a.debug_flags = debug_flags
    a.sink = _ptr(sink)
    a.q_scale = _ptr(q_scale)
    a.kv_scale = _ptr(kv_scale)
    return a


def mla_decode_paged(args: MlaDecodeArgs, stream=None):
    _check(lib().mla_decode_paged(ctypes.byref(args), _stream(stream)), "mla_decode_paged")


def mla_decode_paged_noalloc(args: MlaDecodeArgs, stream=None):
    """Paged decode using the library's built-in workspace (args.workspace must
    be None and args.workspace_bytes 0). For callers that cannot allocate
    device memory at decode time."""
    _check(lib().mla_decode_paged_noalloc(ctypes.byref(args), _stream(stream)), "mla_decode_paged_noalloc")


def mla_decode_sparse(args: MlaDecodeArgs, indices, topk: int, stream=None):
    _check(lib().mla_decode_sparse(ctypes.byref(args), _ptr(indices), topk, _stream(stream)),
           "mla_decode_sparse")


def mla_combine(workspace, workspace_bytes, num_splits, num_units, rows_per_unit, num_sm_parts, out, lse,
                stream=None):
    _check(lib().mla_combine(_ptr(workspace), workspace_bytes, _ptr(num_splits), num_units, rows_per_unit,
                             num_sm_parts, _ptr(out), _ptr(lse), _stream(stream)), "mla_combine")


def mla_combine_sink(workspace, workspace_bytes, num_splits, num_units, rows_per_unit, num_sm_parts, h_q, sink,
                     out, lse, stream=None):
    _check(lib().mla_combine_sink(_ptr(workspace), workspace_bytes, _ptr(num_splits), num_units, rows_per_unit,
                                  num_sm_parts, h_q, _ptr(sink), _ptr(out), _ptr(lse), _stream(stream)),
           "mla_combine_sink")


def mla_query_device_status(workspace, stream=None):
    """Returns (status code, raw bits); blocks until the stream reaches here."""
    bits = ctypes.c_uint32(0)
    code = lib().mla_query_device_status(_ptr(workspace), ctypes.byref(bits), _stream(stream))
    return code, bits.value


def mla_clear_device_status(workspace, stream=None):
    _check(lib().mla_clear_device_status(_ptr(workspace), _stream(stream)), "mla_clear_device_status")


def mla_q_norm_rope(q, q_out, batch, s_q, h_q, d_qk, gamma, eps, rope_cos, rope_sin, stream=None):
    _check(lib().mla_q_norm_rope(_ptr(q), _ptr(q_out), batch, s_q, h_q, d_qk, _ptr(gamma), float(eps),
                                 _ptr(rope_cos), _ptr(rope_sin), _stream(stream)), "mla_q_norm_rope")


def mla_out_rope_fp8(out, batch, s_q, h_q, d_qk, rope_cos, rope_sin, out_fp8, out_scale, stream=None):
    _check(lib().mla_out_rope_fp8(_ptr(out), batch, s_q, h_q, d_qk, _ptr(rope_cos), _ptr(rope_sin),
                                  _ptr(out_fp8), _ptr(out_scale), _stream(stream)), "mla_out_rope_fp8")
