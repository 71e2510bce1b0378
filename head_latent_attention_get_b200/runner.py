"""Buffer plumbing around the C ABI for one decode problem.

PyTorch only allocates device memory here; the scheduler, decode and combine
all run inside libmla_b200.so. Mirrors the plan-once / run-per-layer shape of
the paged MLA decode APIs (metadata computed once per decode step and reused
by every layer: "Qu'est-ce que FlashMLA ?", section "Exécuter le décodage
MLA").
"""
from __future__ import annotations

import torch

from . import _capi as C


class DecodeRunner:
    def __init__(self, q, kcache, block_table, cache_seqlens, *, softmax_scale, causal=False,
                 indices=None, num_sm_parts=None, timeout_ns=0, debug_flags=0, sink=None, q_scale=None,
                 kv_scale=None):
        """q bf16 [B, s_q, h_q, 576] with a bf16 or FP8-record cache, or (NVFP4)
        packed uint8 [B, s_q, h_q, 256] with q_scale/kv_scale and a packed
        uint8 [pages, 64, 256] cache."""
        dev = q.device
        assert dev.type == "cuda", "the decode path runs on a CUDA device only"
        self.batch, self.s_q, self.h_q, d = q.shape
        self.topk = int(indices.shape[-1]) if indices is not None else 0
        if q.dtype == torch.uint8:
            assert d == 256 and kcache.shape[-1] == 256 and q_scale is not None and kv_scale is not None
            self.kv_format, d_qk = C.MLA_KV_NVFP4, 512
        else:
            assert d == 576
            self.kv_format = C.MLA_KV_BF16 if kcache.dtype == torch.bfloat16 else C.MLA_KV_FP8_E4M3
            d_qk = 576
        self.q_scale, self.kv_scale = q_scale, kv_scale
        upr, self.rows = C.mla_decode_geometry(self.s_q, self.h_q, 1, self.topk)
        self.units = self.batch * upr
        self.parts = num_sm_parts or C.mla_get_num_sm_parts(dev.index or 0, self.s_q, self.h_q, 1, self.topk)
        self.tile_md = torch.empty(self.parts * C.MLA_TILE_MD_INTS, dtype=torch.int32, device=dev)
        self.num_splits = torch.empty(self.units + 1, dtype=torch.int32, device=dev)
        ws_bytes = C.mla_workspace_size(self.batch, self.s_q, self.h_q, 1, self.topk, self.parts)
        self.workspace = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
        self.out = torch.empty(self.batch, self.s_q, self.h_q, 512, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(self.batch, self.s_q, self.h_q, dtype=torch.float32, device=dev)
        self.q, self.kcache, self.block_table, self.cache_seqlens = q, kcache, block_table, cache_seqlens
        self.indices = indices
        if sink is not None:
            assert sink.device == dev and sink.dtype == torch.float32 and sink.shape == (self.h_q,)
            sink = sink.contiguous()
        self.sink = sink
        self.args = C.make_args(
            q=q, kcache=kcache, block_table=block_table, cache_seqlens=cache_seqlens,
            tile_md=self.tile_md, num_splits=self.num_splits, out=self.out, lse=self.lse,
            workspace=self.workspace, batch=self.batch, s_q=self.s_q, h_q=self.h_q, h_kv=1,
            num_pages=kcache.shape[0], num_sm_parts=self.parts, softmax_scale=softmax_scale,
            causal=causal, kv_format=self.kv_format, timeout_ns=timeout_ns, debug_flags=debug_flags,
            sink=sink, d_qk=d_qk, q_scale=q_scale, kv_scale=kv_scale)

    def plan(self, stream=None):
        C.mla_get_metadata(self.cache_seqlens, self.batch, self.s_q, self.h_q, 1, self.topk, self.parts,
                           self.tile_md, self.num_splits, stream)

    def run(self, stream=None):
        if self.topk:
            C.mla_decode_sparse(self.args, self.indices, self.topk, stream)
        else:
            C.mla_decode_paged(self.args, stream)
        return self.out, self.lse

    def status(self, stream=None):
        return C.mla_query_device_status(self.workspace, stream)
