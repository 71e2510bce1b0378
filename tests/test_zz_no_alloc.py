"""mla_decode_paged_noalloc: paged decoding for callers that cannot allocate
device memory when they decode (the split-KV workspace lives in a built-in
device array instead of a caller buffer).

Called through the C ABI twice in a row and compared with mla_decode_paged on
the same inputs: it runs the same kernels on the same schedule, so the outputs
must agree bit for bit; both are also held to the oracle within the parity
tolerances of the other GPU tests. This file is collected last so that a run
stopping at the first failure has already run every other test; it also
passes on its own in a fresh process.
"""
import dataclasses

import numpy as np
import pytest
import torch

import head_latent_attention_get_b200 as M
from head_latent_attention_get_b200 import _capi as C
from tests import gpu_helpers as G
from workloads import mla_workloads as W

pytestmark = pytest.mark.gpu


def _case():
    w = dataclasses.replace(W.get_workload("dsv3"), batch=6, seqlens=[4096, 70, 1000, 129, 3000, 1],
                            seed=4242)
    return W.make_inputs(w, poison_tail=True)


def test_noalloc_matches_workspace_entry_point_twice():
    inp = _case()
    d = G.to_device(inp)
    w = inp.workload
    ref = M.DecodeRunner(d["q"], d["kcache"], d["block_table"], d["cache_seqlens"], softmax_scale=w.scale)
    ref.plan()
    out_ref, lse_ref = ref.run()
    torch.cuda.synchronize()
    out_ref = out_ref.float().cpu().numpy()
    lse_ref = lse_ref.cpu().numpy()

    out = torch.empty_like(ref.out)
    lse = torch.empty_like(ref.lse)
    args = C.make_args(q=d["q"], kcache=d["kcache"], block_table=d["block_table"],
                       cache_seqlens=d["cache_seqlens"], tile_md=ref.tile_md, num_splits=ref.num_splits,
                       out=out, lse=lse, workspace=None, workspace_bytes=0, batch=w.batch, s_q=w.s_q,
                       h_q=w.h_q, h_kv=1, num_pages=inp.num_pages, num_sm_parts=ref.parts,
                       softmax_scale=w.scale, causal=w.causal, kv_format=C.MLA_KV_BF16)
    ref_o, ref_l = G.oracle_for(inp)
    G.compare(out_ref, lse_ref, ref_o, ref_l, "workspace entry point vs oracle")
    for call in range(2):
        out.fill_(float("nan"))
        lse.fill_(float("nan"))
        C.mla_decode_paged_noalloc(args)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref.out.view(torch.int16)), f"noalloc call {call}: out bits"
        assert torch.equal(lse.view(torch.int32), ref.lse.view(torch.int32)), f"noalloc call {call}: lse bits"
        G.compare(out.float().cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, f"noalloc call {call} vs oracle")


def test_noalloc_out_of_range_page_leaves_other_requests_exact():
    """A page id outside the cache is skipped on the device (no fault); the
    requests that do not use it still match the oracle exactly as before."""
    inp = _case()
    inp.block_table[0, 3] = inp.num_pages + 11
    d = G.to_device(inp)
    w = inp.workload
    plan = M.DecodeRunner(d["q"], d["kcache"], d["block_table"], d["cache_seqlens"], softmax_scale=w.scale)
    plan.plan()
    out = torch.empty_like(plan.out)
    lse = torch.empty_like(plan.lse)
    args = C.make_args(q=d["q"], kcache=d["kcache"], block_table=d["block_table"],
                       cache_seqlens=d["cache_seqlens"], tile_md=plan.tile_md, num_splits=plan.num_splits,
                       out=out, lse=lse, workspace=None, workspace_bytes=0, batch=w.batch, s_q=w.s_q,
                       h_q=w.h_q, h_kv=1, num_pages=inp.num_pages, num_sm_parts=plan.parts,
                       softmax_scale=w.scale, causal=w.causal, kv_format=C.MLA_KV_BF16)
    C.mla_decode_paged_noalloc(args)
    torch.cuda.synchronize()
    keep = list(range(1, w.batch))
    ref_o, ref_l = G.oracle_for(G.restrict(inp, keep))
    G.compare(out[1:].float().cpu().numpy(), lse[1:].cpu().numpy(), ref_o, ref_l, "noalloc, other requests")


def test_noalloc_rejects_a_workspace_and_oversized_problems():
    inp = _case()
    d = G.to_device(inp)
    w = inp.workload
    ref = M.DecodeRunner(d["q"], d["kcache"], d["block_table"], d["cache_seqlens"], softmax_scale=w.scale)
    common = dict(q=d["q"], kcache=d["kcache"], block_table=d["block_table"], cache_seqlens=d["cache_seqlens"],
                  tile_md=ref.tile_md, num_splits=ref.num_splits, out=ref.out, lse=ref.lse, s_q=1,
                  h_q=w.h_q, h_kv=1, num_pages=inp.num_pages, softmax_scale=w.scale, causal=False,
                  kv_format=C.MLA_KV_BF16)
    with_ws = C.make_args(workspace=ref.workspace, batch=w.batch, num_sm_parts=ref.parts, **common)
    with pytest.raises(C.MLAError) as e:
        C.mla_decode_paged_noalloc(with_ws)
    assert e.value.code == C.MLA_ERR_INVALID_ARG
    # a batch whose split-KV partials cannot fit in the built-in array
    huge = C.make_args(workspace=None, workspace_bytes=0, batch=4096, num_sm_parts=148, **common)
    assert M.mla_workspace_size(4096, 1, 128, 1, 0, 148) > C.MLA_NOALLOC_WORKSPACE_BYTES
    with pytest.raises(C.MLAError) as e:
        C.mla_decode_paged_noalloc(huge)
    assert e.value.code == C.MLA_ERR_WORKSPACE_TOO_SMALL
