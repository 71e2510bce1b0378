"""GPU parity of paged decoding over NVFP4 rows (512 values that are both K
and V; E2M1 codes with UE4M3 block-16 scales, query and cache) against the
oracle run on the dequantised values. Every E2M1 x UE4M3 value is exact in
bf16, so the kernel's inputs to the tensor cores are the oracle's values and
the bar is the one of the BF16 path (out 1e-2, LSE 1e-3, cosine 0.99999),
tighter than the pages' NVFP4 bar (atol 0.1, LSE 0.05), which covers their
FP8 probabilities and requantised V."""
import dataclasses

import numpy as np
import pytest
import torch

import head_latent_attention_get_b200 as M
from head_latent_attention_get_b200 import _capi as C
from tests import gpu_helpers as G
from workloads import mla_workloads as W

pytestmark = pytest.mark.gpu


def _nvfp4(**over):
    base = dataclasses.replace(W.get_workload("tiny"), kv="nvfp4", scale=512 ** -0.5)
    return dataclasses.replace(base, **over)


def _check(inp, where, **kw):
    out, lse, r = G.run_gpu(inp, runner_kwargs=kw)
    ref_o, ref_l = G.oracle_for(inp)
    G.compare(out, lse, ref_o, ref_l, where, inp=inp)
    assert r.status()[0] == C.MLA_OK
    return out, lse


@pytest.mark.parametrize("lens,s_q,h_q,causal,parts", [
    ([70, 129], 1, 16, False, None),
    ([1, 63, 64, 65, 300], 1, 64, False, None),
    ([700, 1500], 1, 128, False, None),            # two row groups per unit
    ([5, 2000, 64], 6, 64, True, None),            # q_len 6 x 64 heads: three 128-row units
    ([900, 4000, 130], 2, 32, True, 7),            # split units
    ([0, 100, 3], 3, 16, True, None),              # empty request, causal rows with no key
])
def test_nvfp4_vs_oracle(lens, s_q, h_q, causal, parts):
    w = _nvfp4(batch=len(lens), seqlens=lens, s_q=s_q, h_q=h_q, causal=causal, seed=7 + sum(lens))
    inp = W.make_inputs(w, poison_tail=True, extra_pages=2)
    _check(inp, f"nvfp4 {lens} s_q={s_q} h_q={h_q}", num_sm_parts=parts)


@pytest.mark.parametrize("parts", [1, 3, 148])
def test_nvfp4_split_counts(parts):
    w = _nvfp4(batch=3, seqlens=[2500, 130, 6000], s_q=6, h_q=16, causal=True, seed=19)
    inp = W.make_inputs(w, poison_tail=True)
    _check(inp, f"nvfp4 parts={parts}", num_sm_parts=parts)


def test_nvfp4_with_sink():
    w = _nvfp4(batch=3, seqlens=[4, 900, 3000], s_q=3, h_q=64, causal=True, seed=23)
    inp = W.with_sink(W.make_inputs(w, poison_tail=True), seed=5)
    for parts in (None, 7):
        _check(inp, f"nvfp4 sink parts={parts}", num_sm_parts=parts)


def test_nvfp4_full_size_every_request():
    """32 requests x 6 query tokens x 64 heads, 8192 NVFP4 tokens each."""
    inp = W.make_inputs(W.get_workload("nvfp4"))
    out, lse, _ = G.run_gpu(inp)
    G.compare_full(inp, out, lse, "nvfp4", few_keys=True)


def test_nvfp4_rejected_for_sparse_and_bad_dims():
    w = _nvfp4(batch=1, seqlens=[64], h_q=16, seed=3)
    inp = W.make_inputs(w)
    d = G.to_device(inp)
    r = M.DecodeRunner(d["q"], d["kcache"], d["block_table"], d["cache_seqlens"], softmax_scale=w.scale,
                       q_scale=d["q_scale"], kv_scale=d["kv_scale"])
    idx = torch.zeros((1, 1, 64), dtype=torch.int32, device="cuda")
    assert C.lib().mla_decode_sparse(C.ctypes.byref(r.args), idx.data_ptr(), 64, None) == C.MLA_ERR_UNSUPPORTED
    r.args.d_qk = 576
    assert C.lib().mla_decode_paged(C.ctypes.byref(r.args), None) == C.MLA_ERR_INVALID_ARG
    r.args.d_qk = 512
    r.args.kv_scale = None
    assert C.lib().mla_decode_paged(C.ctypes.byref(r.args), None) == C.MLA_ERR_INVALID_ARG
