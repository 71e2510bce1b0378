"""GPU parity when block tables alias physical pages, as a paged cache with
prefix sharing produces: requests that share their first pages, a request
that reads one physical page at several logical positions, two requests with
the same table, and a block table with unused padding columns (a row stride
wider than any request needs). The kernels only read the cache, so every row
must match the oracle, which resolves each logical page through the same
table ("Qu'est-ce que FlashMLA ?", paged KV cache with a block table).
"""
import dataclasses

import pytest
import torch

from head_latent_attention_get_b200 import _capi as C
from tests import gpu_helpers as G
from workloads import mla_workloads as W

pytestmark = pytest.mark.gpu

LENS = [1000, 1500, 700, 1000]   # request 0: 15 full pages and a 40-token last page


def _aliased_inputs(kv, h_q, topk):
    over = dict(batch=len(LENS), seqlens=LENS, s_q=1, h_q=h_q, causal=False, kv=kv, topk=topk,
                seed=2024 + h_q + topk)
    if kv == "nvfp4":
        over["scale"] = 512 ** -0.5
    if topk:
        over["neg_frac"] = 0.05
    inp = W.make_inputs(dataclasses.replace(W.get_workload("tiny"), **over), poison_tail=True)
    bt = inp.block_table.clone()
    bt[1, :10] = bt[0, :10]        # a shared 640-token prefix (full pages only)
    bt[2, 0:10:2] = bt[0, 3]       # one full page at five logical positions
    bt[3, :16] = bt[0, :16]        # the same table as request 0 (its last page included)
    pad = torch.full((bt.shape[0], 8), -1, dtype=bt.dtype)
    return dataclasses.replace(inp, block_table=torch.cat([bt, pad], dim=1))


@pytest.mark.parametrize("kv,h_q,topk,kernel", [
    ("bf16", 16, 0, "row group"),
    ("bf16", 128, 0, "CTA pair"),
    ("fp8", 64, 0, "page kernel"),
    ("nvfp4", 64, 0, "page kernel"),
    ("bf16", 128, 2048, "CTA pair, token-sparse"),
])
def test_aliased_pages_vs_oracle(kv, h_q, topk, kernel):
    inp = _aliased_inputs(kv, h_q, topk)
    out, lse, r = G.run_gpu(inp)
    assert r.status()[0] == C.MLA_OK
    ref_o, ref_l = G.oracle_for(inp)
    G.compare(out, lse, ref_o, ref_l, f"aliased pages, {kv} h_q={h_q} topk={topk} ({kernel})", inp=inp)
