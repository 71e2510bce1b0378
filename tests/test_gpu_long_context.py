"""GPU parity at the longest context the pages discuss: a 128K-token KV cache
("[flashinfer] FlashInfer, NVFP4 DeepSeek-V4 decoding", benchmark table: KV
length 128K), on each decode kernel.

A single request of 131072 tokens (1024 tiles) is cut by the scheduler into
as many pieces as there are parts, so these cases also exercise the largest
split count per unit that the combine merges, and the lazily rescaled
accumulator over a thousand tiles. Every output row is compared with the
oracle.
"""
import dataclasses

import numpy as np
import pytest

from head_latent_attention_get_b200 import _capi as C
from tests import gpu_helpers as G
from workloads import mla_workloads as W

pytestmark = pytest.mark.gpu

LONG = 131072


def _workload(kv, lens, s_q, h_q, seed):
    over = dict(batch=len(lens), seqlens=lens, s_q=s_q, h_q=h_q, causal=s_q > 1, seed=seed, kv=kv)
    if kv == "nvfp4":
        over["scale"] = 512 ** -0.5  # the NVFP4 rows are 512 values, K and V alike
    return dataclasses.replace(W.get_workload("tiny"), **over)


@pytest.mark.parametrize("kv,lens,s_q,h_q,kernel", [
    ("bf16", [LONG], 1, 16, "row group"),
    ("bf16", [LONG, 1], 1, 128, "CTA pair"),
    ("fp8", [LONG], 1, 64, "page kernel"),
    ("nvfp4", [LONG], 6, 64, "page kernel, three 128-row units"),
])
def test_128k_context_vs_oracle(kv, lens, s_q, h_q, kernel):
    inp = W.make_inputs(_workload(kv, lens, s_q, h_q, seed=131 + h_q), poison_tail=True)
    out, lse, r = G.run_gpu(inp)
    assert r.status()[0] == C.MLA_OK
    # pieces per unit: about parts / units (148 CTAs, 74 CTA pairs, or 74
    # parts of two row-group CTAs for the NVFP4 rows, over three units)
    splits = np.diff(r.num_splits.cpu().numpy())
    assert splits.max() >= 20, f"the long unit was cut into only {splits.max()} pieces"
    ref_o, ref_l = G.oracle_for(inp)
    G.compare(out, lse, ref_o, ref_l, f"{kv} {lens} s_q={s_q} h_q={h_q} ({kernel})", inp=inp)
