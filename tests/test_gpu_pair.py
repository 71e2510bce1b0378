"""GPU parity of the CTA-pair decode path (units of 65-128 query rows, BF16
paged cache) against the oracle: ragged tile counts (a pair step whose second
tile lies past the piece), empty requests, partially filled row halves,
causal rows, split counts, run-to-run determinism and the timeout path."""
import dataclasses

import numpy as np
import pytest

from head_latent_attention_get_b200 import _capi as C
from tests import gpu_helpers as G
from workloads import mla_workloads as W

pytestmark = pytest.mark.gpu


def _dense(**kw):
    return dataclasses.replace(W.get_workload("tiny"), **kw)


@pytest.mark.parametrize("lens,s_q,h_q,causal", [
    ([1], 1, 128, False),                                   # one tile: the odd CTA's tile is empty
    ([127, 128, 129, 255, 256, 257, 385], 1, 128, False),   # odd and even tile counts, partial pages
    ([0, 300, 0, 64], 1, 128, False),                       # empty requests
    ([4000, 65], 1, 96, False),                             # odd CTA holds 32 of its 64 rows
    ([2049, 3000, 1], 1, 80, False),                        # odd CTA holds 16 rows
    ([5, 700, 1030], 2, 64, True),                          # 128 rows = 2 query tokens x 64 heads
])
def test_pair_shapes_vs_oracle(lens, s_q, h_q, causal):
    w = _dense(batch=len(lens), seqlens=lens, s_q=s_q, h_q=h_q, causal=causal, seed=101 + sum(lens))
    inp = W.make_inputs(w, poison_tail=True, extra_pages=2)
    out, lse, r = G.run_gpu(inp)
    ref_o, ref_l = G.oracle_for(inp)
    G.compare(out, lse, ref_o, ref_l, f"pair {lens} s_q={s_q} h_q={h_q}")
    assert r.status()[0] == C.MLA_OK


@pytest.mark.parametrize("parts", [1, 2, 3, 7, 74])
def test_pair_split_counts_vs_oracle(parts):
    w = _dense(batch=3, seqlens=[900, 4000, 130], h_q=128, seed=7)
    inp = W.make_inputs(w, poison_tail=True)
    out, lse, r = G.run_gpu(inp, runner_kwargs={"num_sm_parts": parts})
    ref_o, ref_l = G.oracle_for(inp)
    G.compare(out, lse, ref_o, ref_l, f"pair parts={parts}")
    assert r.status()[0] == C.MLA_OK


def test_pair_is_deterministic():
    w = _dense(batch=4, seqlens=[3000, 17, 1500, 2222], h_q=128, seed=8)
    inp = W.make_inputs(w, poison_tail=True)
    o1, l1, _ = G.run_gpu(inp)
    o2, l2, _ = G.run_gpu(inp)
    assert np.array_equal(o1.view(np.uint32), o2.view(np.uint32))
    assert np.array_equal(l1.view(np.uint32), l2.view(np.uint32))


def test_pair_timeout_status_and_context_survives():
    w = _dense(batch=2, seqlens=[700, 1300], h_q=128, seed=9)
    inp = W.make_inputs(w)
    _, _, r = G.run_gpu(inp, runner_kwargs={"timeout_ns": 20_000_000,
                                            "debug_flags": C.MLA_DEBUG_WITHHOLD_SCORES})
    code, bits = r.status()
    assert code == C.MLA_ERR_DEVICE_TIMEOUT and bits & C.MLA_DEVICE_STATUS_TIMEOUT
    out, lse, r2 = G.run_gpu(inp)
    ref_o, ref_l = G.oracle_for(inp)
    G.compare(out, lse, ref_o, ref_l, "pair after timeout")
    assert r2.status()[0] == C.MLA_OK
