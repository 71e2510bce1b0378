"""GPU parity at row counts the named workloads do not reach: a single row,
counts that are not multiples of 16, 65 rows (one row in the second CTA of
a pair or row group), and 127; on every cache format."""
import dataclasses

import pytest

from head_latent_attention_get_b200 import _capi as C
from tests import gpu_helpers as G
from workloads import mla_workloads as W

pytestmark = pytest.mark.gpu


def _check(inp, where, **kw):
    out, lse, r = G.run_gpu(inp, runner_kwargs=kw)
    ref_o, ref_l = G.oracle_for(inp)
    G.compare(out, lse, ref_o, ref_l, where, inp=inp)
    assert r.status()[0] == C.MLA_OK


@pytest.mark.parametrize("h_q,s_q,causal", [(1, 1, False), (7, 1, False), (33, 2, True), (65, 1, False),
                                            (100, 1, False), (127, 1, False), (1, 5, True)])
def test_bf16_odd_rows(h_q, s_q, causal):
    w = dataclasses.replace(W.get_workload("tiny"), batch=3, seqlens=[1, 200, 1500], h_q=h_q, s_q=s_q,
                            causal=causal, seed=h_q + 17 * s_q)
    inp = W.make_inputs(w, poison_tail=True, extra_pages=1)
    _check(inp, f"bf16 h_q={h_q} s_q={s_q}")
    _check(inp, f"bf16 h_q={h_q} s_q={s_q} split", num_sm_parts=5)


@pytest.mark.parametrize("kv,h_q", [("fp8", 65), ("fp8", 7), ("nvfp4", 65), ("nvfp4", 1)])
def test_quantised_odd_rows(kv, h_q):
    base = dataclasses.replace(W.get_workload("tiny"), kv=kv, batch=2, seqlens=[130, 900], h_q=h_q, seed=h_q + 3)
    if kv == "nvfp4":
        base = dataclasses.replace(base, scale=512 ** -0.5)
    inp = W.make_inputs(base, poison_tail=True)
    _check(inp, f"{kv} h_q={h_q}")


@pytest.mark.parametrize("kv,h_q", [("bf16", 65), ("bf16", 1), ("fp8", 65), ("fp8", 100)])
def test_sparse_odd_rows(kv, h_q):
    w = dataclasses.replace(W.get_workload("sparse"), kv=kv, batch=2, seqlens=[500, 3000], h_q=h_q, topk=192,
                            seed=h_q + 11)
    inp = W.make_inputs(w)
    _check(inp, f"sparse {kv} h_q={h_q}")
