"""GPU parity of paged decoding with more than 128 query rows per request
(q_len up to six query tokens per request, as in the FlashInfer README's
DeepSeek-V4 geometry, or more than 128 heads): the rows of a request are cut
into equal row blocks of at most 128 rows that each read the whole key set."""
import dataclasses

import numpy as np
import pytest

import head_latent_attention_get_b200 as M
from head_latent_attention_get_b200 import _capi as C
from tests import gpu_helpers as G
from workloads import mla_workloads as W

pytestmark = pytest.mark.gpu


def _dense(name="tiny", **over):
    return dataclasses.replace(W.get_workload(name), **over)


def _check(inp, where, **kw):
    out, lse, r = G.run_gpu(inp, runner_kwargs=kw)
    ref_o, ref_l = G.oracle_for(inp)
    G.compare(out, lse, ref_o, ref_l, where, inp=inp)
    assert r.status()[0] == C.MLA_OK
    return out, lse, r


@pytest.mark.parametrize("lens,s_q,h_q,causal,blocks", [
    ([1, 5, 64, 700, 3000], 6, 64, True, (3, 128)),     # six query tokens x 64 heads: CTA pairs
    ([2, 129, 2000], 3, 64, True, (2, 96)),             # 96-row blocks: 32 rows in the odd CTA
    ([300, 4000], 5, 32, True, (2, 80)),
    ([1000, 70], 4, 128, True, (4, 128)),
    ([1500, 64, 3], 1, 256, False, (2, 128)),           # 256 heads, one query token
    ([700, 2, 1300], 3, 43, True, (3, 43)),             # 43-row blocks: row-group kernel
    ([6, 900], 6, 16, True, (1, 96)),                   # 96 rows: one unit per request
])
def test_row_blocks_vs_oracle(lens, s_q, h_q, causal, blocks):
    assert M.mla_decode_geometry(s_q, h_q, 1, 0) == blocks
    w = _dense(batch=len(lens), seqlens=lens, s_q=s_q, h_q=h_q, causal=causal, seed=3 + sum(lens))
    inp = W.make_inputs(w, poison_tail=True, extra_pages=2)
    _check(inp, f"{lens} s_q={s_q} h_q={h_q}")


@pytest.mark.parametrize("parts", [1, 3, 74, 148])
def test_row_blocks_split_counts(parts):
    w = _dense(batch=3, seqlens=[2500, 130, 6000], s_q=6, h_q=64, causal=True, seed=19)
    inp = W.make_inputs(w, poison_tail=True)
    _check(inp, f"parts={parts}", num_sm_parts=parts)


def test_row_blocks_with_sink():
    """The sink's head follows the row through the blocks (row r of unit u is
    head (u*rows + r) mod h_q), split and unsplit."""
    w = _dense(batch=3, seqlens=[4, 900, 3000], s_q=3, h_q=64, causal=True, seed=23)
    inp = W.with_sink(W.make_inputs(w, poison_tail=True), seed=5)
    for parts in (None, 7):
        _check(inp, f"sink parts={parts}", num_sm_parts=parts)


@pytest.mark.parametrize("s_q,h_q", [(6, 64), (3, 48)])
def test_row_blocks_fp8(s_q, h_q):
    w = _dense("fp8", batch=2, seqlens=[700, 2100], s_q=s_q, h_q=h_q, causal=True, seed=29 + s_q)
    inp = W.make_inputs(w, poison_tail=True, extra_pages=1)
    _check(inp, f"fp8 s_q={s_q} h_q={h_q}")


def test_row_blocks_larger_batch_every_request():
    """64 requests x 6 query tokens x 64 heads, 4096 tokens each; every
    request checked against the oracle."""
    w = _dense(batch=64, seqlens=[4096] * 64, s_q=6, h_q=64, causal=True, seed=31)
    inp = W.make_inputs(w)
    out, lse, _ = G.run_gpu(inp)
    G.compare_full(inp, out, lse, "s_q=6 h_q=64", few_keys=True)
