"""GPU parity of token-sparse decoding over the FP8 token-record cache (the
FP8 token-sparse combination of the pages' sparse-decoding figures) against
the oracle run on the same dequantised values, and the bit-exact handling of
ignored (-1) index slots."""
import dataclasses

import numpy as np
import pytest
import torch

from head_latent_attention_get_b200 import _capi as C
from tests import gpu_helpers as G
from workloads import mla_workloads as W

pytestmark = pytest.mark.gpu


def _fp8_sparse(batch, seqlens, s_q, h_q, topk, neg_frac=0.05, seed=1):
    w = dataclasses.replace(W.get_workload("sparse"), batch=batch, seqlens=seqlens, s_q=s_q, h_q=h_q,
                            topk=topk, neg_frac=neg_frac, seed=seed, kv="fp8")
    return W.make_inputs(w)


def _run(inp, **kw):
    return G.run_gpu(inp, runner_kwargs=kw)


@pytest.mark.parametrize("seqlens,s_q,h_q,topk,parts", [
    ([300, 1000], 1, 16, 128, None),
    ([300, 1000], 1, 64, 192, None),          # last 128-slot tile half full
    ([4000, 129, 2000], 2, 32, 256, 5),       # s_q = 2, split units
    ([5000, 3000], 1, 128, 512, None),        # 128 rows: two row groups per part
    ([300, 1000, 70], 1, 128, 192, 2),
])
def test_fp8_sparse_vs_oracle(seqlens, s_q, h_q, topk, parts):
    inp = _fp8_sparse(len(seqlens), seqlens, s_q, h_q, topk, seed=sum(seqlens) + topk)
    out, lse, r = _run(inp, num_sm_parts=parts)
    ref_o, ref_l = G.oracle_for(inp)
    G.compare(out, lse, ref_o, ref_l, f"fp8 sparse {seqlens} s_q={s_q} h_q={h_q} topk={topk}", inp=inp)
    assert r.status()[0] == C.MLA_OK


def test_fp8_sparse_with_sink_and_empty_rows():
    inp = W.with_sink(_fp8_sparse(2, [700, 700], 1, 64, 128, neg_frac=0.0, seed=9), seed=2)
    inp.indices[1, 0, :] = -1                 # empty key set: out 0, lse = sink
    out, lse, r = _run(inp)
    ref_o, ref_l = G.oracle_for(inp)
    G.compare(out, lse, ref_o, ref_l, "fp8 sparse sink", inp=inp)
    assert np.all(out[1] == 0) and np.array_equal(lse[1, 0], inp.sink.numpy())


@pytest.mark.parametrize("h_q", [64, 128])
def test_fp8_sparse_ignored_slots_are_bit_exact(h_q):
    """(i) NaN in every byte of every token record no valid index reaches
    (codes, scales and RoPE dims) changes no bit; (ii) a tile of -1 slots
    appended changes no bit."""
    inp = _fp8_sparse(2, [900, 2000], 1, h_q, 256, neg_frac=0.1, seed=21)
    base_o, base_l, _ = _run(inp, num_sm_parts=2)
    pois = dataclasses.replace(inp, kcache=inp.kcache.clone())
    bt = inp.block_table.numpy()
    for b, L in enumerate(inp.cache_seqlens.tolist()):
        used = set(int(x) for x in inp.indices[b, 0].tolist() if x >= 0)
        for t in range(L):
            if t not in used:
                pois.kcache[bt[b, t // 64], t % 64] = 0xFF   # e4m3 NaN, fp32 NaN, bf16 NaN
    po, pl, _ = _run(pois, num_sm_parts=2)
    assert np.array_equal(po.view(np.uint32), base_o.view(np.uint32))
    assert np.array_equal(pl.view(np.uint32), base_l.view(np.uint32))
    one_o, one_l, _ = _run(inp, num_sm_parts=1)
    ext = dataclasses.replace(inp, workload=dataclasses.replace(inp.workload, topk=384),
                              indices=torch.cat([inp.indices, torch.full((2, 1, 128), -1, dtype=torch.int32)], -1))
    eo, el, _ = _run(ext, num_sm_parts=1)
    assert np.array_equal(eo.view(np.uint32), one_o.view(np.uint32))
    assert np.array_equal(el.view(np.uint32), one_l.view(np.uint32))


@pytest.mark.parametrize("h_q", [64, 128])
def test_fp8_all_positions_in_order_match_fp8_dense(h_q):
    """Indices that list every position in order select the dense key set, so
    the token-sparse path and the paged FP8 kernel must both reproduce the
    oracle's dense result. The two kernels tile the keys differently (128-slot
    tiles against 64-token pages), so they agree to rounding, not bitwise."""
    w = dataclasses.replace(W.get_workload("fp8"), batch=2, seqlens=[300, 190], h_q=h_q, seed=5)
    dense = W.make_inputs(w)
    idx = torch.full((2, 1, 320), -1, dtype=torch.int32)
    for b, L in enumerate([300, 190]):
        idx[b, 0, :L] = torch.arange(L, dtype=torch.int32)
    sp = dataclasses.replace(dense, workload=dataclasses.replace(w, topk=320), indices=idx)
    do, dl, _ = _run(dense, num_sm_parts=1)
    so, sl, _ = _run(sp, num_sm_parts=1)
    ref_o, ref_l = G.oracle_for(dense)
    G.compare(do, dl, ref_o, ref_l, f"fp8 dense h_q={h_q}")
    G.compare(so, sl, ref_o, ref_l, f"fp8 all positions h_q={h_q}")


def test_fp8_sparse_full_size_every_request():
    """32 requests x 128 heads, 32768-token FP8 caches, topk 2048, 5% -1."""
    w = dataclasses.replace(W.get_workload("sparse"), kv="fp8")
    inp = W.make_inputs(w)
    out, lse, r = _run(inp)
    G.compare_full(inp, out, lse, "fp8 sparse")
    assert r.status()[0] == C.MLA_OK
