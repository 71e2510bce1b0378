"""GPU parity of token-sparse decoding (mla_decode_sparse) against the oracle,
and the bit-exact handling of ignored (-1) index slots."""
import dataclasses

import numpy as np
import pytest
import torch

import head_latent_attention_get_b200 as M
from head_latent_attention_get_b200 import _capi as C
from tests import gpu_helpers as G
from workloads import mla_workloads as W

pytestmark = pytest.mark.gpu


def _sparse(batch, seqlens, s_q, h_q, topk, neg_frac=0.05, seed=1):
    w = dataclasses.replace(W.get_workload("sparse"), batch=batch, seqlens=seqlens, s_q=s_q, h_q=h_q,
                            topk=topk, neg_frac=neg_frac, seed=seed)
    return W.make_inputs(w)


def _run(inp, **kw):
    out, lse, r = G.run_gpu(inp, runner_kwargs=kw)
    return out, lse, r


@pytest.mark.parametrize("seqlens,s_q,h_q,topk", [
    ([300, 1000], 1, 16, 128),
    ([300, 1000], 1, 64, 192),          # last 128-slot tile is half full
    ([4000, 129, 2000], 2, 32, 256),    # s_q = 2: one unit per (request, query token)
    ([5000, 3000], 1, 128, 512),        # 128 rows: CTA pairs
    ([300, 1000, 70], 1, 128, 192),     # CTA pairs, half-full last tile, odd tile count
    ([4000, 129], 2, 96, 256),          # CTA pairs with 32 rows in the odd CTA, s_q = 2
])
def test_sparse_vs_oracle(seqlens, s_q, h_q, topk):
    inp = _sparse(len(seqlens), seqlens, s_q, h_q, topk, seed=sum(seqlens) + topk)
    out, lse, r = _run(inp)
    ref_o, ref_l = G.oracle_for(inp)
    G.compare(out, lse, ref_o, ref_l, f"sparse {seqlens} s_q={s_q} h_q={h_q} topk={topk}")
    assert r.status()[0] == C.MLA_OK


@pytest.mark.parametrize("h_q", [32, 128])  # 128 rows run on CTA pairs
def test_sparse_duplicates_and_all_ignored_rows(h_q):
    inp = _sparse(2, [700, 700], 1, h_q, 128, neg_frac=0.0, seed=9)
    idx = inp.indices
    idx[0, 0, 64:] = idx[0, 0, :64]        # every key of request 0 counted twice
    idx[1, 0, :] = -1                      # request 1: empty key set -> out 0, lse -inf
    out, lse, r = _run(inp)
    ref_o, ref_l = G.oracle_for(inp)
    G.compare(out, lse, ref_o, ref_l, "duplicates / all -1")
    assert np.all(out[1] == 0) and np.all(np.isneginf(lse[1]))
    assert r.status()[0] == C.MLA_OK


@pytest.mark.parametrize("h_q", [16, 128])
def test_out_of_range_indices_are_ignored_and_reported(h_q):
    inp = _sparse(2, [500, 300], 1, h_q, 128, seed=3)
    inp.indices[0, 0, 5] = 500             # == seqlen: out of range
    inp.indices[1, 0, 7] = -5              # negative but not -1
    out, lse, r = _run(inp)
    code, bits = r.status()
    assert code == C.MLA_ERR_DEVICE_BOUNDS and bits & C.MLA_DEVICE_STATUS_BOUNDS
    ref_o, ref_l = G.oracle_for(inp)       # the oracle ignores them too
    G.compare(out, lse, ref_o, ref_l, "out-of-range ignored")


@pytest.mark.parametrize("h_q", [64, 128])
def test_ignored_slots_are_bit_exact(h_q):
    """(i) NaN in every cache row that no valid index reaches changes no bit;
    (ii) appending a tile of -1 slots changes no bit."""
    inp = _sparse(2, [900, 2000], 1, h_q, 256, neg_frac=0.1, seed=21)
    base_o, base_l, _ = _run(inp, num_sm_parts=2)
    # (i) poison all unreferenced tokens of both requests
    pois = dataclasses.replace(inp, kcache=inp.kcache.clone())
    bt = inp.block_table.numpy()
    for b, L in enumerate(inp.cache_seqlens.tolist()):
        used = set(int(x) for x in inp.indices[b, 0].tolist() if x >= 0)
        for t in range(L):
            if t not in used:
                pois.kcache[bt[b, t // 64], t % 64] = float("nan")
    po, pl, _ = _run(pois, num_sm_parts=2)
    assert np.array_equal(po.view(np.uint32), base_o.view(np.uint32))
    assert np.array_equal(pl.view(np.uint32), base_l.view(np.uint32))
    # (ii) an extra tile of ignored slots (same single-part schedule: no splits)
    one_o, one_l, _ = _run(inp, num_sm_parts=1)
    ext = dataclasses.replace(inp, workload=dataclasses.replace(inp.workload, topk=384),
                              indices=torch.cat([inp.indices, torch.full((2, 1, 128), -1, dtype=torch.int32)], -1))
    eo, el, _ = _run(ext, num_sm_parts=1)
    assert np.array_equal(eo.view(np.uint32), one_o.view(np.uint32))
    assert np.array_equal(el.view(np.uint32), one_l.view(np.uint32))


@pytest.mark.parametrize("h_q", [64, 128])
def test_all_positions_in_order_equal_dense(h_q):
    w = dataclasses.replace(W.get_workload("tiny"), batch=2, seqlens=[300, 190], h_q=h_q, seed=5)
    dense = W.make_inputs(w)
    idx = torch.full((2, 1, 320), -1, dtype=torch.int32)
    for b, L in enumerate([300, 190]):
        idx[b, 0, :L] = torch.arange(L, dtype=torch.int32)
    sp = dataclasses.replace(dense, workload=dataclasses.replace(w, topk=320), indices=idx)
    do, dl, _ = _run(dense, num_sm_parts=1)
    so, sl, _ = _run(sp, num_sm_parts=1)
    assert np.array_equal(so.view(np.uint32), do.view(np.uint32))
    assert np.array_equal(sl.view(np.uint32), dl.view(np.uint32))


def test_sparse_full_size_every_request():
    """32 requests x 128 heads, 32768-token caches, topk 2048 with 5% -1."""
    inp = W.make_inputs(W.get_workload("sparse"))
    out, lse, r = _run(inp)
    G.compare_full(inp, out, lse, "sparse")
    assert r.status()[0] == C.MLA_OK
