"""GPU parity of the per-head attention sink (mla_decode_args.sink) against the
oracle, on every kernel that writes outputs: the row-group decode (BF16 and
FP8 caches, paged and sparse), the CTA-pair decode (128 rows, paged and
sparse), and the combine (split units, units with no split at all)."""
import dataclasses

import numpy as np
import pytest
import torch

import head_latent_attention_get_b200 as M
from head_latent_attention_get_b200 import _capi as C
from oracle import mla_oracle as O
from tests import gpu_helpers as G
from workloads import mla_workloads as W

pytestmark = pytest.mark.gpu


def _dense(name="tiny", **over):
    return dataclasses.replace(W.get_workload(name), **over)


def _sparse(batch, seqlens, s_q, h_q, topk, neg_frac=0.05, seed=1):
    return dataclasses.replace(W.get_workload("sparse"), batch=batch, seqlens=seqlens, s_q=s_q, h_q=h_q,
                               topk=topk, neg_frac=neg_frac, seed=seed)


def _check(inp, where, **kw):
    out, lse, r = G.run_gpu(inp, runner_kwargs=kw)
    ref_o, ref_l = G.oracle_for(inp)
    info = G.compare(out, lse, ref_o, ref_l, where, inp=inp)
    assert r.status()[0] == C.MLA_OK
    return out, lse, info


@pytest.mark.parametrize("lens,s_q,h_q,causal,parts", [
    ([1, 63, 65, 300], 1, 16, False, None),       # row-group kernel, 16 rows, unsplit
    ([900, 4000, 130], 1, 64, False, 7),          # split units: the sink joins in the combine
    ([0, 1, 129, 4000], 2, 16, True, None),       # seqlen 0 unit (combine) + causal row with no key
    ([700, 1500], 1, 128, False, None),           # CTA pairs, unsplit
    ([700, 5000, 3], 1, 128, False, 3),           # CTA pairs, split
    ([3000, 1], 2, 64, True, 148),                # CTA pairs (2 x 64 rows), causal
])
def test_sink_dense_vs_oracle(lens, s_q, h_q, causal, parts):
    w = _dense(batch=len(lens), seqlens=lens, s_q=s_q, h_q=h_q, causal=causal, seed=5 + sum(lens))
    inp = W.with_sink(W.make_inputs(w, poison_tail=True, extra_pages=2), seed=sum(lens))
    out, lse, _ = _check(inp, f"sink {lens} s_q={s_q} h_q={h_q}", num_sm_parts=parts)
    for b, L in enumerate(lens):
        if L == 0:                                  # empty key set: out 0, lse = sink of the head
            assert np.all(out[b] == 0)
            assert np.array_equal(lse[b], np.broadcast_to(inp.sink.numpy(), lse[b].shape))


@pytest.mark.parametrize("lens,h_q", [([70, 129], 16), ([1000, 2000], 128)])
def test_sink_fp8_vs_oracle(lens, h_q):
    w = _dense("fp8", batch=len(lens), seqlens=lens, h_q=h_q, seed=41 + sum(lens))
    inp = W.with_sink(W.make_inputs(w, poison_tail=True, extra_pages=1), seed=3)
    _check(inp, f"sink fp8 {lens}")


@pytest.mark.parametrize("seqlens,s_q,h_q,topk,parts", [
    ([300, 1000], 1, 16, 128, None),
    ([4000, 129, 2000], 2, 32, 256, 5),
    ([5000, 3000], 1, 128, 512, None),            # CTA pairs
    ([300, 1000, 70], 1, 128, 192, 2),            # CTA pairs, split
])
def test_sink_sparse_vs_oracle(seqlens, s_q, h_q, topk, parts):
    inp = W.with_sink(W.make_inputs(_sparse(len(seqlens), seqlens, s_q, h_q, topk, seed=topk + 1)), seed=topk)
    _check(inp, f"sink sparse {seqlens} h_q={h_q}", num_sm_parts=parts)


@pytest.mark.parametrize("h_q", [32, 128])
def test_sink_all_ignored_rows(h_q):
    """A sparse row whose indices are all -1 has an empty key set: out 0 and
    lse = sink of its head, exactly."""
    inp = W.with_sink(W.make_inputs(_sparse(2, [700, 700], 1, h_q, 128, neg_frac=0.0, seed=9)), seed=1)
    inp.indices[1, 0, :] = -1
    out, lse, _ = _check(inp, "sink all -1")
    assert np.all(out[1] == 0) and np.array_equal(lse[1, 0], inp.sink.numpy())


@pytest.mark.parametrize("h_q,parts", [(16, None), (64, 7), (128, None), (128, 3)])
def test_minus_inf_sink_changes_no_bit(h_q, parts):
    w = _dense(batch=3, seqlens=[900, 4000, 130], h_q=h_q, seed=77)
    inp = W.make_inputs(w, poison_tail=True)
    o0, l0, _ = G.run_gpu(inp, runner_kwargs={"num_sm_parts": parts})
    inp_s = dataclasses.replace(inp, sink=torch.full((h_q,), -float("inf")))
    o1, l1, _ = G.run_gpu(inp_s, runner_kwargs={"num_sm_parts": parts})
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)


def test_dominant_sink():
    """sigma far above every score: the output vanishes and lse -> sigma
    (no overflow in the fold)."""
    w = _dense(batch=2, seqlens=[500, 3000], h_q=64, seed=8)
    inp = W.make_inputs(w)
    inp = dataclasses.replace(inp, sink=torch.full((64,), 80.0))
    out, lse, _ = _check(inp, "dominant sink", num_sm_parts=7)
    assert np.abs(out).max() < 1e-6 and np.allclose(lse, 80.0, atol=1e-4)


def test_combine_sink_matches_oracle_merge():
    rng = np.random.default_rng(6)
    U, h_q, s_q, parts = 3, 8, 2, 4
    R = s_q * h_q
    n_splits = [3, 1, 0]            # unit 1 untouched (single split), unit 2 empty
    ptr = np.concatenate([[0], np.cumsum(n_splits)]).astype(np.int32)
    ws_bytes = M.mla_workspace_size(U, s_q, h_q, 1, 0, parts)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    q = rng.standard_normal((R, 576))
    k = rng.standard_normal((300, 576))
    sink = (rng.standard_normal(h_q) + 1.0).astype(np.float32)
    cuts = [0, 64, 64, 300]           # the middle split has no keys
    parts_o, parts_l = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        o, l = O.attend(q, k[a:b], 1 / 24)
        parts_o.append(o)
        parts_l.append(l)
    max_splits = U + parts
    lse_off = 256
    o_off = -(-(lse_off + max_splits * R * 4) // 256) * 256
    lse_buf = np.zeros((max_splits, R), np.float32)
    o_buf = np.zeros((max_splits, R, 512), np.float32)
    for s in range(3):
        lse_buf[s] = parts_l[s]
        o_buf[s] = parts_o[s]
    ws[lse_off:lse_off + lse_buf.nbytes] = torch.from_numpy(lse_buf.view(np.uint8).ravel()).cuda()
    ws[o_off:o_off + o_buf.nbytes] = torch.from_numpy(o_buf.view(np.uint8).ravel()).cuda()
    out = torch.full((U * R, 512), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((U * R,), 7.0, dtype=torch.float32, device="cuda")
    sink_d = torch.from_numpy(sink).cuda()
    M.mla_combine_sink(ws, ws_bytes, torch.from_numpy(ptr).cuda(), U, R, parts, h_q, sink_d, out, lse)
    torch.cuda.synchronize()
    row_sink = np.tile(sink.astype(np.float64), s_q)           # head of row r is r % h_q
    ref_o, ref_l = O.combine(np.stack(parts_o), np.stack(parts_l), sink=row_sink)
    G.compare(out[:R].float().cpu().numpy(), lse[:R].cpu().numpy(), ref_o, ref_l, "combine sink")
    assert torch.all(out[R:2 * R] == 7.0) and torch.all(lse[R:2 * R] == 7.0)      # single split: untouched
    assert torch.all(out[2 * R:] == 0)                                              # empty unit
    assert np.array_equal(lse[2 * R:].cpu().numpy(), row_sink.astype(np.float32))
