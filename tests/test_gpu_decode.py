"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle."""
import dataclasses

import numpy as np
import pytest
import torch

import head_latent_attention_get_b200 as M
from head_latent_attention_get_b200 import _capi as C
from oracle import mla_oracle as O
from tests import gpu_helpers as G
from tests import sched_checks as S
from workloads import mla_workloads as W

pytestmark = pytest.mark.gpu


def _dense(name="tiny", **over):
    return dataclasses.replace(W.get_workload(name), **over)


# ------------------------------------------------------------------ scheduler
@pytest.mark.parametrize("lens,s_q,h_q,topk,parts", [
    ([70, 129], 1, 16, 0, None), ([4096] * 64, 1, 128, 0, None), ([0, 5, 0, 300, 9000], 2, 16, 0, None),
    (list(range(0, 30000, 97)), 1, 64, 0, None), ([32768] * 32, 1, 128, 2048, None),   # equal units, 2 pieces each
    ([100] * 5, 2, 32, 128, None),
    ([(37 * i) % 5000 for i in range(13000)], 1, 16, 0, None),  # more units than the shared-memory prefix holds
    ([3000] * 5000, 1, 128, 0, 10003),                          # the same, equal units, 2 pieces each
    ([4096] * 64, 6, 64, 0, None)])                             # three row-block units per request
def test_metadata_device_matches_host_twin(lens, s_q, h_q, topk, parts):
    B = len(lens)
    parts = parts or M.mla_get_num_sm_parts(0, s_q, h_q, 1, topk)
    U = B * M.mla_decode_geometry(s_q, h_q, 1, topk)[0]
    md_h = np.zeros(parts * 8, np.int32)
    ns_h = np.zeros(U + 1, np.int32)
    lens_np = np.asarray(lens, np.int32)
    assert M.mla_get_metadata_host(lens_np, B, s_q, h_q, 1, topk, parts, md_h, ns_h) == 0
    md_d = torch.full((parts * 8,), -7, dtype=torch.int32, device="cuda")
    ns_d = torch.full((U + 1,), -7, dtype=torch.int32, device="cuda")
    M.mla_get_metadata(torch.from_numpy(lens_np).cuda(), B, s_q, h_q, 1, topk, parts, md_d, ns_d)
    torch.cuda.synchronize()
    assert np.array_equal(md_d.cpu().numpy(), md_h) and np.array_equal(ns_d.cpu().numpy(), ns_h)
    S.check_schedule(md_h, ns_h, lens, B, s_q, topk, parts, h_q=h_q)


# ------------------------------------------------------------------ combine
def test_combine_matches_oracle_merge():
    rng = np.random.default_rng(5)
    U, R, parts = 3, 16, 4
    n_splits = [3, 1, 0]            # unit 1 untouched (single split), unit 2 empty
    ptr = np.concatenate([[0], np.cumsum(n_splits)]).astype(np.int32)
    ws_bytes = M.mla_workspace_size(U, 1, R, 1, 0, parts)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    q = rng.standard_normal((R, 576))
    k = rng.standard_normal((300, 576))
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
    M.mla_combine(ws, ws_bytes, torch.from_numpy(ptr).cuda(), U, R, parts, out, lse)
    torch.cuda.synchronize()
    ref_o, ref_l = O.combine(np.stack(parts_o), np.stack(parts_l))
    G.compare(out[:R].float().cpu().numpy(), lse[:R].cpu().numpy(), ref_o, ref_l, "combine")
    assert torch.all(out[R:2 * R] == 7.0) and torch.all(lse[R:2 * R] == 7.0)      # single split: untouched
    assert torch.all(out[2 * R:] == 0) and torch.all(torch.isneginf(lse[2 * R:]))  # empty unit


# ------------------------------------------------------------------ dense bf16
def test_tiny_workload_full():
    inp = W.make_inputs(W.get_workload("tiny"), poison_tail=True, extra_pages=2)
    out, lse, _ = G.run_gpu(inp)
    ref_o, ref_l = G.oracle_for(inp)
    G.compare(out, lse, ref_o, ref_l, "tiny")


@pytest.mark.parametrize("lens,s_q,h_q,causal", [
    ([1, 63, 64, 65], 1, 16, False),
    ([127, 128, 129, 255, 256, 257], 1, 32, False),
    ([300, 1000, 2049], 1, 64, False),
    ([700, 1500], 1, 128, False),
    ([1, 2, 65, 129, 4000], 2, 16, True),
    ([5, 300], 2, 32, True),
    ([0, 100, 0], 1, 16, False),
    ([3000], 2, 64, True),
])
def test_dense_shapes_vs_oracle(lens, s_q, h_q, causal):
    w = _dense(batch=len(lens), seqlens=lens, s_q=s_q, h_q=h_q, causal=causal, seed=11 + sum(lens))
    inp = W.make_inputs(w, poison_tail=True, extra_pages=3)
    out, lse, r = G.run_gpu(inp)
    ref_o, ref_l = G.oracle_for(inp)
    G.compare(out, lse, ref_o, ref_l, f"{lens} s_q={s_q} h_q={h_q}")
    assert r.status()[0] == C.MLA_OK


@pytest.mark.parametrize("kv,parts", [("bf16", 1), ("bf16", 2), ("bf16", 7), ("bf16", 148),
                                      ("fp8", 1), ("fp8", 3), ("fp8", 7), ("fp8", 148)])
def test_split_counts_do_not_change_results(kv, parts):
    """Pieces that start and end inside a request (odd page counts, a last
    half tile, one-page requests) give the same results for any split count."""
    w = _dense(batch=3, seqlens=[900, 4000, 130], h_q=64, seed=77, kv=kv)
    inp = W.make_inputs(w, poison_tail=True)
    out, lse, _ = G.run_gpu(inp, runner_kwargs={"num_sm_parts": parts})
    ref_o, ref_l = G.oracle_for(inp)
    G.compare(out, lse, ref_o, ref_l, f"parts={parts}")


def test_dsv3_full_size_every_request():
    """64 requests x 128 heads x 4096 tokens: every output row against the oracle."""
    inp = W.make_inputs(W.get_workload("dsv3"))
    out, lse, r = G.run_gpu(inp)
    G.compare_full(inp, out, lse, "dsv3")
    assert r.status()[0] == C.MLA_OK


def test_mtp_full_size_every_request():
    """128 requests, s_q=2 causal, 16 heads, U[1024,16384] plus one 65536."""
    inp = W.make_inputs(W.get_workload("mtp"))
    out, lse, r = G.run_gpu(inp)
    G.compare_full(inp, out, lse, "mtp")
    assert r.status()[0] == C.MLA_OK


# ------------------------------------------------------------------ fp8 cache
@pytest.mark.parametrize("lens,h_q", [([70, 129], 16), ([1, 64, 300], 64), ([1000, 2000], 128)])
def test_fp8_vs_oracle_on_dequantised_values(lens, h_q):
    w = _dense("fp8", batch=len(lens), seqlens=lens, h_q=h_q, seed=31 + sum(lens))
    inp = W.make_inputs(w, poison_tail=True, extra_pages=1)
    out, lse, _ = G.run_gpu(inp)
    ref_o, ref_l = G.oracle_for(inp)
    G.compare(out, lse, ref_o, ref_l, f"fp8 {lens}")


def test_fp8_full_size_every_request():
    """64 requests x 64 heads x 8192 FP8 tokens, against the oracle on the
    dequantised values."""
    inp = W.make_inputs(W.get_workload("fp8"))
    out, lse, r = G.run_gpu(inp)
    G.compare_full(inp, out, lse, "fp8")
    assert r.status()[0] == C.MLA_OK


# ------------------------------------------------------------------ device status
def test_bounds_status_without_fault():
    w = _dense(batch=2, seqlens=[130, 64])
    inp = W.make_inputs(w)
    inp.block_table[0, 1] = inp.num_pages + 5          # out-of-range page id
    out, lse, r = G.run_gpu(inp)
    code, bits = r.status()
    assert code == C.MLA_ERR_DEVICE_BOUNDS and bits & C.MLA_DEVICE_STATUS_BOUNDS
    # the request that is in range is still exact
    sub = G.restrict(inp, [1])
    ref_o, ref_l = G.oracle_for(sub)
    G.compare(out[1:], lse[1:], ref_o, ref_l, "unaffected request")


@pytest.mark.parametrize("kv", ["bf16", "fp8", "nvfp4"])
def test_timeout_status_and_context_survives(kv):
    """Scores withheld from the softmax: every bounded wait gives up, the
    status word says so and the next call on the same context is exact (the
    bf16 row-group kernel and the page kernel with FP8 and NVFP4 pages)."""
    over = {"scale": 512 ** -0.5} if kv == "nvfp4" else {}
    inp = W.make_inputs(_dense("tiny", kv=kv, **over))
    _, _, r = G.run_gpu(inp, runner_kwargs={"timeout_ns": 20_000_000,
                                            "debug_flags": C.MLA_DEBUG_WITHHOLD_SCORES})
    code, bits = r.status()
    assert code == C.MLA_ERR_DEVICE_TIMEOUT and bits & C.MLA_DEVICE_STATUS_TIMEOUT
    # the context is still usable: a normal call succeeds afterwards
    out, lse, r2 = G.run_gpu(inp)
    ref_o, ref_l = G.oracle_for(inp)
    G.compare(out, lse, ref_o, ref_l, "after timeout")
    assert r2.status()[0] == C.MLA_OK


def test_combine_strides_over_more_items_than_blocks():
    """400 requests x 64 heads of mixed lengths: 400 units x 16 row chunks =
    6400 combine items for a grid of at most 8 x 148 blocks, with many units
    split across parts; every request against the oracle."""
    rng = np.random.default_rng(404)
    lens = [int(x) for x in rng.integers(1, 3000, size=400)]
    w = _dense(batch=400, seqlens=lens, h_q=64, seed=404)
    inp = W.make_inputs(w, poison_tail=True)
    out, lse, r = G.run_gpu(inp)
    ns = r.num_splits.cpu().numpy()
    assert (np.diff(ns) > 1).sum() > 50            # many units are split
    G.compare_full(inp, out, lse, "400 requests, 6400 combine items")
    assert r.status()[0] == C.MLA_OK


@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_repeated_calls_on_one_workspace_are_identical(kv):
    """Five calls on one workspace, with split requests and empty ones among
    them, give the same bits each time (nothing a call leaves in the
    workspace changes the next)."""
    w = _dense(batch=5, seqlens=[3000, 0, 129, 5000, 0], h_q=64, seed=808, kv=kv)
    inp = W.make_inputs(w, poison_tail=True)
    out, lse, r = G.run_gpu(inp, runner_kwargs={"num_sm_parts": 7})
    assert (np.diff(r.num_splits.cpu().numpy()) > 1).any()
    G.compare_full(inp, out, lse, f"{kv} first call")
    for _ in range(4):
        o2, l2 = r.run()
        torch.cuda.synchronize()
        assert torch.equal(o2.float().cpu(), torch.from_numpy(out))
        assert np.array_equal(l2.cpu().numpy().view(np.uint32), lse.view(np.uint32))
    assert r.status()[0] == C.MLA_OK
